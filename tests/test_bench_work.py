"""The bench's algorithmic work counts, pinned to closed forms and to brute force.

Every TFLOP/s and GB/s the bench prints divides one of these counts by a measured time,
so a wrong count would skew every figure.  The FLOP convention counts only the visible
(query, key) pairs, 4 * 128 flops per pair and query head (Q K^T and P V); the byte
convention of decode counts the visible K and V rows once plus the new token's q, k, v,
gate and output.  The causal and window counts follow from the masks of the English page
("Two attention paths in one decoder": keys t-511 .. t in a local layer, 0 .. t in a
global one); the cache size per token from its "KV memory" section (2 x 8 x 128 values
per token and layer).
"""
import numpy as np
import pytest

import bench
import workloads as wl


def _brute_pairs(T, window):
    t = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = j <= t
    if window is not None:
        vis &= t - j <= window - 1
    return int(vis.sum())


@pytest.mark.parametrize("T", [1, 2, 7, 129, 511, 512, 513, 1030])
@pytest.mark.parametrize("window", [None, 1, 4, 512])
def test_visible_pairs_equal_brute_force(T, window):
    assert wl.visible_pairs(T, window) == _brute_pairs(T, window)


def test_batched_prefill_flops_closed_forms():
    T = 8192
    # global: T (T + 1) / 2 pairs per sequence; local: the first 512 rows see t + 1 keys,
    # every later row 512
    assert wl.visible_pairs(T, None) == T * (T + 1) // 2 == 33_558_528
    assert wl.visible_pairs(T, 512) == 512 * 513 // 2 + (T - 512) * 512 == 4_063_488
    assert bench.HEAD_FLOPS_PER_PAIR == 4 * 128 * 48
    g = bench.prefill_flops(4, T, wl.GLOBAL)
    loc = bench.prefill_flops(4, T, wl.LOCAL)
    assert g == 4 * 33_558_528 * 24_576
    assert loc == 4 * 4_063_488 * 24_576
    assert abs(g / 1e12 - 3.299) < 5e-4 and abs(loc / 1e12 - 0.3995) < 5e-4


def test_long_global_prefill_flops():
    T = 131_072
    assert bench.prefill_flops(1, T, wl.GLOBAL) == T * (T + 1) // 2 * 24_576
    assert abs(bench.prefill_flops(1, T, wl.GLOBAL) / 1e12 - 211.1) < 0.05


def test_decode_bytes_at_one_million():
    """The 52-layer step at context 2^20: nine global layers read every cached row, the 43
    local layers their 512-slot rings; 4096 bytes per row in bf16, 2048 in FP8."""
    ctx = [1 << 20]
    per_global = bench.decode_kv_bytes(ctx, wl.GLOBAL)
    per_local = bench.decode_kv_bytes(ctx, wl.LOCAL)
    io = 2 * (3 * 48 * 128 + 2 * 8 * 128)
    assert per_global == (1 << 20) * 4096 + io
    assert per_local == 512 * 4096 + io
    kv = 9 * (1 << 20) * 4096 + 43 * 512 * 4096
    assert kv == 38_744_883_200            # 36.08 GiB of K and V per step
    assert 9 * per_global + 43 * per_local == kv + 52 * io
    assert bench.decode_kv_bytes(ctx, wl.GLOBAL, elem_bytes=1) == (1 << 20) * 2048 + io


def test_layer_schedule_matches_the_bench_step():
    kinds = [wl.layer_kind(i) for i in range(1, wl.N_LAYERS + 1)]
    assert kinds.count(wl.GLOBAL) == 9 and kinds.count(wl.LOCAL) == 43
