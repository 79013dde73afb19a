"""Chunked prefill over FP8 E4M3 caches (beam_attn_prefill_chunk_fp8) through the
C ABI, against the fp64 oracle (oracle.prefill_chunk_rows_fp8).

Cache codes before the call are seeded E4M3 codes given to both sides.  The chunk's
new keys and values are written as codes first and read back with the cached ones
(English page, "KV memory": the FP8 cache; a continuing call reads the earlier keys
from the cache).  Outputs use the parity bar of the other GPU tests; the written
codes are checked as in the FP8 append test (value codes bit for bit, key codes
within one E4M3 step, every other code unchanged).  Scales are not powers of two,
as an amax / 448 rule gives.
"""
import numpy as np
import pytest

import workloads as wl
from test_gpu_fp8 import _codes_close
from test_gpu_parity import assert_close, dev, env, host_bits, oracle_params  # noqa: F401

pytestmark = pytest.mark.gpu

K_SCALE, V_SCALE = 0.0173, 3.7


def _codes(shape, seed, tag, scale):
    return wl.normal_e4m3(shape, seed, tag, scale)


def run_chunk_fp8(torch, beam, ci, params, kc0, vc0, ks, vs, status=None, kc=None, vc=None):
    layout = beam.beam_kv_layout_fp8(ci.kind, params, ci.B, ci.slots)
    q, k, v, g = (dev(torch, x) for x in (ci.q, ci.k, ci.v, ci.gate))
    qw = torch.from_numpy(ci.q_norm_w).cuda()
    kw = torch.from_numpy(ci.k_norm_w).cuda()
    bias = torch.from_numpy(ci.gate_bias).cuda()
    pos0 = torch.from_numpy(ci.pos0).cuda()
    if kc is None:
        kc = torch.from_numpy(np.ascontiguousarray(kc0)).cuda().view(-1)
        vc = torch.from_numpy(np.ascontiguousarray(vc0)).cuda().view(-1)
    out = torch.full((ci.B, ci.T, 48 * 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    beam.beam_attn_prefill_chunk_fp8(ci.kind, params, q, k, v, g, qw, kw, bias, pos0, out, kc, vc,
                                     layout, ks, vs, dev_status=status)
    torch.cuda.synchronize()
    return out, kc, vc


def check_codes(orc, ci, params, kc, vc, kc0, vc0, ks, vs):
    P = oracle_params(orc, params)
    S = ci.slots
    kh = kc.cpu().numpy().reshape(ci.B, 8, S, 128)
    vh = vc.cpu().numpy().reshape(ci.B, 8, S, 128)
    kexp, vexp = kc0.copy(), vc0.copy()
    for b in range(ci.B):
        p0 = int(ci.pos0[b])
        first = max(0, ci.T - S) if ci.kind == wl.LOCAL else 0
        for i in range(first, ci.T):
            t = p0 + i
            s = orc.cache_slot(ci.kind, t, S)
            kr, vr = orc.kv_row_fp8(ci.kind, P, ci.k[b, i], ci.v[b, i], ci.k_norm_w, t, ks, vs)
            assert _codes_close(kh[b, :, s], kr), (b, t)
            kexp[b, :, s] = kh[b, :, s]
            vexp[b, :, s] = vr
    np.testing.assert_array_equal(vh, vexp)    # new value codes exact, nothing else moved
    np.testing.assert_array_equal(kh, kexp)


@pytest.mark.parametrize("kind,pos0,T,window,slots", [
    (wl.LOCAL, [0, 100, 2000], 300, 512, 512),    # no history, a partial window, a full ring
    (wl.LOCAL, [1000], 700, 512, 512),            # T > window
    (wl.LOCAL, [37, 5], 129, 100, 100),           # window inside a tile, ragged T
    (wl.LOCAL, [511, 512, 513], 1, 512, 512),     # one-token chunks across the ring's wrap
    (wl.LOCAL, [0, 100, 2000], 8, 512, 512),      # multi-token decode path
    (wl.LOCAL, [510, 511, 520], 16, 512, 512),
    (wl.LOCAL, [3000, 700], 8, 2048, 2048),       # more splits per head (merge kernel)
    (wl.GLOBAL, [0, 1000, 127], 333, 512, 2048),  # unaligned history lengths
    (wl.GLOBAL, [4000], 130, 512, 4200),          # padding stops at the capacity
    (wl.GLOBAL, [0, 1000, 127], 16, 512, 2048),   # multi-token decode path
    (wl.GLOBAL, [0, 4090], 5, 512, 4096),
    (wl.GLOBAL, [5], 1, 512, 64),
])
def test_chunk_fp8_matches_oracle_and_writes_codes(env, kind, pos0, T, window, slots):
    torch, beam, orc = env
    params = beam.default_params(window=window)
    ci = wl.chunk_inputs(kind, T, pos0, slots, 51 + T, layer=f"c8{kind}{window}", with_cache=False)
    shape = (ci.B, 8, slots, 128)
    kc0 = _codes(shape, 51 + T, f"c8{kind}/kc", K_SCALE)
    vc0 = _codes(shape, 51 + T, f"c8{kind}/vc", V_SCALE)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, kc, vc = run_chunk_fp8(torch, beam, ci, params, kc0, vc0, K_SCALE, V_SCALE, status)
    assert int(status.item()) == 0
    ref = orc.prefill_chunk_fp8(kind, oracle_params(orc, params), ci.q, ci.k, ci.v, ci.gate,
                                ci.q_norm_w, ci.k_norm_w, ci.gate_bias, ci.pos0, kc0, vc0,
                                K_SCALE, V_SCALE)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"fp8 chunk kind={kind} pos0={pos0} T={T}")
    check_codes(orc, ci, params, kc, vc, kc0, vc0, K_SCALE, V_SCALE)


@pytest.mark.parametrize("kind", [wl.GLOBAL, wl.LOCAL])
def test_chunked_prefill_workload_fp8_sampled_rows(env, kind):
    """The chunked-prefill workload (8192 new tokens after 57,344 cached) over FP8 caches
    drawn on the device; sampled rows against the oracle."""
    torch, beam, orc = env
    params = beam.default_params()
    w = wl.workload("chunked_prefill")
    slots = w.extra["global_slots"] if kind == wl.GLOBAL else wl.WINDOW
    ci = wl.chunk_inputs(kind, w.T, [w.extra["pos0"]] * w.B, slots, w.seed, layer=f"f8full{kind}",
                         with_cache=False)
    layout = beam.beam_kv_layout_fp8(kind, params, w.B, slots)
    kc = torch.empty(layout.bytes_k, dtype=torch.uint8, device="cuda")
    vc = torch.empty_like(kc)
    wl.device_normal_e4m3_(kc, w.seed, f"f8full{kind}/kc", K_SCALE)
    wl.device_normal_e4m3_(vc, w.seed, f"f8full{kind}/vc", V_SCALE)
    kc0 = kc.cpu().numpy().reshape(w.B, 8, slots, 128).copy()
    vc0 = vc.cpu().numpy().reshape(w.B, 8, slots, 128).copy()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, *_ = run_chunk_fp8(torch, beam, ci, params, None, None, K_SCALE, V_SCALE, status, kc, vc)
    assert int(status.item()) == 0
    rng = wl.rng(w.seed, f"f8rows{kind}")
    ri = np.unique(np.concatenate([[0, 127, 128, 4095, w.T - 1], rng.integers(0, w.T, 7)]))
    rb = np.zeros_like(ri)
    ref = orc.prefill_chunk_rows_fp8(kind, oracle_params(orc, params), ci.q, ci.k, ci.v, ci.gate,
                                     ci.q_norm_w, ci.k_norm_w, ci.gate_bias, ci.pos0, kc0, vc0,
                                     K_SCALE, V_SCALE, rb, ri)
    got = host_bits(out).reshape(w.B, w.T, 48, 128)[0, ri]
    assert_close(got, ref, f"fp8 chunked_prefill kind={kind}")


def test_multi_token_decode_fp8_long_context(env):
    """Eight new tokens (a drafted block) after 262,136 cached ones over an FP8 global cache
    drawn on the device: every output row against the oracle."""
    torch, beam, orc = env
    params = beam.default_params()
    T, ctx = 8, 262144
    ci = wl.chunk_inputs(wl.GLOBAL, T, [ctx - T], ctx, 61, layer="f8m", with_cache=False)
    layout = beam.beam_kv_layout_fp8(wl.GLOBAL, params, 1, ctx)
    kc = torch.empty(layout.bytes_k, dtype=torch.uint8, device="cuda")
    vc = torch.empty_like(kc)
    wl.device_normal_e4m3_(kc, 61, "f8m/kc", K_SCALE)
    wl.device_normal_e4m3_(vc, 61, "f8m/vc", V_SCALE)
    kc0 = kc.cpu().numpy().reshape(1, 8, ctx, 128).copy()
    vc0 = vc.cpu().numpy().reshape(1, 8, ctx, 128).copy()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, *_ = run_chunk_fp8(torch, beam, ci, params, None, None, K_SCALE, V_SCALE, status, kc, vc)
    assert int(status.item()) == 0
    ref = orc.prefill_chunk_fp8(wl.GLOBAL, oracle_params(orc, params), ci.q, ci.k, ci.v, ci.gate,
                                ci.q_norm_w, ci.k_norm_w, ci.gate_bias, ci.pos0, kc0, vc0,
                                K_SCALE, V_SCALE)
    assert_close(host_bits(out).reshape(ref.shape), ref, "fp8 multi-token decode")


def test_chunk_fp8_out_of_range_sequence_sets_status(env):
    """A global sequence whose chunk does not fit is neither written nor attended; the
    others are (status BEAM_ERR_CAPACITY)."""
    torch, beam, orc = env
    params = beam.default_params()
    T, slots = 40, 300
    ci = wl.chunk_inputs(wl.GLOBAL, T, [10, 290], slots, 71, layer="f8bad", with_cache=False)
    shape = (2, 8, slots, 128)
    kc0 = _codes(shape, 71, "f8bad/kc", K_SCALE)
    vc0 = _codes(shape, 71, "f8bad/vc", V_SCALE)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, kc, vc = run_chunk_fp8(torch, beam, ci, params, kc0, vc0, K_SCALE, V_SCALE, status)
    assert int(status.item()) == -5
    got = host_bits(out).reshape(2, T, 48, 128)
    assert np.all(np.isnan(wl.bf16_bits_to_f32(got[1])))        # untouched
    np.testing.assert_array_equal(kc.cpu().numpy().reshape(shape)[1], kc0[1])
    np.testing.assert_array_equal(vc.cpu().numpy().reshape(shape)[1], vc0[1])
    ref = orc.prefill_chunk_rows_fp8(wl.GLOBAL, oracle_params(orc, params), ci.q[:1], ci.k[:1],
                                     ci.v[:1], ci.gate[:1], ci.q_norm_w, ci.k_norm_w,
                                     ci.gate_bias, ci.pos0[:1], kc0[:1], vc0[:1], K_SCALE,
                                     V_SCALE, np.zeros(T, np.int64), np.arange(T))
    assert_close(got[0].reshape(ref.shape), ref, "fp8 chunk, the sequence that fits")
