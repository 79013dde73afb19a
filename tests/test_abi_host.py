"""Host-side checks of the C ABI: the library loads on a machine without a GPU,
exports every function the header declares, computes cache layouts that match
the pages' byte counts, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="module")
def beam():
    from global_nope_gqa_b200 import build
    build.build()
    import global_nope_gqa_b200 as g
    g.lib()
    return g


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"BEAM_API\s+[\w\s\*]+?\b(beam_\w+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(beam):
    declared = _declared()
    assert len(declared) >= 8
    out = subprocess.check_output(["nm", "-D", "--defined-only", beam.LIB_PATH], text=True)
    exported = set(re.findall(r"\bT (beam_\w+)", out))
    missing = [n for n in declared if n not in exported]
    assert not missing, missing
    for n in declared:
        assert hasattr(beam.lib(), n)
    assert set(beam.EXPORTS) == set(declared)


def test_build_targets_sm100a_only():
    from global_nope_gqa_b200 import build
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1


def test_default_params(beam):
    p = beam.default_params()
    assert (p.n_q_heads, p.n_kv_heads, p.head_dim, p.window) == (48, 8, 128, 512)
    assert p.rope_theta == 10000.0 and p.ssmax_base == 2048.0
    assert p.ssmax_exp == pytest.approx(0.1) and p.rms_eps == pytest.approx(1e-6)
    assert p.softmax_scale == pytest.approx(1 / np.sqrt(128))


def _golden_bytes():
    vals = {}
    with open(os.path.join(GOLDEN, "kv_bytes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, v, unit, tol = line.split()
                vals[name] = (float(v), unit, float(tol))
    return vals


def test_kv_layout_matches_page_byte_counts(beam):
    """Section 'KV memory: nine growing caches, not 52' and the Arabic page:
    36 KiB vs 208 KiB per token, 36.08 GiB vs 208 GiB at 1M, 4.6 vs 26 GiB at 128K,
    FP8 halves: 18 KiB, 18.04 GiB, 104 GiB, ~43 MiB of local caches."""
    p = beam.default_params()
    g = _golden_bytes()
    unit = {"KiB": 1024, "MiB": 1024 ** 2, "GiB": 1024 ** 3}

    def per_layer(kind, tokens):
        L = beam.beam_kv_layout(kind, p, 1, tokens)
        return L.bytes_k + L.bytes_v

    one = per_layer(beam.GLOBAL, 1)
    assert one == 4096
    n_global, n_local = 9, 43

    def check(name, value_bytes):
        v, u, tol = g[name]
        assert abs(value_bytes / unit[u] - v) <= tol, (name, value_bytes / unit[u], v)

    check("per_token_global_bf16", n_global * one)
    check("per_token_global_fp8", n_global * one // 2)
    check("per_token_all_global_bf16", 52 * one)
    local = per_layer(beam.LOCAL, 1 << 30)   # a ring ignores the capacity
    assert local == 512 * 4096
    check("local_caches_fp8", n_local * local // 2)
    for tokens, tag in ((1 << 20, "1m"), (128 * 1024, "128k")):
        total = n_global * per_layer(beam.GLOBAL, tokens) + n_local * local
        check(f"at_{tag}_bf16", total)
        check(f"at_{tag}_all_global_bf16", 52 * per_layer(beam.GLOBAL, tokens))
    check("at_1m_fp8", (n_global * per_layer(beam.GLOBAL, 1 << 20) + n_local * local) // 2)
    check("at_1m_all_global_fp8", 52 * per_layer(beam.GLOBAL, 1 << 20) // 2)
    assert n_global * per_layer(beam.GLOBAL, 1 << 20) + n_local * local == 38_744_883_200


def test_kv_layout_strides(beam):
    p = beam.default_params()
    L = beam.beam_kv_layout(beam.GLOBAL, p, 4, 1000)
    assert (L.slots_per_seq, L.stride_slot, L.stride_head, L.stride_seq) == (1000, 128, 128000, 1024000)
    assert L.bytes_k == 4 * 1024000 * 2
    L = beam.beam_kv_layout(beam.LOCAL, p, 2, 5)
    assert L.slots_per_seq == 512


def _status(beam, fn, *args):
    return getattr(beam.lib(), fn)(*args)


def test_host_validation_rejects_before_launch(beam):
    """Every rejection below returns before any CUDA call, so it runs without a GPU."""
    L = beam.lib()
    p = beam.default_params()
    P = ctypes.byref(p)
    A = 1 << 20  # a fake, 16-byte aligned device address: never dereferenced on the host
    ws = beam.beam_prefill_workspace_bytes(p, 1, 16)
    assert ws == 16 * 8 * 128 * 2 + 16 * 128 * 4   # prepared keys + RoPE cos/sin table
    args = lambda **kw: [kw.get("kind", 0), kw.get("P", P), kw.get("B", 1), kw.get("T", 16),
                         kw.get("q", A), A, A, A, A, A, A, kw.get("out", A), kw.get("kc", None),
                         kw.get("vc", None), kw.get("layout", None), kw.get("ws", A),
                         kw.get("ws_bytes", ws), None, None]
    assert L.beam_attn_prefill(*args(kind=2)) == -1
    assert L.beam_attn_prefill(*args(P=None)) == -1
    assert L.beam_attn_prefill(*args(B=-1)) == -1
    assert L.beam_attn_prefill(*args(T=0)) == 0          # empty input: a no-op
    assert L.beam_attn_prefill(*args(B=0)) == 0
    assert L.beam_attn_prefill(*args(q=None)) == -1
    assert L.beam_attn_prefill(*args(out=A + 2)) == -7
    assert L.beam_attn_prefill(*args(ws_bytes=ws - 1)) == -6
    assert L.beam_attn_prefill(*args(ws=None)) == -6
    assert L.beam_attn_prefill(*args(kc=A)) == -1        # K cache without V cache
    small = beam.beam_kv_layout(beam.GLOBAL, p, 1, 15)
    assert L.beam_attn_prefill(*args(kind=1, kc=A, vc=A, layout=ctypes.byref(small))) == -5
    bad = beam.beam_kv_layout(beam.GLOBAL, p, 1, 64)
    bad.stride_slot = 64
    assert L.beam_attn_prefill(*args(kind=1, kc=A, vc=A, layout=ctypes.byref(bad))) == -1
    ring = beam.beam_kv_layout(beam.GLOBAL, p, 1, 100)   # a local layer needs `window` slots
    assert L.beam_attn_prefill(*args(kind=0, kc=A, vc=A, layout=ctypes.byref(ring))) == -1
    for field, value in (("n_q_heads", 64), ("n_kv_heads", 4), ("head_dim", 64)):
        q = beam.default_params(**{field: value})
        assert L.beam_attn_prefill(*args(P=ctypes.byref(q))) == -2
    assert L.beam_attn_prefill(*args(P=ctypes.byref(beam.default_params(window=0)))) == -1

    glob = beam.beam_kv_layout(beam.GLOBAL, p, 2, 4096)
    dws = beam.beam_decode_workspace_bytes(beam.GLOBAL, p, 2, glob)
    assert dws > 2 * 48 * 128 * 2
    # a local (ring) decode merges on chip: a small nonzero size, whatever the batch
    ring512 = beam.beam_kv_layout(beam.LOCAL, p, 4096, 512)
    assert beam.beam_decode_workspace_bytes(beam.LOCAL, p, 4096, ring512) == 16
    dargs = lambda **kw: [kw.get("kind", 1), P, kw.get("B", 2), A, A, A, A, A, A, A,
                          kw.get("pos", A), A, A, kw.get("layout", ctypes.byref(glob)), A,
                          kw.get("ws", A), kw.get("ws_bytes", dws), None, None]
    assert L.beam_attn_decode(*dargs(B=0)) == 0
    assert L.beam_attn_decode(*dargs(pos=None)) == -1
    assert L.beam_attn_decode(*dargs(pos=A + 4)) == -7
    assert L.beam_attn_decode(*dargs(layout=None)) == -1
    assert L.beam_attn_decode(*dargs(kind=0)) == -1      # ring layout must have 512 slots

    assert L.beam_kv_append(1, P, 1, 4, A, A, A, None, A, A, ctypes.byref(glob), None, None) == -1
    assert L.beam_kv_append(1, P, 1, 0, A, A, A, A, A, A, ctypes.byref(glob), None, None) == 0
    # chunked prefill: the cache is required, pos0 is a device int64 array
    ring = beam.beam_kv_layout(beam.LOCAL, p, 1, 0)
    cws = beam.beam_prefill_chunk_workspace_bytes(beam.LOCAL, p, 1, 17, ring)
    assert cws == 2 * (511 + 17) * 8 * 128 * 2 + 17 * 128 * 4   # earlier + new K/V rows, RoPE table
    assert beam.beam_prefill_chunk_workspace_bytes(beam.GLOBAL, p, 1, 17, glob) == 0
    # up to 16 new tokens: also the split-K partials, growing with the cache capacity
    few = beam.beam_prefill_chunk_workspace_bytes(beam.LOCAL, p, 1, 16, ring)
    assert few > 2 * (511 + 16) * 8 * 128 * 2 + 16 * 128 * 4
    g1 = beam.beam_prefill_chunk_workspace_bytes(beam.GLOBAL, p, 1, 8, glob)
    g2 = beam.beam_prefill_chunk_workspace_bytes(beam.GLOBAL, p, 1, 8,
                                                 beam.beam_kv_layout(beam.GLOBAL, p, 1, 1 << 20))
    assert 0 < g1 <= g2
    cargs = lambda **kw: [kw.get("kind", 0), P, kw.get("B", 1), kw.get("T", 17), A, A, A, A, A, A,
                          A, kw.get("pos0", A), A, kw.get("kc", A), A,
                          kw.get("layout", ctypes.byref(ring)), kw.get("ws", A),
                          kw.get("ws_bytes", cws), None, None]
    assert L.beam_attn_prefill_chunk(*cargs(T=0)) == 0
    assert L.beam_attn_prefill_chunk(*cargs(pos0=None)) == -1
    assert L.beam_attn_prefill_chunk(*cargs(pos0=A + 4)) == -7
    assert L.beam_attn_prefill_chunk(*cargs(kc=None)) == -1
    assert L.beam_attn_prefill_chunk(*cargs(layout=None)) == -1
    assert L.beam_attn_prefill_chunk(*cargs(ws_bytes=cws - 1)) == -6
    assert L.beam_attn_prefill_chunk(*cargs(ws=None)) == -6
    small = beam.beam_kv_layout(beam.GLOBAL, p, 1, 15)
    assert L.beam_attn_prefill_chunk(*cargs(kind=1, layout=ctypes.byref(small), ws=None,
                                            ws_bytes=0)) == -5          # T = 17 > 15 slots
    assert L.beam_attn_prefill_chunk(*cargs(kind=0, layout=ctypes.byref(small))) == -1

    # FP8 cache: one byte per element, rows on 16 bytes, positive finite scales
    f8 = beam.beam_kv_layout_fp8(beam.GLOBAL, p, 2, 4096)
    assert f8.bytes_k == 2 * 8 * 4096 * 128 and f8.stride_slot == 128
    assert L.beam_kv_append_fp8(1, P, 1, 4, A, A, A, A, A, A, ctypes.byref(f8), 0.0, 1.0, None,
                                None) == -1
    assert L.beam_kv_append_fp8(1, P, 1, 4, A, A, A, A, A, A, ctypes.byref(f8), 1.0,
                                float("inf"), None, None) == -1
    odd = beam.beam_kv_layout_fp8(beam.GLOBAL, p, 1, 4096)
    odd.stride_head = 4096 * 128 + 8         # a bf16-aligned but not FP8-aligned row stride
    odd.stride_seq = 8 * odd.stride_head
    assert L.beam_kv_append_fp8(1, P, 1, 4, A, A, A, A, A, A, ctypes.byref(odd), 1.0, 1.0, None,
                                None) == -7
    f8args = lambda **kw: [1, P, 2, A, A, A, A, A, A, A, A, A, A, ctypes.byref(f8),
                           kw.get("ks", 1.0), kw.get("vs", 1.0), A, A, dws, None, None]
    assert L.beam_attn_decode_fp8(*f8args(ks=-1.0)) == -1
    assert L.beam_attn_decode_fp8(*f8args(vs=float("nan"))) == -1

    for s in (0, -1, -2, -3, -4, -5, -6, -7, -8, 99):
        assert isinstance(beam.beam_status_string(s), str)
