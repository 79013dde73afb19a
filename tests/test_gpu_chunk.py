"""Chunked prefill against an existing cache (beam_attn_prefill_chunk) through
the C ABI, against the fp64 oracle.

Sequence b adds T new tokens at positions pos0[b] .. pos0[b] + T - 1 after pos0[b]
tokens already in the cache.  Cache contents before the call are seeded synthetic
rows given to both sides (the oracle reads them as the earlier keys), so the
comparison isolates the chunk's own arithmetic and indexing.  Outputs use the
parity bar of the other GPU tests; the appended cache rows are checked as in the
plain prefill's fused append; untouched slots must keep their bits.
"""
import numpy as np
import pytest

import workloads as wl
from test_gpu_parity import (K_ABS, as_f64, assert_close, dev, env, host_bits,  # noqa: F401
                             oracle_params, run_prefill)

pytestmark = pytest.mark.gpu


def run_chunk(torch, beam, ci, params, status=None, kc=None, vc=None):
    layout = beam.beam_kv_layout(ci.kind, params, ci.B, ci.slots)
    assert layout.slots_per_seq == ci.slots
    q, k, v, g = (dev(torch, x) for x in (ci.q, ci.k, ci.v, ci.gate))
    qw = torch.from_numpy(ci.q_norm_w).cuda()
    kw = torch.from_numpy(ci.k_norm_w).cuda()
    bias = torch.from_numpy(ci.gate_bias).cuda()
    pos0 = torch.from_numpy(ci.pos0).cuda()
    if kc is None:
        kc = dev(torch, ci.k_cache).view(-1)
        vc = dev(torch, ci.v_cache).view(-1)
    out = torch.full((ci.B, ci.T, 48 * 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    beam.beam_attn_prefill_chunk(ci.kind, params, q, k, v, g, qw, kw, bias, pos0, out, kc, vc,
                                 layout, dev_status=status)
    torch.cuda.synchronize()
    return out, kc, vc


def oracle_chunk(orc, beam, ci, params, rows=None):
    P = oracle_params(orc, params)
    if rows is None:
        return orc.prefill_chunk(ci.kind, P, ci.q, ci.k, ci.v, ci.gate, ci.q_norm_w, ci.k_norm_w,
                                 ci.gate_bias, ci.pos0, ci.k_cache, ci.v_cache)
    rb, ri = rows
    return orc.prefill_chunk_rows(ci.kind, P, ci.q, ci.k, ci.v, ci.gate, ci.q_norm_w, ci.k_norm_w,
                                  ci.gate_bias, ci.pos0, ci.k_cache, ci.v_cache, rb, ri)


def check_cache(orc, ci, params, kc, vc, skip=()):
    """New rows at their slots (V bit-exact, K within one bf16 step of the oracle);
    every other slot unchanged, except a global cache's zeroed value padding."""
    P = oracle_params(orc, params)
    S = ci.slots
    kh = host_bits(kc).reshape(ci.B, 8, S, 128)
    vh = host_bits(vc).reshape(ci.B, 8, S, 128)
    written = np.zeros((ci.B, S), bool)
    padded = np.zeros((ci.B, S), bool)
    for b in range(ci.B):
        if b in skip:
            continue
        p0 = int(ci.pos0[b])
        first = max(0, ci.T - S) if ci.kind == wl.LOCAL else 0
        for i in range(first, ci.T):
            t = p0 + i
            s = orc.cache_slot(ci.kind, t, S)
            kr, vr = orc.kv_row(ci.kind, P, ci.k[b, i], ci.v[b, i], ci.k_norm_w, t)
            np.testing.assert_array_equal(vh[b, :, s], vr)
            d = np.abs(as_f64(kh[b, :, s]) - as_f64(kr))
            assert np.all(d <= np.abs(as_f64(kr)) * 2.0 ** -7 + K_ABS), (b, t)
            written[b, s] = True
        if ci.kind == wl.GLOBAL:   # the attention kernels read whole 128-key blocks
            end = p0 + ci.T
            padded[b, end:min(S, (end + 127) // 128 * 128)] = True
    keep = ~written
    assert np.array_equal(kh.transpose(0, 2, 1, 3)[keep], ci.k_cache.transpose(0, 2, 1, 3)[keep])
    vkeep = keep & ~padded
    assert np.array_equal(vh.transpose(0, 2, 1, 3)[vkeep], ci.v_cache.transpose(0, 2, 1, 3)[vkeep])
    assert np.all(vh.transpose(0, 2, 1, 3)[padded] == 0)


@pytest.mark.parametrize("kind,pos0,T,window,slots", [
    (wl.LOCAL, [0, 100, 2000], 300, 512, 512),    # no history, a partial window, a full ring
    (wl.LOCAL, [1000], 700, 512, 512),            # T > window: the ring is overwritten
    (wl.LOCAL, [37, 5], 129, 100, 100),           # window inside a tile, ragged T
    (wl.LOCAL, [3], 130, 1, 1),                   # window of one
    (wl.LOCAL, [511, 512, 513], 1, 512, 512),     # one-token chunks across the ring's wrap
    (wl.GLOBAL, [0, 1000, 127], 333, 512, 2048),  # unaligned history lengths
    (wl.GLOBAL, [5], 1, 512, 64),
    (wl.GLOBAL, [4000], 130, 512, 4200),          # padding stops at the capacity
    (wl.GLOBAL, [1, 128, 255], 128, 512, 640),
    # up to 16 new tokens: the multi-token decode path (one CTA per KV head writing the
    # gated output when the keys fit it, else split-K partials and a merge)
    (wl.LOCAL, [0, 100, 2000], 8, 512, 512),
    (wl.LOCAL, [37, 5], 3, 100, 100),
    (wl.LOCAL, [3], 16, 1, 1),
    (wl.LOCAL, [510, 511, 520], 16, 512, 512),
    (wl.LOCAL, [3000, 700], 8, 2048, 2048),       # a wider window: more splits per head
    (wl.GLOBAL, [0, 1000, 127], 16, 512, 2048),
    (wl.GLOBAL, [0, 4090], 5, 512, 4096),
    (wl.GLOBAL, [70000], 2, 512, 70002),
])
def test_chunk_matches_oracle_and_appends(env, kind, pos0, T, window, slots):
    torch, beam, orc = env
    params = beam.default_params(window=window)
    ci = wl.chunk_inputs(kind, T, pos0, slots, 31 + T, layer=f"c{kind}{window}")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, kc, vc = run_chunk(torch, beam, ci, params, status)
    assert int(status.item()) == 0
    ref = oracle_chunk(orc, beam, ci, params)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"kind={kind} pos0={pos0} T={T}")
    check_cache(orc, ci, params, kc, vc)


def test_long_global_history_sampled_rows(env):
    """65,573 cached tokens, then a chunk of 1000: sampled rows (first, last, a
    tile edge, random) against the oracle."""
    torch, beam, orc = env
    params = beam.default_params()
    P0, T = 65573, 1000
    ci = wl.chunk_inputs(wl.GLOBAL, T, [P0], P0 + T + 300, 41, layer="long")
    out, kc, vc = run_chunk(torch, beam, ci, params)
    rng = wl.rng(41, "rows")
    ri = np.unique(np.concatenate([[0, 1, 127, 128, T - 1], rng.integers(0, T, 7)]))
    rb = np.zeros_like(ri)
    ref = oracle_chunk(orc, beam, ci, params, (rb, ri))
    got = host_bits(out).reshape(1, T, 48, 128)[0, ri]
    assert_close(got, ref, "long global chunk")


@pytest.mark.parametrize("kind", [wl.GLOBAL, wl.LOCAL])
def test_chunked_prefill_workload_sampled_rows(env, kind):
    """The chunked-prefill workload at full size, in the call the bench times: 8192
    new tokens after 57,344 cached ones; sampled rows against the oracle."""
    torch, beam, orc = env
    params = beam.default_params()
    w = wl.workload("chunked_prefill")
    slots = w.extra["global_slots"] if kind == wl.GLOBAL else wl.WINDOW
    ci = wl.chunk_inputs(kind, w.T, [w.extra["pos0"]] * w.B, slots, w.seed, layer=f"full{kind}")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, *_ = run_chunk(torch, beam, ci, params, status)
    assert int(status.item()) == 0
    rng = wl.rng(w.seed, f"rows{kind}")
    ri = np.unique(np.concatenate([[0, 127, 128, 4095, w.T - 1], rng.integers(0, w.T, 7)]))
    rb = np.zeros_like(ri)
    ref = oracle_chunk(orc, beam, ci, params, (rb, ri))
    got = host_bits(out).reshape(w.B, w.T, 48, 128)[0, ri]
    assert_close(got, ref, f"chunked_prefill kind={kind}")


def test_multi_token_decode_1m_context_sampled(env):
    """Eight new tokens after 1,048,568 cached ones in a global layer (the
    verification of an 8-token drafted block at 1M context): every output of the
    first, fourth and last new token against the oracle; cache drawn on the device."""
    torch, beam, orc = env
    params = beam.default_params()
    P = oracle_params(orc, params)
    T, slots = 8, wl.MAX_CONTEXT
    ci = wl.chunk_inputs(wl.GLOBAL, T, [slots - T], slots, 53, layer="m1m", with_cache=False)
    layout = beam.beam_kv_layout(wl.GLOBAL, params, 1, slots)
    kc = torch.empty(layout.bytes_k // 2, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    wl.device_normal_bf16_(kc, 53, "m1m/kc")
    wl.device_normal_bf16_(vc, 53, "m1m/vc")
    ci.k_cache = host_bits(kc).reshape(1, 8, slots, 128)
    ci.v_cache = host_bits(vc).reshape(1, 8, slots, 128)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, *_ = run_chunk(torch, beam, ci, params, status, kc=kc, vc=vc)
    assert int(status.item()) == 0
    ri = np.array([0, 3, T - 1])
    ref = oracle_chunk(orc, beam, ci, params, (np.zeros_like(ri), ri))
    assert_close(host_bits(out).reshape(1, T, 48, 128)[0, ri], ref, "multi-token decode 1M")


@pytest.mark.parametrize("kind", [wl.GLOBAL, wl.LOCAL])
def test_prefill_then_chunk_equals_one_shot(env, kind):
    """The GPU's own prefill fills the cache with the first T1 tokens, then one chunk
    adds T2 more: the chunk rows equal the oracle's one-shot prefill rows T1 ..
    T1 + T2 - 1 of the whole sequence (the cache's bf16 keys are the only
    difference, inside the tolerance)."""
    torch, beam, orc = env
    params = beam.default_params()
    T1, T2 = 700, 333
    _prefill_then_chunk(torch, beam, orc, kind, params, T1, T2)
    _prefill_then_chunk(torch, beam, orc, kind, params, 1000, 9)   # the few-token path


def _prefill_then_chunk(torch, beam, orc, kind, params, T1, T2):
    full = wl.prefill_inputs(1, T1 + T2, 51, layer=f"two{kind}")
    layout = beam.beam_kv_layout(kind, params, 1, T1 + T2)
    kc = torch.zeros(layout.bytes_k // 2, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    q, k, v, g = (dev(torch, x[:, :T1]) for x in (full.q, full.k, full.v, full.gate))
    qw = torch.from_numpy(full.q_norm_w).cuda()
    kw = torch.from_numpy(full.k_norm_w).cuda()
    bias = torch.from_numpy(full.gate_bias).cuda()
    out1 = torch.empty((1, T1, 6144), dtype=torch.bfloat16, device="cuda")
    beam.beam_attn_prefill(kind, params, q, k, v, g, qw, kw, bias, out1, kc, vc, layout)
    q, k, v, g = (dev(torch, x[:, T1:]) for x in (full.q, full.k, full.v, full.gate))
    out2 = torch.full((1, T2, 6144), float("nan"), dtype=torch.bfloat16, device="cuda")
    pos0 = torch.tensor([T1], dtype=torch.int64, device="cuda")
    beam.beam_attn_prefill_chunk(kind, params, q, k, v, g, qw, kw, bias, pos0, out2, kc, vc,
                                 layout)
    torch.cuda.synchronize()
    P = oracle_params(orc, params)
    rows = np.arange(T1, T1 + T2)
    ref = orc.prefill_rows(kind, P, full.q, full.k, full.v, full.gate, full.q_norm_w,
                           full.k_norm_w, full.gate_bias, np.zeros_like(rows), rows)
    assert_close(host_bits(out2).reshape(T2, 48, 128), ref, f"two calls kind={kind}")


def test_global_chunk_at_zero_is_bit_identical_to_prefill(env):
    """pos0 = 0: a global chunk reads its keys from the cache the prefill would have
    read from its workspace, over the same key blocks: identical bits."""
    torch, beam, orc = env
    params = beam.default_params()
    B, T = 2, 1000
    ci = wl.chunk_inputs(wl.GLOBAL, T, [0, 0], T, 61, layer="zero")
    out_c, *_ = run_chunk(torch, beam, ci, params)
    inp = wl.PrefillInputs(B, T, ci.q, ci.k, ci.v, ci.gate, ci.q_norm_w, ci.k_norm_w,
                           ci.gate_bias)
    out_p, *_ = run_prefill(torch, beam, wl.GLOBAL, inp, params)
    assert np.array_equal(host_bits(out_c), host_bits(out_p))


def test_chunk_out_of_range_sequences_set_status_and_write_nothing(env):
    """A global sequence whose chunk would pass the capacity, and a local one with a
    negative pos0, are skipped (status BEAM_ERR_CAPACITY, output rows and cache
    untouched); the valid sequence in the same call is still correct."""
    torch, beam, orc = env
    params = beam.default_params()
    for kind, pos0, slots in ((wl.GLOBAL, [10, 1990], 2048), (wl.LOCAL, [10, -3], 512)):
        ci = wl.chunk_inputs(kind, 100, pos0, slots, 71, layer=f"cap{kind}")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out, kc, vc = run_chunk(torch, beam, ci, params, status)
        assert int(status.item()) == -5
        o = host_bits(out)
        assert np.all(np.isnan(as_f64(o[1])))
        good = wl.ChunkInputs(1, ci.T, kind, ci.pos0[:1], ci.q[:1], ci.k[:1], ci.v[:1],
                              ci.gate[:1], ci.q_norm_w, ci.k_norm_w, ci.gate_bias, slots,
                              ci.k_cache[:1], ci.v_cache[:1])
        ref = oracle_chunk(orc, beam, good, params)
        assert_close(o[:1].reshape(ref.shape), ref, f"valid sequence kind={kind}")
        kh = host_bits(kc).reshape(2, 8, slots, 128)
        vh = host_bits(vc).reshape(2, 8, slots, 128)
        assert np.array_equal(kh[1], ci.k_cache[1]) and np.array_equal(vh[1], ci.v_cache[1])


@pytest.mark.parametrize("kind,T", [(wl.LOCAL, 8), (wl.GLOBAL, 8), (wl.LOCAL, 300),
                                    (wl.GLOBAL, 300)])
def test_back_to_back_calls_sharing_one_workspace(env, kind, T):
    """Three chunk calls issued on one stream with no synchronisation between them, all
    with the same workspace: a call's prologue must not overwrite the workspace rows, RoPE
    table or merge tickets that the previous call's attention kernel still reads (the
    launches overlap under programmatic dependent launch).  Each output against the oracle."""
    torch, beam, orc = env
    params = beam.default_params()
    slots = 512 if kind == wl.LOCAL else 4096
    cases = [wl.chunk_inputs(kind, T, pos0, slots, 81 + n, layer=f"b2b{kind}{T}/{n}")
             for n, pos0 in enumerate(([700, 3], [3000, 1200], [40, 2500]))]
    layout = beam.beam_kv_layout(kind, params, 2, slots)
    need = max(beam.beam_prefill_chunk_workspace_bytes(kind, params, 2, T, layout), 256)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    outs = []
    for ci in cases:
        q, k, v, g = (dev(torch, x) for x in (ci.q, ci.k, ci.v, ci.gate))
        kc = dev(torch, ci.k_cache).view(-1)
        vc = dev(torch, ci.v_cache).view(-1)
        out = torch.full((2, T, 48 * 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        beam.beam_attn_prefill_chunk(kind, params, q, k, v, g, torch.from_numpy(ci.q_norm_w).cuda(),
                                     torch.from_numpy(ci.k_norm_w).cuda(),
                                     torch.from_numpy(ci.gate_bias).cuda(),
                                     torch.from_numpy(ci.pos0).cuda(), out, kc, vc, layout,
                                     workspace=ws)
        outs.append((out, q, k, v, g, kc, vc))   # keep every buffer alive until the sync
    torch.cuda.synchronize()
    for n, (ci, o) in enumerate(zip(cases, outs)):
        ref = oracle_chunk(orc, beam, ci, params)
        assert_close(host_bits(o[0]).reshape(ref.shape), ref, f"back-to-back call {n}")
