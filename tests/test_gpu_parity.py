"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Every floating-point output is checked element by element with the bar
|y_gpu - y_ref| <= 1e-2 + 1e-2 * |y_ref| (bf16 outputs, fp32 accumulation).
Masks and cache indexing are checked bit-exactly: which outputs are exactly
zero under a one-hot probe, which cache slots were written, and the written
value bits.
"""
import numpy as np
import pytest

import workloads as wl

pytestmark = pytest.mark.gpu

ATOL = 1e-2
RTOL = 1e-2
# Prepared keys are formed in fp32 on the device and in double by the oracle, then
# both are rounded to bf16: the two may sit one bf16 step apart, and where RoPE
# cancels (a small coordinate from O(1) terms) the fp32 rounding adds ~1e-6.
K_ABS = 1e-5


@pytest.fixture(scope="module")
def env():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import global_nope_gqa_b200 as beam
    beam.lib()  # fails loudly if the CUDA library is missing
    import oracle
    oracle.build()
    return torch, beam, oracle


def dev(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t):
    return t.detach().cpu().contiguous().view(dtype=__import__("torch").int16).numpy().view(np.uint16)


def as_f64(bits):
    return wl.bf16_bits_to_f32(bits).astype(np.float64)


def assert_close(got_bits, ref, what=""):
    got = as_f64(got_bits)
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert not np.any(np.isnan(got)), f"{what}: NaN in GPU output"
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; "
                           f"max err {err.max():.3e} at {np.unravel_index(np.argmax(err - bound), err.shape)}")


def run_prefill(torch, beam, kind, inp, params=None, cache=False, status=None):
    params = params or beam.default_params()
    B, T = inp.B, inp.T
    q, k, v, g = (dev(torch, x) for x in (inp.q, inp.k, inp.v, inp.gate))
    qw = torch.from_numpy(inp.q_norm_w).cuda()
    kw = torch.from_numpy(inp.k_norm_w).cuda()
    bias = torch.from_numpy(inp.gate_bias).cuda()
    out = torch.full((B, T, 48 * 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    kc = vc = layout = None
    if cache:
        layout = beam.beam_kv_layout(kind, params, B, T)
        n = layout.bytes_k // 2
        kc = torch.full((n,), -7.0, dtype=torch.bfloat16, device="cuda")
        vc = torch.full((n,), -7.0, dtype=torch.bfloat16, device="cuda")
    beam.beam_attn_prefill(kind, params, q, k, v, g, qw, kw, bias, out, kc, vc, layout,
                           dev_status=status)
    torch.cuda.synchronize()
    return out, kc, vc, layout


def oracle_params(orc, params):
    return orc.params(window=params.window, rope_theta=params.rope_theta, rms_eps=params.rms_eps,
                      ssmax_base=params.ssmax_base, ssmax_exp=params.ssmax_exp,
                      softmax_scale=float(np.float32(params.softmax_scale)))


# ------------------------------------------------------------------ prefill
@pytest.mark.parametrize("kind", [wl.LOCAL, wl.GLOBAL])
def test_prefill_tiny_workload_all_rows(env, kind):
    """Tiny prefill workload (B=1, T=768): every output element."""
    torch, beam, orc = env
    w = wl.workload("tiny_prefill")
    inp = wl.prefill_inputs(w.B, w.T, w.seed, layer=f"kind{kind}")
    out, *_ = run_prefill(torch, beam, kind, inp)
    ref = orc.prefill(kind, oracle_params(orc, beam.default_params()), inp.q, inp.k, inp.v,
                      inp.gate, inp.q_norm_w, inp.k_norm_w, inp.gate_bias)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"tiny kind={kind}")


@pytest.mark.parametrize("kind", [wl.LOCAL, wl.GLOBAL])
def test_prefill_gate_and_output_only_16_byte_aligned(env, kind):
    """Gate and output buffers that start 16 bytes past a 32-byte boundary (the API asks
    for 16): the kernel then moves those rows with 16-byte accesses instead of 32-byte
    ones.  Every output element against the oracle, and the guard words around the
    output untouched."""
    torch, beam, orc = env
    B, T = 1, 300
    inp = wl.prefill_inputs(B, T, 97, layer=f"align{kind}")
    params = beam.default_params()
    n = B * T * 48 * 128
    q, k, v = (dev(torch, x) for x in (inp.q, inp.k, inp.v))
    gbuf = torch.zeros(n + 16, dtype=torch.bfloat16, device="cuda")
    gbuf[8:8 + n].copy_(dev(torch, inp.gate).reshape(-1))
    obuf = torch.full((n + 16,), float("nan"), dtype=torch.bfloat16, device="cuda")
    obuf[:8] = 3.0
    obuf[8 + n:] = 3.0
    g, out = gbuf[8:8 + n], obuf[8:8 + n]
    assert g.data_ptr() % 32 == 16 and out.data_ptr() % 32 == 16
    qw = torch.from_numpy(inp.q_norm_w).cuda()
    kw = torch.from_numpy(inp.k_norm_w).cuda()
    bias = torch.from_numpy(inp.gate_bias).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    beam.beam_attn_prefill(kind, params, q, k, v, g, qw, kw, bias, out, None, None, None,
                           dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    guard = host_bits(torch.cat([obuf[:8], obuf[8 + n:]]))
    assert (guard == host_bits(torch.full((16,), 3.0, dtype=torch.bfloat16))).all()
    ref = orc.prefill(kind, oracle_params(orc, params), inp.q, inp.k, inp.v, inp.gate,
                      inp.q_norm_w, inp.k_norm_w, inp.gate_bias)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"16-byte aligned kind={kind}")


@pytest.mark.parametrize("kind,B,T,window", [
    (wl.LOCAL, 2, 333, 512), (wl.GLOBAL, 2, 333, 512), (wl.LOCAL, 1, 1000, 100),
    (wl.LOCAL, 1, 700, 64), (wl.GLOBAL, 3, 1, 512), (wl.LOCAL, 1, 1, 1), (wl.LOCAL, 1, 130, 1),
    (wl.GLOBAL, 1, 129, 512),
])
def test_prefill_ragged_and_windows(env, kind, B, T, window):
    """Ragged tails (T not a multiple of the tiles), windows inside a tile, T = 1."""
    torch, beam, orc = env
    params = beam.default_params(window=window)
    inp = wl.prefill_inputs(B, T, 77 + T, layer=f"r{kind}{window}")
    out, *_ = run_prefill(torch, beam, kind, inp, params)
    ref = orc.prefill(kind, oracle_params(orc, params), inp.q, inp.k, inp.v, inp.gate,
                      inp.q_norm_w, inp.k_norm_w, inp.gate_bias)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"B={B} T={T} W={window}")


@pytest.mark.parametrize("kind,T,window", [(wl.LOCAL, 1030, 512), (wl.LOCAL, 300, 100),
                                           (wl.GLOBAL, 300, 512)])
def test_prefill_masks_bit_exact(env, kind, T, window):
    """Q = 0 gives a uniform softmax over the visible keys; V is one-hot on key j0
    and the gate logits are +30 (sigmoid rounds to 1 in fp32), so an output is
    exactly zero iff j0 is invisible to that row.  The zero pattern must match the
    oracle's bit for bit; the non-zero values are 1/n within tolerance."""
    torch, beam, orc = env
    params = beam.default_params(window=window)
    inp = wl.prefill_inputs(1, T, 5, layer="mask")
    inp.q[:] = 0
    inp.gate[:] = wl.f32_to_bf16_bits(np.float32([30.0]))[0]
    inp.gate_bias[:] = 0
    for j0 in (0, T // 3, T - 1 - window // 2, T - 1):
        v = np.zeros_like(inp.v)
        v[0, j0, :] = wl.f32_to_bf16_bits(np.float32([1.0]))[0]   # every KV head, every coord
        inp.v = v
        out, *_ = run_prefill(torch, beam, kind, inp, params)
        got = as_f64(host_bits(out)).reshape(T, 48, 128)
        ref = orc.prefill(kind, oracle_params(orc, params), inp.q, inp.k, inp.v, inp.gate,
                          inp.q_norm_w, inp.k_norm_w, inp.gate_bias)[0]
        np.testing.assert_array_equal(got == 0.0, ref == 0.0)
        assert_close(host_bits(out).reshape(ref.shape), ref, f"probe j0={j0}")


def _rows_sample(B, T, seed, n_random):
    """Per sequence: both rows at every 128-row tile boundary (128k - 1, 128k), the rows
    at the window's edges (the first rows whose window is full, 510 .. 514), the first and
    last rows, and n_random seeded rows."""
    rng = np.random.default_rng(seed)
    rows = []
    edges = [0, 1, 2, 510, 511, 512, 513, 514, T - 1]
    tiles = [t for k in range(1, (T + 127) // 128) for t in (128 * k - 1, 128 * k)]
    for b in range(B):
        rnd = rng.integers(0, T, size=n_random)
        rows += [(b, int(t)) for t in sorted(set([t for t in edges + tiles if t < T] + list(rnd)))]
    return np.array([r[0] for r in rows]), np.array([r[1] for r in rows])


def _device_prefill_inputs(torch, B, T, seed, tag):
    """Full-size inputs drawn on the device (torch Philox, seeded)."""
    shapes = {"q": 48 * 128, "k": 8 * 128, "v": 8 * 128, "gate": 48 * 128}
    t = {}
    for name, width in shapes.items():
        x = torch.empty((B, T, width), dtype=torch.bfloat16, device="cuda")
        wl.device_normal_bf16_(x, seed, f"{tag}/{name}")
        t[name] = x
    inp = wl.prefill_inputs(1, 1, seed, layer=tag)  # norm weights and bias only
    return t, inp


@pytest.mark.parametrize("kind", [wl.LOCAL, wl.GLOBAL])
def test_prefill_batched_workload_sampled_rows(env, kind):
    """Batched prefill workload (B=4, T=8192) in the bench's launch configuration: over
    540 rows (every 128-row tile boundary and the window edges of each sequence, plus
    random rows), all 48 heads, against the oracle."""
    torch, beam, orc = env
    w = wl.workload("batched_prefill")
    x, inp = _device_prefill_inputs(torch, w.B, w.T, w.seed, f"bp{kind}")
    params = beam.default_params()
    qw, kw = torch.from_numpy(inp.q_norm_w).cuda(), torch.from_numpy(inp.k_norm_w).cuda()
    bias = torch.from_numpy(inp.gate_bias).cuda()
    out = torch.empty_like(x["q"])
    layout = beam.beam_kv_layout(kind, params, w.B, w.T)
    kc = torch.empty(layout.bytes_k // 2, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    beam.beam_attn_prefill(kind, params, x["q"], x["k"], x["v"], x["gate"], qw, kw, bias, out, kc,
                           vc, layout)
    torch.cuda.synchronize()
    rb, rt = _rows_sample(w.B, w.T, 3, 6)
    assert rb.size >= 512
    qh = host_bits(x["q"]); kh = host_bits(x["k"]); vh = host_bits(x["v"]); gh = host_bits(x["gate"])
    ref = orc.prefill_rows(kind, oracle_params(orc, params), qh, kh, vh, gh, inp.q_norm_w,
                           inp.k_norm_w, inp.gate_bias, rb, rt)
    got = host_bits(out)[rb, rt].reshape(ref.shape)
    assert_close(got, ref, f"batched kind={kind}")


def test_prefill_long_global_sampled_rows(env):
    """Long-context global prefill (B=1, T=131072): a(p) up to p = 131072.  A stratified
    sample of 2,048 rows: the first 512 rows with all 48 heads, then the last 512 rows and
    1,024 seeded random rows, each with the two heads of one work unit (head pair r mod
    24, so every pair is covered many times over) -- a row near the end reads 131,072
    keys, and one head pair keeps the fp64 oracle within tens of seconds."""
    torch, beam, orc = env
    w = wl.workload("long_global_prefill")
    x, inp = _device_prefill_inputs(torch, w.B, w.T, w.seed, "long")
    params = beam.default_params()
    qw, kw = torch.from_numpy(inp.q_norm_w).cuda(), torch.from_numpy(inp.k_norm_w).cuda()
    bias = torch.from_numpy(inp.gate_bias).cuda()
    out = torch.empty_like(x["q"])
    beam.beam_attn_prefill(wl.GLOBAL, params, x["q"], x["k"], x["v"], x["gate"], qw, kw, bias, out)
    torch.cuda.synchronize()
    T = w.T
    qh, kh, vh, gh = (host_bits(x[n]) for n in ("q", "k", "v", "gate"))
    got = host_bits(out)
    P = oracle_params(orc, params)
    first = np.arange(512)
    ref = orc.prefill_rows(wl.GLOBAL, P, qh, kh, vh, gh, inp.q_norm_w, inp.k_norm_w,
                           inp.gate_bias, np.zeros_like(first), first)
    assert_close(got[0, first].reshape(ref.shape), ref, "long global, first 512 rows")
    rnd = np.random.default_rng(17).choice(np.arange(512, T - 512), 1024, replace=False)
    deep = np.concatenate([np.arange(T - 512, T), np.sort(rnd)])
    pair = np.arange(deep.size) % 24
    rt = np.repeat(deep, 2)
    rh = np.stack([2 * pair, 2 * pair + 1], axis=1).ravel()
    ref = orc.prefill_row_heads(wl.GLOBAL, P, qh, kh, vh, gh, inp.q_norm_w, inp.k_norm_w,
                                inp.gate_bias, np.zeros_like(rt), rt, rh)
    g = got[0].reshape(T, 48, 128)[rt, rh]
    assert_close(g, ref, "long global, last 512 and 1,024 random rows")


# ------------------------------------------------------------------ caches
@pytest.mark.parametrize("kind,B,T", [(wl.GLOBAL, 2, 300), (wl.LOCAL, 2, 700), (wl.LOCAL, 1, 100)])
def test_prefill_fused_append_bit_exact(env, kind, B, T):
    """The prefill's fused cache append: V bits copied exactly to the right slot,
    K equal to the oracle's prepared key within one bf16 step, and untouched slots
    still holding their sentinel."""
    torch, beam, orc = env
    params = beam.default_params()
    inp = wl.prefill_inputs(B, T, 9, layer=f"app{kind}")
    _, kc, vc, layout = run_prefill(torch, beam, kind, inp, params, cache=True)
    S = layout.slots_per_seq
    kh = host_bits(kc).reshape(B, 8, S, 128)
    vh = host_bits(vc).reshape(B, 8, S, 128)
    sentinel = wl.f32_to_bf16_bits(np.float32([-7.0]))[0]
    P = oracle_params(orc, params)
    written = np.zeros((B, S), bool)
    for b in range(B):
        for t in range(max(0, T - S) if kind == wl.LOCAL else 0, T):
            s = orc.cache_slot(kind, t, S)
            kr, vr = orc.kv_row(kind, P, inp.k[b, t], inp.v[b, t], inp.k_norm_w, t)
            np.testing.assert_array_equal(vh[b, :, s], vr)
            d = np.abs(as_f64(kh[b, :, s]) - as_f64(kr))
            assert np.all(d <= np.abs(as_f64(kr)) * 2.0 ** -7 + K_ABS), (b, t)
            written[b, s] = True
    assert np.all(kh.transpose(0, 2, 1, 3)[~written] == sentinel)
    assert np.all(vh.transpose(0, 2, 1, 3)[~written] == sentinel)


@pytest.mark.parametrize("kind", [wl.GLOBAL, wl.LOCAL])
def test_kv_append_positions_bit_exact(env, kind):
    torch, beam, orc = env
    params = beam.default_params()
    B, T = 3, 600
    pos0 = np.array([0, 5, 1000], np.int64)
    cap = 2000
    layout = beam.beam_kv_layout(kind, params, B, cap)
    S = layout.slots_per_seq
    k = wl.normal_bf16((B, T, 1024), 4, "ak")
    v = wl.normal_bf16((B, T, 1024), 4, "av")
    kw = wl.norm_weight(4, "akw")
    kc = torch.full((layout.bytes_k // 2,), -7.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, -7.0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    beam.beam_kv_append(kind, params, dev(torch, k), dev(torch, v), torch.from_numpy(kw).cuda(),
                        torch.from_numpy(pos0).cuda(), kc, vc, layout, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kh = host_bits(kc).reshape(B, 8, S, 128)
    vh = host_bits(vc).reshape(B, 8, S, 128)
    P = oracle_params(orc, params)
    written = np.zeros((B, S), bool)
    for b in range(B):
        first = max(0, T - S) if kind == wl.LOCAL else 0
        for i in range(first, T):
            t = int(pos0[b]) + i
            s = orc.cache_slot(kind, t, S)
            kr, vr = orc.kv_row(kind, P, k[b, i], v[b, i], kw, t)
            np.testing.assert_array_equal(vh[b, :, s], vr)
            d = np.abs(as_f64(kh[b, :, s]) - as_f64(kr))
            assert np.all(d <= np.abs(as_f64(kr)) * 2.0 ** -7 + K_ABS), (b, i)
            written[b, s] = True
    sentinel = wl.f32_to_bf16_bits(np.float32([-7.0]))[0]
    assert np.all(vh.transpose(0, 2, 1, 3)[~written] == sentinel)
    assert np.all(kh.transpose(0, 2, 1, 3)[~written] == sentinel)


def test_kv_append_capacity_sets_status(env):
    torch, beam, orc = env
    params = beam.default_params()
    layout = beam.beam_kv_layout(wl.GLOBAL, params, 1, 10)
    k = dev(torch, wl.normal_bf16((1, 4, 1024), 1, "k"))
    kc = torch.full((layout.bytes_k // 2,), -7.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, -7.0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos0 = torch.tensor([8], dtype=torch.int64, device="cuda")
    beam.beam_kv_append(wl.GLOBAL, params, k, k, torch.ones(128, device="cuda"), pos0, kc, vc,
                        layout, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -5
    h = host_bits(vc).reshape(8, 10, 128)
    sentinel = wl.f32_to_bf16_bits(np.float32([-7.0]))[0]
    assert np.all(h[:, :8] == sentinel) and not np.any(h[:, 8:] == sentinel)


# ------------------------------------------------------------------ decode
def run_decode(torch, beam, di, params=None, status=None):
    params = params or beam.default_params()
    layout = beam.beam_kv_layout(di.kind, params, di.B, di.slots)
    kc, vc = dev(torch, di.k_cache).view(-1), dev(torch, di.v_cache).view(-1)
    out = torch.full((di.B, 48 * 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    beam.beam_attn_decode(di.kind, params, dev(torch, di.q), dev(torch, di.k), dev(torch, di.v),
                          dev(torch, di.gate), torch.from_numpy(di.q_norm_w).cuda(),
                          torch.from_numpy(di.k_norm_w).cuda(), torch.from_numpy(di.gate_bias).cuda(),
                          torch.from_numpy(di.pos).cuda(), kc, vc, layout, out, dev_status=status)
    torch.cuda.synchronize()
    return out, kc, vc


@pytest.mark.parametrize("kind", [wl.GLOBAL, wl.LOCAL])
def test_decode_edge_contexts(env, kind):
    """Contexts 1, 2, 63, 64, 65, 511, 512, 513, 1000 and 5000 visible keys (ring
    wrap-around for the local layer)."""
    torch, beam, orc = env
    ctx = np.array([1, 2, 63, 64, 65, 511, 512, 513, 1000, 5000], np.int64)
    slots = 5000 if kind == wl.GLOBAL else 512
    di = wl.decode_inputs(kind, ctx, slots, 21, layer=f"edge{kind}")
    k0, v0 = di.k_cache.copy(), di.v_cache.copy()
    out, kc, vc = run_decode(torch, beam, di)
    ref = orc.decode(kind, oracle_params(orc, beam.default_params()), di.q, di.k, di.v, di.gate,
                     di.q_norm_w, di.k_norm_w, di.gate_bias, di.pos, k0, v0)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"decode kind={kind}")
    # the new row sits at slot t (global) or t mod 512 (local); nothing else moved
    vh = host_bits(vc).reshape(di.B, 8, slots, 128)
    expect = v0.copy()
    for b, t in enumerate(di.pos):
        expect[b, :, orc.cache_slot(kind, int(t), slots)] = di.v[b].reshape(8, 128)
    np.testing.assert_array_equal(vh, expect)


def test_decode_batched_workload_all_sequences(env):
    """Batched decode workload: 64 sequences, contexts uniform in [1024, 32768],
    one local and one global layer; every output element of all 64 sequences."""
    torch, beam, orc = env
    w = wl.workload("batched_decode")
    ctx = np.array(w.ctx)
    params = beam.default_params()
    P = oracle_params(orc, params)
    for kind, slots in ((wl.GLOBAL, w.extra["global_slots"]), (wl.LOCAL, 512)):
        di = wl.decode_inputs(kind, ctx, slots, w.seed, layer=f"bd{kind}")
        k0, v0 = di.k_cache.copy(), di.v_cache.copy()
        out, *_ = run_decode(torch, beam, di)
        ref = orc.decode(kind, P, di.q, di.k, di.v, di.gate, di.q_norm_w, di.k_norm_w,
                         di.gate_bias, di.pos, k0, v0)
        assert_close(host_bits(out).reshape(ref.shape), ref, f"batched decode kind={kind}")


def test_decode_1m_context(env):
    """1M-token decode: one global layer with a 4 GiB bf16 cache (context
    1,048,576, a(p) = 513^0.1) and one local ring; cache drawn on the device."""
    torch, beam, orc = env
    params = beam.default_params()
    P = oracle_params(orc, params)
    ctx = np.array([wl.MAX_CONTEXT], np.int64)
    for kind, slots in ((wl.GLOBAL, wl.MAX_CONTEXT), (wl.LOCAL, 512)):
        di = wl.decode_inputs(kind, ctx, slots, 31, layer=f"m{kind}", with_cache=False)
        layout = beam.beam_kv_layout(kind, params, 1, slots)
        kc = torch.empty(layout.bytes_k // 2, dtype=torch.bfloat16, device="cuda")
        vc = torch.empty_like(kc)
        wl.device_normal_bf16_(kc, 31, f"m{kind}/kc")
        wl.device_normal_bf16_(vc, 31, f"m{kind}/vc")
        k0 = host_bits(kc).reshape(1, 8, slots, 128)
        v0 = host_bits(vc).reshape(1, 8, slots, 128)
        out = torch.empty((1, 6144), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        beam.beam_attn_decode(kind, params, dev(torch, di.q), dev(torch, di.k), dev(torch, di.v),
                              dev(torch, di.gate), torch.from_numpy(di.q_norm_w).cuda(),
                              torch.from_numpy(di.k_norm_w).cuda(),
                              torch.from_numpy(di.gate_bias).cuda(), torch.from_numpy(di.pos).cuda(),
                              kc, vc, layout, out, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = orc.decode(kind, P, di.q, di.k, di.v, di.gate, di.q_norm_w, di.k_norm_w,
                         di.gate_bias, di.pos, k0, v0)
        assert_close(host_bits(out).reshape(ref.shape), ref, f"1M decode kind={kind}")
        del kc, vc, k0, v0


def test_decode_position_past_capacity_sets_status(env):
    torch, beam, orc = env
    di = wl.decode_inputs(wl.GLOBAL, np.array([100, 65], np.int64), 64, 3, layer="cap")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, kc, vc = run_decode(torch, beam, di, status=status)
    assert int(status.item()) == -5
    o = host_bits(out).reshape(2, -1)
    assert np.all(np.isnan(as_f64(o)))            # untouched: still the NaN fill
    np.testing.assert_array_equal(host_bits(vc).reshape(di.v_cache.shape), di.v_cache)
