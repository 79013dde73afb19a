"""FP8 E4M3 KV cache through the C ABI against the fp64 oracle.

Cache contents are seeded E4M3 codes given to both sides.  The FP8 decode is
compared with oracle_decode_fp8 at the parity bar of the other GPU tests.  Codes
the device writes are compared with the oracle's expected codes: value codes bit
for bit at any finite positive scale (both sides take the nearest code of the
quotient value / scale formed in fp64, rounding it once to E4M3), key codes within
one E4M3 step (the device rounds its fp32 normalised key, the oracle the exact one).
The scales include ones an amax / 448 rule gives (0.0173, 3.7, not powers of two)
and one that makes large values saturate at 448 (0.0051).  One test writes every
finite bf16 value through the append and checks each code.
"""
import numpy as np
import pytest

import workloads as wl
from test_gpu_parity import assert_close, dev, env, host_bits, oracle_params  # noqa: F401

pytestmark = pytest.mark.gpu


def _codes_close(got, ref):
    """Equal, or neighbours in the ordered code line (same sign)."""
    got, ref = got.astype(np.int32), ref.astype(np.int32)
    sg, sr = got >> 7, ref >> 7
    mg, mr = got & 0x7F, ref & 0x7F
    near = (sg == sr) & (np.abs(mg - mr) <= 1)
    zero = (mg <= 1) & (mr <= 1)        # +-0 and the smallest subnormals around zero
    return np.all(near | zero)


def _f8_layout(beam, kind, params, B, slots):
    layout = beam.beam_kv_layout_fp8(kind, params, B, slots)
    assert layout.bytes_k == B * 8 * layout.slots_per_seq * 128
    return layout


@pytest.mark.parametrize("kind", [wl.GLOBAL, wl.LOCAL])
@pytest.mark.parametrize("k_scale,v_scale", [(0.5, 1.0), (1.0, 0.25), (0.0173, 3.7),
                                             (3.7, 0.0051)])
def test_kv_append_fp8_codes(env, kind, k_scale, v_scale):
    torch, beam, orc = env
    params = beam.default_params()
    P = oracle_params(orc, params)
    B, T, cap = 3, 600, 2000
    pos0 = np.array([0, 5, 1000], np.int64)
    layout = _f8_layout(beam, kind, params, B, cap)
    S = layout.slots_per_seq
    k = wl.normal_bf16((B, T, 1024), 4, "f8k")
    v = wl.normal_bf16((B, T, 1024), 4, "f8v")
    kw = wl.norm_weight(4, "f8kw")
    kc = torch.full((layout.bytes_k,), 0x5A, dtype=torch.uint8, device="cuda")
    vc = torch.full_like(kc, 0x5A)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    beam.beam_kv_append_fp8(kind, params, dev(torch, k), dev(torch, v),
                            torch.from_numpy(kw).cuda(), torch.from_numpy(pos0).cuda(), kc, vc,
                            layout, k_scale, v_scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kh = kc.cpu().numpy().reshape(B, 8, S, 128)
    vh = vc.cpu().numpy().reshape(B, 8, S, 128)
    written = np.zeros((B, S), bool)
    for b in range(B):
        first = max(0, T - S) if kind == wl.LOCAL else 0
        for i in range(first, T):
            t = int(pos0[b]) + i
            s = orc.cache_slot(kind, t, S)
            kr, vr = orc.kv_row_fp8(kind, P, k[b, i], v[b, i], kw, t, k_scale, v_scale)
            np.testing.assert_array_equal(vh[b, :, s], vr)
            assert _codes_close(kh[b, :, s], kr), (b, t)
            written[b, s] = True
    assert np.all(kh.transpose(0, 2, 1, 3)[~written] == 0x5A)
    assert np.all(vh.transpose(0, 2, 1, 3)[~written] == 0x5A)


@pytest.mark.parametrize("v_scale", [3.7, 0.0173, 1.0, 0.0051])
def test_kv_append_fp8_every_bf16_value(env, v_scale):
    """Every finite bf16 bit pattern (non-finite ones replaced by zero) as a value, 64
    tokens of 1024: each written code must be the oracle's nearest code of value / scale --
    the ties, the subnormal codes and the saturation at 448 included."""
    torch, beam, orc = env
    params = beam.default_params()
    P = oracle_params(orc, params)
    T = 64
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = wl.bf16_bits_to_f32(bits)
    bits = np.where(np.isfinite(vals), bits, 0).astype(np.uint16)
    v = bits.reshape(1, T, 1024)
    k = wl.normal_bf16((1, T, 1024), 5, "allk")
    kw = wl.norm_weight(5, "allkw")
    layout = _f8_layout(beam, wl.GLOBAL, params, 1, T)
    kc = torch.zeros((layout.bytes_k,), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    beam.beam_kv_append_fp8(wl.GLOBAL, params, dev(torch, k), dev(torch, v),
                            torch.from_numpy(kw).cuda(),
                            torch.zeros(1, dtype=torch.int64, device="cuda"), kc, vc, layout, 1.0,
                            v_scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    vh = vc.cpu().numpy().reshape(8, T, 128).transpose(1, 0, 2)   # [token][head][d]
    for t in range(T):
        _, vr = orc.kv_row_fp8(wl.GLOBAL, P, k[0, t], v[0, t], kw, t, 1.0, v_scale)
        np.testing.assert_array_equal(vh[t].reshape(-1), vr.reshape(-1), err_msg=f"token {t}")


def run_decode_fp8(torch, beam, di, kc0, vc0, k_scale, v_scale, params=None, status=None):
    params = params or beam.default_params()
    layout = _f8_layout(beam, di.kind, params, di.B, di.slots)
    kc = torch.from_numpy(np.ascontiguousarray(kc0)).cuda().view(-1)
    vc = torch.from_numpy(np.ascontiguousarray(vc0)).cuda().view(-1)
    out = torch.full((di.B, 48 * 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    beam.beam_attn_decode_fp8(di.kind, params, dev(torch, di.q), dev(torch, di.k),
                              dev(torch, di.v), dev(torch, di.gate),
                              torch.from_numpy(di.q_norm_w).cuda(),
                              torch.from_numpy(di.k_norm_w).cuda(),
                              torch.from_numpy(di.gate_bias).cuda(),
                              torch.from_numpy(di.pos).cuda(), kc, vc, layout, k_scale, v_scale,
                              out, dev_status=status)
    torch.cuda.synchronize()
    return out, kc, vc


@pytest.mark.parametrize("kind,ctx,slots", [
    (wl.GLOBAL, [1, 2, 63, 64, 65, 700, 4097, 9000], 9000),
    (wl.LOCAL, [1, 3, 511, 512, 513, 2000, 70], 512),
])
@pytest.mark.parametrize("k_scale,v_scale", [(0.5, 2.0), (1.0, 1.0), (0.0173, 3.7),
                                             (3.7, 0.0051)])
def test_decode_fp8_matches_oracle_and_appends(env, kind, ctx, slots, k_scale, v_scale):
    torch, beam, orc = env
    params = beam.default_params()
    P = oracle_params(orc, params)
    di = wl.decode_inputs(kind, np.array(ctx, np.int64), slots, 41, layer=f"f8{kind}",
                          with_cache=False)
    shape = (di.B, 8, slots, 128)
    kc0 = wl.normal_e4m3(shape, 41, f"f8{kind}/kc", k_scale)
    vc0 = wl.normal_e4m3(shape, 41, f"f8{kind}/vc", v_scale)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, kc, vc = run_decode_fp8(torch, beam, di, kc0, vc0, k_scale, v_scale, params, status)
    assert int(status.item()) == 0
    ref = orc.decode_fp8(kind, P, di.q, di.k, di.v, di.gate, di.q_norm_w, di.k_norm_w,
                         di.gate_bias, di.pos, kc0, vc0, k_scale, v_scale)
    assert_close(host_bits(out).reshape(ref.shape), ref, f"fp8 decode kind={kind}")
    kh = kc.cpu().numpy().reshape(shape)
    vh = vc.cpu().numpy().reshape(shape)
    kexp, vexp = kc0.copy(), vc0.copy()
    for b, t in enumerate(di.pos):
        s = orc.cache_slot(kind, int(t), slots)
        kr, vr = orc.kv_row_fp8(kind, P, di.k[b], di.v[b], di.k_norm_w, int(t), k_scale, v_scale)
        assert _codes_close(kh[b, :, s], kr)
        kexp[b, :, s] = kh[b, :, s]
        vexp[b, :, s] = vr
    np.testing.assert_array_equal(vh, vexp)        # the new value codes, nothing else moved
    np.testing.assert_array_equal(kh, kexp)


def test_decode_fp8_1m_context(env):
    """1M-token decode over FP8 caches: one global layer (2 x 1 GiB of codes, context
    1,048,576) and one local ring; codes drawn on the device."""
    torch, beam, orc = env
    params = beam.default_params()
    P = oracle_params(orc, params)
    ctx = np.array([wl.MAX_CONTEXT], np.int64)
    for kind, slots in ((wl.GLOBAL, wl.MAX_CONTEXT), (wl.LOCAL, 512)):
        di = wl.decode_inputs(kind, ctx, slots, 43, layer=f"m8{kind}", with_cache=False)
        layout = _f8_layout(beam, kind, params, 1, slots)
        kc = torch.empty(layout.bytes_k, dtype=torch.uint8, device="cuda")
        vc = torch.empty_like(kc)
        wl.device_normal_e4m3_(kc, 43, f"m8{kind}/kc", 0.5)
        wl.device_normal_e4m3_(vc, 43, f"m8{kind}/vc", 1.0)
        k0 = kc.cpu().numpy().reshape(1, 8, slots, 128)
        v0 = vc.cpu().numpy().reshape(1, 8, slots, 128)
        out = torch.empty((1, 6144), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        beam.beam_attn_decode_fp8(kind, params, dev(torch, di.q), dev(torch, di.k),
                                  dev(torch, di.v), dev(torch, di.gate),
                                  torch.from_numpy(di.q_norm_w).cuda(),
                                  torch.from_numpy(di.k_norm_w).cuda(),
                                  torch.from_numpy(di.gate_bias).cuda(),
                                  torch.from_numpy(di.pos).cuda(), kc, vc, layout, 0.5, 1.0, out,
                                  dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = orc.decode_fp8(kind, P, di.q, di.k, di.v, di.gate, di.q_norm_w, di.k_norm_w,
                             di.gate_bias, di.pos, k0, v0, 0.5, 1.0)
        assert_close(host_bits(out).reshape(ref.shape), ref, f"1M fp8 decode kind={kind}")
        del kc, vc, k0, v0


def test_decode_fp8_position_past_capacity_sets_status(env):
    torch, beam, orc = env
    params = beam.default_params()
    di = wl.decode_inputs(wl.GLOBAL, np.array([11, 5], np.int64), 10, 45, layer="f8cap",
                          with_cache=False)
    shape = (2, 8, 10, 128)
    kc0 = wl.normal_e4m3(shape, 45, "f8cap/kc")
    vc0 = wl.normal_e4m3(shape, 45, "f8cap/vc")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, kc, vc = run_decode_fp8(torch, beam, di, kc0, vc0, 1.0, 1.0, params, status)
    assert int(status.item()) == -5
    o = host_bits(out)
    assert np.all(np.isnan(wl.bf16_bits_to_f32(o[0])))     # position 10 of 10 slots: untouched
    assert not np.any(np.isnan(wl.bf16_bits_to_f32(o[1])))
    np.testing.assert_array_equal(kc.cpu().numpy().reshape(shape)[0], kc0[0])
