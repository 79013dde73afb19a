"""Pins of the fp64 oracle against what the source pages and mathematics fix.

Source: "Beam 1.0: Local RoPE, Global NoPE and Scalable Softmax" (flozi.net,
English page).  Every pin is chosen so that a plausible slip in the oracle (a
wrong sign, an index off by one, a transposed pairing, a(p) applied at p = t or
squared, the wrong KV head for a query head, a per-head instead of
per-coordinate gate) fails at least one test here.
"""
import math
import os

import numpy as np
import pytest

import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _bf16(x):
    return wl.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _rand(shape, seed, tag):
    return wl.normal_bf16(shape, seed, tag)


BF16_30 = int(_bf16([30.0])[0])   # sigmoid(30) = 1 - 9.4e-14


# ---------------------------------------------------------------- a(p)
def test_ssmax_factor_printed_values(orc):
    """Section 'What scalable softmax changes mathematically' prints a(p)."""
    for p, a_printed in _golden("ssmax_factor.txt"):
        assert abs(orc.ssmax_factor(int(p)) - float(a_printed)) <= 5e-5


def test_ssmax_factor_closed_form(orc):
    assert orc.ssmax_factor(2048) == pytest.approx(2.0 ** 0.1, rel=1e-15)
    assert orc.ssmax_factor(65536) == pytest.approx(33.0 ** 0.1, rel=1e-15)
    assert orc.ssmax_factor(1048576) == pytest.approx(513.0 ** 0.1, rel=1e-15)
    assert orc.ssmax_factor(0) == 1.0


def test_global_query_uses_one_based_position(orc):
    """Only Q is scaled, by a(t+1): at t = 2047 the factor is exactly 2^0.1."""
    P = orc.params(n_q_heads=1, n_kv_heads=1, head_dim=128)
    q = _rand(128, 1, "q")
    w = np.ones(128, np.float32)
    x = np.array([orc.bf16_to_double(b) for b in q])
    plain = orc.rms_norm(x, w.astype(np.float64), 1e-6)
    got = orc.prepare_query(orc.GLOBAL, P, q, w, 2047)
    np.testing.assert_allclose(got / plain, 2.0 ** 0.1, rtol=1e-14)
    # keys of a global layer are neither rotated nor scaled
    kg = orc.prepare_key(orc.GLOBAL, P, q, w, 2047)
    np.testing.assert_allclose(kg, plain, rtol=1e-15)


# ---------------------------------------------------------------- masks
def test_window_includes_current_token_and_511_earlier(orc):
    """Section 'Two attention paths': 511 earlier positions plus the current one."""
    W = 512
    for t in (0, 1, 510, 511, 512, 600, 1029):
        n = sum(orc.visible(orc.LOCAL, t, j, W) for j in range(0, t + 2))
        assert n == min(t + 1, W)
    assert orc.visible(orc.LOCAL, 600, 89, W) and not orc.visible(orc.LOCAL, 600, 88, W)
    assert orc.visible(orc.LOCAL, 600, 600, W) and not orc.visible(orc.LOCAL, 600, 601, W)
    assert orc.visible(orc.GLOBAL, 600, 0, W) and not orc.visible(orc.GLOBAL, 600, 601, W)


@pytest.mark.parametrize("kind,W,T", [(0, 4, 12), (1, 4, 12), (0, 512, 1030)])
def test_masks_brute_force_through_attention(orc, kind, W, T):
    """Q = 0 makes the softmax uniform over the visible keys.  With V one-hot on
    one key j0 (coordinate 0) and gate logits +30, Y[t,0] = sigmoid(30)/n_t when
    j0 is visible to t and exactly 0 otherwise; n_t is counted from the page's
    rule (keys t-W+1..t local, 0..t global), independently of the oracle."""
    d = 8
    P = orc.params(n_q_heads=1, n_kv_heads=1, head_dim=d, window=W)
    q = np.zeros((1, T, d), np.uint16)
    k = _rand((1, T, d), 2, "k")
    gate = np.full((1, T, d), BF16_30, np.uint16)
    ones = np.ones(d, np.float32)
    for j0 in sorted({0, 1, T // 2, T - 2, T - 1}):
        v = np.zeros((1, T, d), np.uint16)
        v[0, j0, 0] = _bf16([1.0])[0]
        y = orc.prefill(kind, P, q, k, v, gate, ones, ones, np.zeros(1, np.float32))[0, :, 0, 0]
        for t in range(T):
            lo = max(0, t - W + 1) if kind == orc.LOCAL else 0
            n_t = t - lo + 1
            if lo <= j0 <= t:
                assert y[t] == pytest.approx(orc.sigmoid(30.0) / n_t, rel=1e-13)
            else:
                assert y[t] == 0.0


def test_window_of_one_returns_own_value(orc):
    """W = 1: only the current key is visible, so O_t = v_t."""
    T, d = 9, 8
    P = orc.params(n_q_heads=2, n_kv_heads=1, head_dim=d, window=1)
    q, k, v = _rand((1, T, 2 * d), 3, "q"), _rand((1, T, d), 3, "k"), _rand((1, T, d), 3, "v")
    gate = np.full((1, T, 2 * d), BF16_30, np.uint16)
    ones = np.ones(d, np.float32)
    y = orc.prefill(orc.LOCAL, P, q, k, v, gate, ones, ones, np.zeros(2, np.float32))
    vd = wl.bf16_bits_to_f32(v).astype(np.float64)
    for h in range(2):
        np.testing.assert_allclose(y[0, :, h, :], vd[0] * orc.sigmoid(30.0), rtol=1e-13)


def test_first_token_sees_only_itself(orc):
    d = 16
    P = orc.params(n_q_heads=4, n_kv_heads=2, head_dim=d)
    q, k, v = _rand((1, 3, 4 * d), 4, "q"), _rand((1, 3, 2 * d), 4, "k"), _rand((1, 3, 2 * d), 4, "v")
    gate = np.full((1, 3, 4 * d), BF16_30, np.uint16)
    ones = np.ones(d, np.float32)
    vd = wl.bf16_bits_to_f32(v).astype(np.float64).reshape(1, 3, 2, d)
    for kind in (orc.LOCAL, orc.GLOBAL):
        y = orc.prefill(kind, P, q, k, v, gate, ones, ones, np.zeros(4, np.float32))
        for h in range(4):
            np.testing.assert_allclose(y[0, 0, h], vd[0, 0, h // 2] * orc.sigmoid(30.0), rtol=1e-13)


# ---------------------------------------------------------------- GQA
@pytest.mark.parametrize("kind", [0, 1])
def test_gqa_equals_explicitly_repeated_kv(orc, kind):
    """Section 'Follow the tensors': six query heads share each KV head without
    stored copies.  Grouped attention (Hq=6 over Hkv=2) equals attention with
    each query head given its own copy of KV head h // 3."""
    T, d = 20, 16
    Pg = orc.params(n_q_heads=6, n_kv_heads=2, head_dim=d, window=7)
    Pr = orc.params(n_q_heads=6, n_kv_heads=6, head_dim=d, window=7)
    q, gate = _rand((1, T, 6 * d), 5, "q"), _rand((1, T, 6 * d), 5, "g")
    k, v = _rand((1, T, 2, d), 5, "k"), _rand((1, T, 2, d), 5, "v")
    kr = np.repeat(k, 3, axis=2)
    vr = np.repeat(v, 3, axis=2)
    w1, w2 = wl.norm_weight(5, "qw")[:d], wl.norm_weight(5, "kw")[:d]
    bias = np.linspace(-1, 1, 6).astype(np.float32)
    yg = orc.prefill(kind, Pg, q, k.reshape(1, T, -1), v.reshape(1, T, -1), gate, w1, w2, bias)
    yr = orc.prefill(kind, Pr, q, kr.reshape(1, T, -1), vr.reshape(1, T, -1), gate, w1, w2, bias)
    np.testing.assert_allclose(yg, yr, rtol=1e-13, atol=1e-15)
    # and the grouping is by contiguous blocks, not h % Hkv
    vr_bad = np.tile(v, (1, 1, 3, 1))
    kr_bad = np.tile(k, (1, 1, 3, 1))
    yb = orc.prefill(kind, Pr, q, kr_bad.reshape(1, T, -1), vr_bad.reshape(1, T, -1), gate, w1, w2, bias)
    assert np.max(np.abs(yb - yg)) > 1e-2


@pytest.mark.parametrize("kind", [wl.LOCAL, wl.GLOBAL])
def test_single_head_items_equal_repeated_kv_rows(orc, kind):
    """prefill_row_heads (one query head per item) against the full-row function run
    with every query head given its own copy of KV head h // 3: the item's head picks
    both its KV head and its output, so a wrong mapping or index fails here."""
    T, d = 30, 16
    Pg = orc.params(n_q_heads=6, n_kv_heads=2, head_dim=d, window=9)
    Pr = orc.params(n_q_heads=6, n_kv_heads=6, head_dim=d, window=9)
    q, gate = _rand((2, T, 6 * d), 8, "q"), _rand((2, T, 6 * d), 8, "g")
    k, v = _rand((2, T, 2, d), 8, "k"), _rand((2, T, 2, d), 8, "v")
    kr, vr = np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2)
    w1, w2 = wl.norm_weight(8, "qw")[:d], wl.norm_weight(8, "kw")[:d]
    bias = np.linspace(-1, 1, 6).astype(np.float32)
    rng = np.random.default_rng(4)
    rb, rt, rh = rng.integers(0, 2, 40), rng.integers(0, T, 40), rng.integers(0, 6, 40)
    got = orc.prefill_row_heads(kind, Pg, q, k.reshape(2, T, -1), v.reshape(2, T, -1), gate, w1,
                                w2, bias, rb, rt, rh)
    full = orc.prefill_rows(kind, Pr, q, kr.reshape(2, T, -1), vr.reshape(2, T, -1), gate, w1, w2,
                            bias, rb, rt)
    np.testing.assert_allclose(got, full[np.arange(40), rh], rtol=1e-13, atol=1e-15)


def test_single_head_items_window_of_one_closed_form(orc):
    """Window 1: each item is its own value row of KV head h // 6, gated per
    coordinate with its head's bias -- written out in numpy."""
    T = 12
    P = orc.params(window=1)
    inp = wl.prefill_inputs(1, T, 3, layer="w1heads")
    rt = np.arange(T)
    rh = (7 * rt + 5) % 48
    got = orc.prefill_row_heads(wl.LOCAL, P, inp.q, inp.k, inp.v, inp.gate, inp.q_norm_w,
                                inp.k_norm_w, inp.gate_bias, np.zeros(T, np.int64), rt, rh)
    v = wl.bf16_bits_to_f32(inp.v[0]).astype(np.float64).reshape(T, 8, 128)
    g = wl.bf16_bits_to_f32(inp.gate[0]).astype(np.float64).reshape(T, 48, 128)
    expect = v[rt, rh // 6] / (1.0 + np.exp(-(g[rt, rh] + inp.gate_bias[rh][:, None])))
    np.testing.assert_allclose(got, expect, rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------- softmax
def test_softmax_toy_distractor_model(orc):
    """Section 'What scalable softmax changes mathematically': P ~ 6.17e-6."""
    (delta, a, n, p_printed), = _golden("toy_probability.txt")
    n = int(n)
    s = np.zeros(n)
    s[0] = float(a) * float(delta)
    p = orc.softmax(s)
    assert abs(p[0] - float(p_printed)) <= 0.005e-6
    assert p[1] == pytest.approx(p[-1])
    assert p.sum() == pytest.approx(1.0, abs=1e-9)   # 2^20 terms summed in double


def test_softmax_rows_sum_to_one_and_sharpen_with_a(orc):
    """Rows sum to 1; H(a) = log Z(a) - a E[z] does not increase with a (its
    derivative is -a Var(z)), and the arg max does not move."""
    z = np.random.default_rng(7).standard_normal(257)
    ents = []
    for a in np.linspace(0.25, 3.0, 12):
        p = orc.softmax(a * z)
        assert abs(1.0 - p.sum()) < 1e-12
        assert int(np.argmax(p)) == int(np.argmax(z))
        ents.append(-(p * np.log(p)).sum())
    assert all(e2 <= e1 + 1e-12 for e1, e2 in zip(ents, ents[1:]))
    # finite-difference derivative equals -a Var_pi(z)
    a, h = 1.4, 1e-5
    Hs = [-(p * np.log(p)).sum() for p in (orc.softmax((a - h) * z), orc.softmax((a + h) * z))]
    p = orc.softmax(a * z)
    var = (p * z * z).sum() - (p * z).sum() ** 2
    assert (Hs[1] - Hs[0]) / (2 * h) == pytest.approx(-a * var, rel=1e-6)


def test_constant_values_give_constant_output(orc):
    T, d = 30, 16
    P = orc.params(n_q_heads=4, n_kv_heads=2, head_dim=d, window=5)
    q, k = _rand((1, T, 4 * d), 8, "q"), _rand((1, T, 2 * d), 8, "k")
    v = np.full((1, T, 2 * d), _bf16([0.75])[0], np.uint16)
    gate = np.full((1, T, 4 * d), BF16_30, np.uint16)
    w = wl.norm_weight(8, "w")[:d]
    for kind in (orc.LOCAL, orc.GLOBAL):
        y = orc.prefill(kind, P, q, k, v, gate, w, w, np.zeros(4, np.float32))
        np.testing.assert_allclose(y, 0.75 * orc.sigmoid(30.0), rtol=1e-13)


def test_ssmax_scales_logits_linearly_two_keys(orc):
    """Two visible keys with hand-computable normalised dot products.  With
    w = 1, q = (1,1,1,1), k0 = q, k1 = (1,-1,1,-1): <q^,k0^> = 4/(1+eps),
    <q^,k1^> = 0, so log(P0/P1) = a(p) * scale * 4/(1+eps) at p = t+1 = 2 for a
    global layer.  Scaling K as well, or using p = t, would change the ratio."""
    d = 4
    P = orc.params(n_q_heads=1, n_kv_heads=1, head_dim=d, softmax_scale=0.5)
    one, m1 = _bf16([1.0])[0], _bf16([-1.0])[0]
    q = np.full((1, 2, d), one, np.uint16)
    k = np.array([[[one] * 4, [one, m1, one, m1]]], np.uint16)
    v = np.zeros((1, 2, d), np.uint16)
    v[0, 0, 0] = one
    v[0, 1, 1] = one
    gate = np.full((1, 2, d), BF16_30, np.uint16)
    w = np.ones(d, np.float32)
    y = orc.prefill(orc.GLOBAL, P, q, k, v, gate, w, w, np.zeros(1, np.float32))[0, 1, 0]
    expect = orc.ssmax_factor(2) * 0.5 * 4.0 / (1.0 + 1e-6)
    assert math.log(y[0] / y[1]) == pytest.approx(expect, rel=1e-12)
    assert y[0] + y[1] == pytest.approx(orc.sigmoid(30.0), rel=1e-13)


# ---------------------------------------------------------------- RoPE
def test_rope_rotate_half_closed_form(orc):
    """Unit vector e_i maps to cos(t f_i) e_i + sin(t f_i) e_{i+64}, f_i = 10000^(-2i/128);
    e_{i+64} maps to -sin(t f_i) e_i + cos(t f_i) e_{i+64}."""
    d = 128
    for i in (0, 1, 17, 63):
        f = 10000.0 ** (-2.0 * i / d)
        for t in (0, 1, 5, 1000, 1048575):
            e = np.zeros(d)
            e[i] = 1.0
            y = orc.rope(e, t)
            expect = np.zeros(d)
            expect[i], expect[i + 64] = math.cos(t * f), math.sin(t * f)
            np.testing.assert_allclose(y, expect, atol=1e-12)
            e = np.zeros(d)
            e[i + 64] = 1.0
            y = orc.rope(e, t)
            expect = np.zeros(d)
            expect[i], expect[i + 64] = -math.sin(t * f), math.cos(t * f)
            np.testing.assert_allclose(y, expect, atol=1e-12)


def test_rope_preserves_norm_and_depends_on_offset_only(orc):
    rng = np.random.default_rng(3)
    x = rng.standard_normal(128)
    for t in (0, 3, 511, 8191, 1048575):
        assert np.linalg.norm(orc.rope(x, t)) == pytest.approx(np.linalg.norm(x), rel=1e-13)
    np.testing.assert_array_equal(orc.rope(x, 0), x)
    y = rng.standard_normal(128)
    for (t, j, delta) in ((5, 2, 100), (600, 89, 7000), (1000, 999, 1047000)):
        s0 = orc.rope(x, t) @ orc.rope(y, j)
        s1 = orc.rope(x, t + delta) @ orc.rope(y, j + delta)
        assert s1 == pytest.approx(s0, rel=1e-9, abs=1e-9)


def test_local_query_and_key_are_normalised_then_rotated(orc):
    P = orc.params(n_q_heads=1, n_kv_heads=1, head_dim=128)
    q = _rand(128, 9, "q")
    w = wl.norm_weight(9, "w")
    x = np.array([orc.bf16_to_double(b) for b in q])
    expect = orc.rope(orc.rms_norm(x, w.astype(np.float64)), 77)
    np.testing.assert_allclose(orc.prepare_query(orc.LOCAL, P, q, w, 77), expect, rtol=1e-14)
    np.testing.assert_allclose(orc.prepare_key(orc.LOCAL, P, q, w, 77), expect, rtol=1e-14)


# ---------------------------------------------------------------- RMSNorm
def test_rms_norm_closed_forms(orc):
    w = np.linspace(0.5, 1.5, 2)
    y = orc.rms_norm([3.0, 4.0], w, 1e-6)
    s = 1.0 / math.sqrt(12.5 + 1e-6)
    np.testing.assert_allclose(y, [3.0 * s * 0.5, 4.0 * s * 1.5], rtol=1e-15)
    x = np.full(128, 2.0)
    np.testing.assert_allclose(orc.rms_norm(x, np.ones(128)), 2.0 / math.sqrt(4.0 + 1e-6), rtol=1e-15)
    z = orc.rms_norm(np.zeros(128), np.ones(128))
    assert np.all(z == 0.0)
    # scale invariance up to epsilon
    r = np.random.default_rng(1).standard_normal(128)
    np.testing.assert_allclose(orc.rms_norm(r * 1000, np.ones(128)), orc.rms_norm(r, np.ones(128)),
                               rtol=2e-6)


# ---------------------------------------------------------------- gate
def test_gate_bias_per_head_and_gate_per_coordinate(orc):
    """Section 'Follow the tensors': only the additive bias is one value per
    head; the gate has one logit per coordinate."""
    T, d, H = 6, 8, 4
    P = orc.params(n_q_heads=H, n_kv_heads=2, head_dim=d)
    q, k, v = _rand((1, T, H * d), 10, "q"), _rand((1, T, 2 * d), 10, "k"), _rand((1, T, 2 * d), 10, "v")
    w = np.ones(d, np.float32)
    zero_gate = np.zeros((1, T, H * d), np.uint16)
    base = orc.prefill(orc.GLOBAL, P, q, k, v, zero_gate, w, w, np.zeros(H, np.float32))
    bias = np.log(np.arange(1, H + 1)).astype(np.float32)
    yb = orc.prefill(orc.GLOBAL, P, q, k, v, zero_gate, w, w, bias)
    for h in range(H):
        s = 1.0 / (1.0 + math.exp(-float(bias[h])))
        np.testing.assert_allclose(yb[0, :, h], base[0, :, h] * 2.0 * s, rtol=1e-13)
    g = zero_gate.copy()
    c = 5
    g[0, :, 2 * d + c] = _bf16([2.0])[0]      # head 2, coordinate 5
    yg = orc.prefill(orc.GLOBAL, P, q, k, v, g, w, w, np.zeros(H, np.float32))
    ratio = yg / base
    np.testing.assert_allclose(ratio[0, :, 2, c], 2.0 / (1.0 + math.exp(-2.0)), rtol=1e-12)
    mask = np.ones_like(ratio, bool)
    mask[0, :, 2, c] = False
    np.testing.assert_allclose(ratio[mask], 1.0, rtol=1e-12)


# ---------------------------------------------------------------- decode vs prefill
@pytest.mark.parametrize("kind,T", [(0, 21), (0, 5), (1, 21)])
def test_decode_after_cache_fill_matches_prefill(orc, kind, T):
    """Fill a cache with the oracle's own per-token rows (bf16), one token at a
    time, then decode the last token: the result equals the prefill's last row
    up to the bf16 rounding of the cached keys.  A wrong ring slot, position or
    append order changes the result by far more."""
    d, Hq, Hkv, W = 16, 6, 2, 8
    P = orc.params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, window=W)
    q, gate = _rand((1, T, Hq * d), 11, "q"), _rand((1, T, Hq * d), 11, "g")
    k, v = _rand((1, T, Hkv * d), 11, "k"), _rand((1, T, Hkv * d), 11, "v")
    qw, kw = wl.norm_weight(11, "qw")[:d], wl.norm_weight(11, "kw")[:d]
    bias = np.linspace(-0.5, 0.5, Hq).astype(np.float32)
    ref = orc.prefill(kind, P, q, k, v, gate, qw, kw, bias)[0, T - 1]
    slots = W if kind == orc.LOCAL else T
    kc = np.zeros((1, Hkv, slots, d), np.uint16)
    vc = np.zeros_like(kc)
    for j in range(T - 1):
        kr, vr = orc.kv_row(kind, P, k[0, j], v[0, j], kw, j)
        s = orc.cache_slot(kind, j, slots)
        kc[0, :, s], vc[0, :, s] = kr, vr
    t = T - 1
    out = orc.decode(kind, P, q[:, t], k[:, t], v[:, t], gate[:, t], qw, kw, bias,
                     np.array([t]), kc, vc)[0]
    np.testing.assert_allclose(out, ref, rtol=2e-2, atol=2e-2)
    # the same decode with the ring read at the wrong slot differs clearly
    if kind == orc.LOCAL and T > W:
        kc2 = np.roll(kc, 1, axis=2)
        vc2 = np.roll(vc, 1, axis=2)
        bad = orc.decode(kind, P, q[:, t], k[:, t], v[:, t], gate[:, t], qw, kw, bias,
                         np.array([t]), kc2, vc2)[0]
        assert np.max(np.abs(bad - ref)) > 0.05


# ---------------------------------------------------------------- chunked prefill
def _small_chunk_problem(B, T, seed, d=16, Hq=6, Hkv=2):
    q, gate = _rand((B, T, Hq * d), seed, "q"), _rand((B, T, Hq * d), seed, "g")
    k, v = _rand((B, T, Hkv * d), seed, "k"), _rand((B, T, Hkv * d), seed, "v")
    qw, kw = wl.norm_weight(seed, "qw")[:d], wl.norm_weight(seed, "kw")[:d]
    bias = np.linspace(-0.5, 0.5, Hq).astype(np.float32)
    return q, k, v, gate, qw, kw, bias


@pytest.mark.parametrize("kind", [0, 1])
def test_chunk_of_one_token_equals_decode(orc, kind):
    """A chunk of one new token is a decode step: same visible keys, same cache
    slots, the new key prepared exactly.  Decode itself is pinned above."""
    d, Hq, Hkv, W = 16, 6, 2, 8
    P = orc.params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, window=W)
    pos = np.array([0, 3, 8, 29], np.int64)
    B, slots = pos.size, (W if kind == orc.LOCAL else 40)
    q, k, v, gate, qw, kw, bias = _small_chunk_problem(B, 1, 21)
    kc = _rand((B, Hkv, slots, d), 21, "kc")
    vc = _rand((B, Hkv, slots, d), 21, "vc")
    got = orc.prefill_chunk(kind, P, q, k, v, gate, qw, kw, bias, pos, kc, vc)[:, 0]
    ref = orc.decode(kind, P, q[:, 0], k[:, 0], v[:, 0], gate[:, 0], qw, kw, bias, pos, kc, vc)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("kind", [0, 1])
def test_chunk_at_position_zero_equals_prefill_and_reads_no_cache(orc, kind):
    """With pos0 = 0 nothing is cached yet: the chunk is a plain prefill, whatever
    the cache buffer holds."""
    d, Hq, Hkv, W = 16, 6, 2, 8
    P = orc.params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, window=W)
    B, T = 2, 19
    q, k, v, gate, qw, kw, bias = _small_chunk_problem(B, T, 22)
    slots = W if kind == orc.LOCAL else T
    kc = np.full((B, Hkv, slots, d), _bf16([1e30])[0], np.uint16)   # poison
    vc = kc.copy()
    got = orc.prefill_chunk(kind, P, q, k, v, gate, qw, kw, bias, np.zeros(B, np.int64), kc, vc)
    ref = orc.prefill(kind, P, q, k, v, gate, qw, kw, bias)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("kind", [0, 1])
def test_chunk_after_cache_fill_matches_prefill(orc, kind):
    """Sequence b's first P_b tokens go into the cache as the oracle's own rows
    (bf16), then the remaining tokens arrive as one chunk: every chunk row equals
    the one-shot prefill row at the same position, up to the bf16 rounding of the
    cached keys.  The ring at the wrong slot, or the chunk's positions off by
    one, differ by far more."""
    d, Hq, Hkv, W = 16, 6, 2, 8
    P = orc.params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, window=W)
    B, Ttot = 2, 27
    pos0 = np.array([5, 13], np.int64)            # chunk lengths 22 and 14: use T = 14
    T = 14
    q, k, v, gate, qw, kw, bias = _small_chunk_problem(B, Ttot, 23)
    ref = orc.prefill(kind, P, q, k, v, gate, qw, kw, bias)
    slots = W if kind == orc.LOCAL else Ttot + 1   # room for the shifted call below
    kc = np.zeros((B, Hkv, slots, d), np.uint16)
    vc = np.zeros_like(kc)
    for b in range(B):
        for j in range(pos0[b]):
            kr, vr = orc.kv_row(kind, P, k[b, j], v[b, j], kw, j)
            s = orc.cache_slot(kind, j, slots)
            kc[b, :, s], vc[b, :, s] = kr, vr
    sl = [np.stack([x[b, pos0[b]:pos0[b] + T] for b in range(B)]) for x in (q, k, v, gate)]
    got = orc.prefill_chunk(kind, P, *sl, qw, kw, bias, pos0, kc, vc)
    want = np.stack([ref[b, pos0[b]:pos0[b] + T] for b in range(B)])
    np.testing.assert_allclose(got, want, rtol=2e-2, atol=2e-2)
    if kind == orc.LOCAL:
        bad = orc.prefill_chunk(kind, P, *sl, qw, kw, bias, pos0, np.roll(kc, 1, axis=2),
                                np.roll(vc, 1, axis=2))
        assert np.max(np.abs(bad[:, 0] - want[:, 0])) > 0.05
    shifted = orc.prefill_chunk(kind, P, *sl, qw, kw, bias, pos0 + 1, kc, vc)
    assert np.max(np.abs(shifted - want)) > 0.05


# ---------------------------------------------------------------- FP8 E4M3 cache
def _torch_e4m3(codes):
    import torch
    t = torch.tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_e4m3_decode_matches_library_and_format_facts(orc):
    """All 256 codes against PyTorch's float8_e4m3fn, and the format's fixed points:
    largest 448, smallest normal 2^-6, smallest subnormal 2^-9, 1.0 = 0x38, NaN only at
    S.1111.111, strictly increasing over 0x00 .. 0x7E, sign symmetric."""
    got = np.array([orc.e4m3_decode(c) for c in range(256)])
    ref = _torch_e4m3(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and set(np.flatnonzero(nan)) == {0x7F, 0xFF}
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x08] == 2.0 ** -6 and got[0x01] == 2.0 ** -9
    assert got[0x38] == 1.0 and got[0xB8] == -1.0
    assert np.all(np.diff(got[:0x7F]) > 0)
    np.testing.assert_array_equal(got[0x80:0xFF], -got[0x00:0x7F])


def test_e4m3_encode_rounds_to_nearest_even_and_saturates(orc):
    vals = np.array([orc.e4m3_decode(c) for c in range(0x7F)])
    for c in range(0x7F):
        assert orc.e4m3_encode(vals[c]) == c
        assert orc.e4m3_encode(-vals[c]) == (c | 0x80)
    for c in range(0x7E):          # midpoints go to the even code, just off them to the nearer
        mid = 0.5 * (vals[c] + vals[c + 1])
        assert orc.e4m3_encode(mid) == (c if c % 2 == 0 else c + 1), hex(c)
        assert orc.e4m3_encode(np.nextafter(mid, 0)) == c
        assert orc.e4m3_encode(np.nextafter(mid, 1e9)) == c + 1
    for x, code in ((448.0, 0x7E), (460.0, 0x7E), (1000.0, 0x7E), (-1e9, 0xFE), (1e-30, 0x00)):
        assert orc.e4m3_encode(x) == code
    # agrees with PyTorch's float -> float8_e4m3fn conversion inside the finite range
    import torch
    r = np.random.default_rng(5).standard_normal(4000) * np.exp(np.random.default_rng(6)
                                                                 .uniform(-8, 5, 4000))
    r = r[np.abs(r) < 440]
    lib = torch.tensor(r).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([orc.e4m3_encode(x) for x in r], np.uint8)
    np.testing.assert_array_equal(mine, lib)


def _fp8_problem(B, seed, d=16, Hq=6, Hkv=2):
    q, gate = _rand((B, Hq * d), seed, "q"), _rand((B, Hq * d), seed, "g")
    k, v = _rand((B, Hkv * d), seed, "k"), _rand((B, Hkv * d), seed, "v")
    qw, kw = wl.norm_weight(seed, "qw")[:d], wl.norm_weight(seed, "kw")[:d]
    bias = np.linspace(-0.5, 0.5, Hq).astype(np.float32)
    return q, k, v, gate, qw, kw, bias


def _grid_bf16(orc, codes, scale):
    """bf16 bits of E4M3^-1(code) * scale (exact for a power-of-two scale)."""
    vals = np.vectorize(orc.e4m3_decode)(codes) * scale
    return _bf16(vals.astype(np.float32))


@pytest.mark.parametrize("kind", [0, 1])
def test_decode_fp8_equals_bf16_decode_of_the_dequantised_cache(orc, kind):
    """With the new token's key zero (RMSNorm keeps it zero, an exact code) and its
    value on the E4M3 grid, the FP8 decode is the BF16 decode of a cache holding the
    dequantised codes: same slots, same scales (k_scale 2, v_scale 1/2)."""
    d, Hq, Hkv, W = 16, 6, 2, 8
    P = orc.params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, window=W)
    pos = np.array([0, 3, 8, 29], np.int64)
    B, slots = pos.size, (W if kind == orc.LOCAL else 40)
    q, k, v, gate, qw, kw, bias = _fp8_problem(B, 31)
    k[:] = 0
    rng = np.random.default_rng(7)
    vcodes_new = rng.integers(0, 0x7F, size=v.shape).astype(np.uint8) | \
        (rng.integers(0, 2, size=v.shape).astype(np.uint8) << 7)
    v = _grid_bf16(orc, vcodes_new, 0.5)      # exactly representable after / 0.5
    kc = rng.integers(0, 256, size=(B, Hkv, slots, d)).astype(np.uint8)
    vc = rng.integers(0, 256, size=(B, Hkv, slots, d)).astype(np.uint8)
    for c in (kc, vc):
        c[(c & 0x7F) == 0x7F] ^= 0x01        # no NaN codes
    got = orc.decode_fp8(kind, P, q, k, v, gate, qw, kw, bias, pos, kc, vc, 2.0, 0.5)
    ref = orc.decode(kind, P, q, k, v, gate, qw, kw, bias, pos, _grid_bf16(orc, kc, 2.0),
                     _grid_bf16(orc, vc, 0.5))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_decode_fp8_window_of_one_is_the_quantised_new_value(orc):
    """W = 1: the output is the new token's value read back from its code, gated."""
    d, Hq, Hkv = 16, 6, 2
    P = orc.params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, window=1)
    q, k, v, gate, qw, kw, bias = _fp8_problem(2, 32)
    kc = np.zeros((2, Hkv, 1, d), np.uint8)
    pos = np.array([0, 77], np.int64)
    vs = 0.75
    got = orc.decode_fp8(orc.LOCAL, P, q, k, v, gate, qw, kw, bias, pos, kc, kc, 1.0, vs)
    vf = wl.bf16_bits_to_f32(v).astype(np.float64).reshape(2, Hkv, d)
    deq = np.vectorize(lambda x: orc.e4m3_decode(orc.e4m3_encode(x / vs)) * vs)(vf)
    assert np.max(np.abs(deq - vf)) > 0            # the quantisation is visible
    g = wl.bf16_bits_to_f32(gate).astype(np.float64).reshape(2, Hq, d)
    sig = 1.0 / (1.0 + np.exp(-(g + bias[None, :, None])))
    ref = deq[:, np.arange(Hq) // (Hq // Hkv)] * sig
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def _nan_free_codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 0x01        # no NaN codes
    return c


@pytest.mark.parametrize("kind", [0, 1])
def test_chunk_fp8_of_one_token_equals_fp8_decode(orc, kind):
    """A one-token chunk over FP8 caches is an FP8 decode step (pinned above): the new
    key and value quantised first, cached codes read back with their scales.  Scales
    that are not powers of two (an amax / 448 rule gives such)."""
    d, Hq, Hkv, W = 16, 6, 2, 8
    P = orc.params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, window=W)
    pos = np.array([0, 3, 8, 29], np.int64)
    B, slots = pos.size, (W if kind == orc.LOCAL else 40)
    q, k, v, gate, qw, kw, bias = _small_chunk_problem(B, 1, 23)
    rng = np.random.default_rng(23)
    kc, vc = _nan_free_codes(rng, (B, Hkv, slots, d)), _nan_free_codes(rng, (B, Hkv, slots, d))
    ks, vs = 0.0173, 3.7
    got = orc.prefill_chunk_fp8(kind, P, q, k, v, gate, qw, kw, bias, pos, kc, vc, ks, vs)[:, 0]
    ref = orc.decode_fp8(kind, P, q[:, 0], k[:, 0], v[:, 0], gate[:, 0], qw, kw, bias, pos, kc,
                         vc, ks, vs)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("kind", [0, 1])
def test_chunk_fp8_equals_bf16_chunk_of_the_dequantised_cache(orc, kind):
    """With the chunk's keys zero (RMSNorm keeps them zero, an exact code) and its values
    on the E4M3 grid, the FP8 chunk is the BF16 chunk (pinned above) over caches holding
    the dequantised codes: same slots, windows across the ring's wrap, power-of-two
    scales (2 and 1/2) so the dequantised values are exact in bf16."""
    d, Hq, Hkv, W, T = 16, 6, 2, 8, 5
    P = orc.params(n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, window=W)
    pos0 = np.array([0, 3, 8, 29], np.int64)
    B, slots = pos0.size, (W if kind == orc.LOCAL else 40)
    q, k, v, gate, qw, kw, bias = _small_chunk_problem(B, T, 24)
    k[:] = 0
    rng = np.random.default_rng(24)
    v = _grid_bf16(orc, _nan_free_codes(rng, v.shape), 0.5)
    kc, vc = _nan_free_codes(rng, (B, Hkv, slots, d)), _nan_free_codes(rng, (B, Hkv, slots, d))
    got = orc.prefill_chunk_fp8(kind, P, q, k, v, gate, qw, kw, bias, pos0, kc, vc, 2.0, 0.5)
    ref = orc.prefill_chunk(kind, P, q, k, v, gate, qw, kw, bias, pos0, _grid_bf16(orc, kc, 2.0),
                            _grid_bf16(orc, vc, 0.5))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_kv_row_fp8_codes_are_nearest_to_the_exact_rows(orc):
    """Each code's value is within half an E4M3 step of the exact prepared key / raw
    value (relative 2^-4 in the normal range); a value on the grid is exact."""
    d, Hkv = 16, 2
    P = orc.params(n_q_heads=6, n_kv_heads=Hkv, head_dim=d, window=8)
    k, v = _rand((Hkv * d,), 33, "k"), _rand((Hkv * d,), 33, "v")
    kw = wl.norm_weight(33, "kw")[:d]
    for kind in (0, 1):
        kr, vr = orc.kv_row_fp8(kind, P, k, v, kw, 5, 0.5, 2.0)
        exact_k = np.stack([orc.prepare_key(kind, P, k[g * d:(g + 1) * d], kw, 5)
                            for g in range(Hkv)])
        exact_v = wl.bf16_bits_to_f32(v).astype(np.float64).reshape(Hkv, d)
        for codes, exact, sc in ((kr, exact_k, 0.5), (vr, exact_v, 2.0)):
            deq = np.vectorize(orc.e4m3_decode)(codes) * sc
            assert np.all(np.abs(deq - exact) <= np.maximum(np.abs(exact) * 2.0 ** -4,
                                                             2.0 ** -10 * sc) * 1.0000001)
    grid = _grid_bf16(orc, np.arange(0x30, 0x50, dtype=np.uint8)[:Hkv * d], 1.0)
    _, vr = orc.kv_row_fp8(1, P, k, grid, kw, 0, 1.0, 1.0)
    np.testing.assert_array_equal(vr.ravel(), np.arange(0x30, 0x50, dtype=np.uint8)[:Hkv * d])


# ---------------------------------------------------------------- bf16
def test_bf16_rounding_ties_to_even(orc):
    cases = {1.0 + 2.0 ** -8: 0x3F80, 1.0 + 3 * 2.0 ** -8: 0x3F82, -2.5: 0xC020,
             1.0 + 2.0 ** -8 + 2.0 ** -20: 0x3F81, 3.140625: 0x4049}
    for x, bits in cases.items():
        assert orc.double_to_bf16(x) == bits
    r = np.random.default_rng(2).standard_normal(2000).astype(np.float32)
    ref = wl.f32_to_bf16_bits(r)
    got = np.array([orc.double_to_bf16(float(x)) for x in r], np.uint16)
    np.testing.assert_array_equal(got, ref)
    for b in (0x3F80, 0xC020, 0x0001, 0x7F7F):
        assert orc.double_to_bf16(orc.bf16_to_double(b)) == b
