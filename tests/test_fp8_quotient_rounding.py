"""The FP8 cache code of a value is the nearest E4M3 code of the exact quotient
value / scale (the reading of the FP8 cache taken for "Beam 1.0: Local RoPE,
Global NoPE and Scalable Softmax", section "The surrounding model and serving
boundary": one scale per cache tensor, code = E4M3(value / scale)).

The device reaches that code in two roundings: the fp64 quotient is brought to
fp32 by round-to-odd (truncate, then set the last bit when anything was
dropped), and the hardware's nearest-even conversion rounds that fp32 value to
E4M3.  Round-to-odd at 24 bits followed by one nearest rounding at 4 bits equals
the nearest rounding of the fp64 quotient (Boldo and Melquiond, 2008).  This CPU
test checks the method itself in numpy, against the oracle's encoder applied to
the fp64 quotient, over values at and around every code boundary; a plain
nearest rounding to fp32 in the middle (double rounding) fails it.
"""
import numpy as np

import workloads as wl


def _round_to_odd_f32(q: np.ndarray) -> np.ndarray:
    f = q.astype(np.float32)                      # nearest
    over = np.abs(f.astype(np.float64)) > np.abs(q)
    f = np.where(over, np.nextafter(f, np.float32(0)), f)   # truncation toward zero
    inexact = f.astype(np.float64) != q
    bits = f.view(np.uint32) | inexact.astype(np.uint32)
    return bits.view(np.float32)


def _quotients():
    rng = np.random.default_rng(11)
    xs = wl.bf16_bits_to_f32(wl.normal_bf16(20000, 5, "q8x")).astype(np.float64)
    scales = np.array([0.0173, 3.7, 0.0051, 1.0 / 3.0, 0.7, 1e-3, 448.0 / 3.1], np.float32)
    q = (xs[:, None] / scales[None, :].astype(np.float64)).ravel()
    # quotients a hair off every E4M3 midpoint (where a middle rounding can go wrong)
    mags = np.array([m * 2.0 ** e for e in range(-9, 9) for m in np.arange(8, 16) + 0.5])
    eps = np.array([-3e-9, -2.0 ** -30, 0.0, 2.0 ** -30, 3e-9])
    near = (mags[:, None] * (1.0 + eps[None, :])).ravel()
    sign = np.where(rng.random(near.size) < 0.5, -1.0, 1.0)
    return np.concatenate([q, near * sign, [0.0, -0.0, 447.9, 448.0, 460.0, 1e6, -1e6]])


def test_round_to_odd_then_nearest_equals_nearest_of_the_quotient(orc):
    q = _quotients()
    via_odd = _round_to_odd_f32(q).astype(np.float64)
    got = np.array([orc.e4m3_encode(float(x)) for x in via_odd])
    ref = np.array([orc.e4m3_encode(float(x)) for x in q])
    np.testing.assert_array_equal(got, ref)


def test_a_nearest_fp32_middle_step_would_double_round(orc):
    """The same check with an ordinary nearest rounding to fp32 in the middle finds
    mismatches on the near-midpoint quotients: the round-to-odd step is needed."""
    q = _quotients()
    via_rn = q.astype(np.float32).astype(np.float64)
    got = np.array([orc.e4m3_encode(float(x)) for x in via_rn])
    ref = np.array([orc.e4m3_encode(float(x)) for x in q])
    assert (got != ref).any()
