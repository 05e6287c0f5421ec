"""The attention softmax evaluates a quarter of its 2^x on the FMA pipe
(range reduction x = j + f, |f| <= 1/2, degree-3 polynomial for 2^f, 2^j added
to the exponent field).  This restates those float32 steps with the kernel's
constants and checks the relative error against the mathematical 2^x over
the input range the softmax feeds it (scores minus the running max, at most
8 above it, clamped below), and that masked scores give zero in fp16."""
import numpy as np

C0, C1, C2, C3 = np.float32(0.9999280572), np.float32(0.6932609677), np.float32(0.2426111251), np.float32(0.0551716685)
SHIFT = np.float32(12582912.0)   # 1.5 * 2^23


def ex2_poly(x):
    x = np.maximum(np.float32(x), np.float32(-125.0)).astype(np.float32)
    t = (x + SHIFT).astype(np.float32)
    f = (x - (t - SHIFT).astype(np.float32)).astype(np.float32)
    q = (C3 * f + C2).astype(np.float32)
    q = (q * f + C1).astype(np.float32)
    q = (q * f + C0).astype(np.float32)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-24.0, 8.0, 400001, dtype=np.float32)   # below 2^-24 fp16 P is zero anyway
    got = ex2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()          # fp16 rounding of P is 4.9e-4 relative


def test_integers_and_halves_exact_enough():
    for j in range(-20, 9):
        for off in (0.0, 0.5, -0.5, 0.25):
            x = np.float32(j + off)
            assert abs(float(ex2_poly(x)) / 2.0 ** float(x) - 1.0) < 1e-4


def test_masked_scores_vanish_in_fp16():
    got = ex2_poly(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(got.astype(np.float16) == 0)
    assert np.all(np.isfinite(got))
