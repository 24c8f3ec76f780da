"""The FMA-pipe exp2 used for part of the forward softmax, restated in numpy
float32 exactly as the kernel evaluates it (range reduction with 1.5 * 2^23,
degree-3 Horner polynomial, exponent add), checked against exp2 in fp64."""
import numpy as np

C = np.array([0.9999280571937561, 0.6932609677314758, 0.2426111251115799, 0.0551716685295105],
             dtype=np.float32)
MAGIC = np.float32(12582912.0)


def exp2_poly3(x):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + MAGIC).astype(np.float32)
    f = (x - (t - MAGIC).astype(np.float32)).astype(np.float32)
    p = ((C[3] * f + C[2]).astype(np.float32) * f + C[1]).astype(np.float32)
    p = (p * f + C[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_relative_error_over_softmax_range():
    # The kernel feeds x = s*scale*log2e - m with x <= 8 (lazy rescale bound);
    # below -125 results sit at the bottom of the normal range (~1e-38) where
    # only the clamp matters.
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_poly3(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1e-4  # far below bf16 rounding of P (2^-9)


def test_integer_and_half_points():
    for n in range(-120, 9):
        for fr in (-0.5, -0.25, 0.0, 0.25, 0.4999):
            x = np.float32(n + fr)
            assert abs(float(exp2_poly3(x)) / 2.0 ** float(x) - 1.0) < 1e-4


def test_underflow_is_clamped_not_wrapped():
    y = exp2_poly3(np.array([-200.0, -1e30, -126.0], dtype=np.float32))
    assert np.all(y > 0) and np.all(y < 2e-38)
