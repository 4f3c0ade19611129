"""The kernels keep the step count t in device memory and evaluate the bias corrections by binary
exponentiation in double (square-and-multiply, every product one round-to-nearest step); the
oracle calls the C library's pow.  The two differ in the last bits of b^t, but the scalars the
update uses are rounded once to fp32: step_size = fl32(lr / (1 - b1^t)) and
sbc2 = fl32(sqrt(1 - b2^t)).  This checks, on the host, that both evaluations give the same
fp32 scalars for every t up to 2,000,000 at the usual betas -- the device's square-and-multiply
restated with numpy float64 products (each rounded to nearest, no fusion)."""
import numpy as np
import pytest

T_MAX = 2_000_000


def pow_binary(b: float, t: np.ndarray) -> np.ndarray:
    r = np.ones(t.shape, np.float64)
    base = np.full(t.shape, b, np.float64)
    e = t.copy()
    while (e > 0).any():
        odd = (e & 1).astype(bool)
        r = np.where(odd, r * base, r)
        base = base * base
        e >>= 1
    return r


@pytest.mark.parametrize("b", [0.9, 0.95, 0.98, 0.999])
def test_bias_corrections_match_pow_after_fp32_rounding(b):
    t = np.arange(1, T_MAX + 1, dtype=np.int64)
    sq = pow_binary(b, t)
    lib = np.power(np.float64(b), t.astype(np.float64))
    lr = 1e-3
    # first moment: the step size lr / (1 - b1^t)
    assert np.array_equal(np.float32(lr / (1.0 + -sq)), np.float32(lr / (1.0 + -lib)))
    # second moment: sqrt(1 - b2^t)
    assert np.array_equal(np.float32(np.sqrt(1.0 + -sq)), np.float32(np.sqrt(1.0 + -lib)))


def test_pow_binary_is_exact_where_pow_is():
    t = np.array([1, 2, 3, 10, 1000], np.int64)
    assert np.array_equal(pow_binary(0.5, t), np.power(0.5, t.astype(np.float64)))  # powers of 2
    assert np.array_equal(pow_binary(1.0, t), np.ones(5))
