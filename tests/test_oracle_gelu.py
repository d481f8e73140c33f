"""The oracle's float64 tanh-form GELU, pinned to an independent implementation of the
same function (PyTorch's CPU gelu with approximate="tanh", in float64), to the same
formula evaluated with 60 significant digits (mpmath), and to identities that any
tanh-form GELU satisfies.  It is the tolerance reference of the GPU's fused epilogue,
whose gate bounds the error of h relative to |h| also in the negative tail, so the
reference must be accurate there relative to |h|, not only to |c|."""
import mpmath
import numpy as np
import pytest
import torch

import oracle


def torch_gelu_tanh(x: np.ndarray) -> np.ndarray:
    return torch.nn.functional.gelu(torch.from_numpy(x.astype(np.float64)), approximate="tanh").numpy()


def test_matches_torch_tanh_gelu_in_float64():
    rng = np.random.default_rng(11)
    grid = np.linspace(-12.0, 12.0, 20001).astype(np.float32)
    mags = (10.0 ** rng.uniform(-30, 30, 20000)).astype(np.float32)
    signs = np.where(rng.random(20000) < 0.5, -1.0, 1.0).astype(np.float32)
    x = np.concatenate([grid, mags * signs, np.float32([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38])])
    got = oracle.gelu_tanh(x)
    ref = torch_gelu_tanh(x)
    xd = x.astype(np.float64)
    assert np.all(np.abs(got - ref) <= 4.0 * np.finfo(np.float64).eps * (np.abs(xd) + np.abs(ref)) + 1e-300)


def test_odd_part_is_the_identity():
    """0.5 x (1 + tanh u(x)) - 0.5 (-x) (1 + tanh u(-x)) = x since u is odd."""
    x = np.linspace(-20.0, 20.0, 4001).astype(np.float32)
    d = oracle.gelu_tanh(x) - oracle.gelu_tanh(-x)
    assert np.all(np.abs(d - x.astype(np.float64)) <= 8.0 * np.finfo(np.float64).eps * np.abs(x) + 1e-300)


def test_limits():
    big = np.float32([10.0, 30.0, 1.0e6, 3.0e38])
    assert np.array_equal(oracle.gelu_tanh(big), big.astype(np.float64))
    small = oracle.gelu_tanh(-big)
    assert np.all(np.abs(small) < 1e-20) and np.all(small <= 0.0)
    assert oracle.gelu_tanh(np.float32([0.0]))[0] == 0.0


def gelu_mp(x: float) -> float:
    """0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) in the tanh form itself, with 60
    significant digits more than the cancellation of 1 + tanh(u) eats (about 2|u| /
    ln 10 digits for u < 0), rounded to the nearest double."""
    u0 = abs(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3))
    with mpmath.workdps(60 + int(2.0 * u0 / np.log(10.0)) if x < 0 else 60):
        X = mpmath.mpf(float(x))
        u = mpmath.sqrt(2 / mpmath.pi) * (X + mpmath.mpf("0.044715") * X ** 3)
        return float(X * (1 + mpmath.tanh(u)) / 2)


@pytest.mark.parametrize("lo,hi", [(-30.0, -3.0), (-3.0, 3.0), (3.0, 12.0)])
def test_relative_accuracy_against_60_digit_evaluation(lo, hi):
    """Within 8 ulp of |h| everywhere, including the negative tail where h is a tiny
    fraction of x (the 0.044715 constant is the decimal of the formula; the float64
    oracle rounds it once, which moves h by at most ~|x^3| 2^-53 relative in u)."""
    x = np.linspace(lo, hi, 601).astype(np.float32)
    got = oracle.gelu_tanh(x)
    ref = np.array([gelu_mp(v) for v in x])
    xd = x.astype(np.float64)
    # rounding of the constant 0.044715 to double and of u: |du| <= ~4 eps |u|, and
    # dh / h = -du * 2 / (1 + exp(2u)) for the quotient form
    u = np.sqrt(2.0 / np.pi) * (xd + 0.044715 * xd ** 3)
    cond = 1.0 + np.abs(u) * 2.0 / (1.0 + np.exp(np.minimum(2.0 * u, 700.0)))
    tol = 8.0 * np.finfo(np.float64).eps * np.abs(ref) * cond + 1e-300
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) / tol))
    # no flush in the tail while h is far above the double range's bottom (h ~ -1e-261
    # at x = -20; exp(-2u) overflows only where |h| < ~1e-306)
    assert np.all((np.abs(ref) < 1e-290) | (got != 0))
