"""The oracle's float64 tanh-form GELU, pinned to an independent implementation of the
same function (PyTorch's CPU gelu with approximate="tanh", in float64) and to identities
that any tanh-form GELU satisfies.  It is the tolerance reference of the GPU's fused
epilogue (h within 2^-16 (|c| + |h|))."""
import numpy as np
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
