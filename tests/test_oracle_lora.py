"""Pins of the oracle's LoRA merge W' = W + scale (B A) (LoRA before quantization)
against what the arithmetic fixes, not against a retyped copy of the loop."""
import numpy as np

import oracle
import synth


def test_zero_factors_leave_the_weight_unchanged():
    rng = np.random.default_rng(1)
    w = rng.standard_normal((7, 48)).astype(np.float32)
    b = rng.standard_normal((7, 5)).astype(np.float32)
    zero_a = np.zeros((5, 48), np.float32)
    assert np.array_equal(oracle.lora_merge(w, b, zero_a, 3.0), w)
    assert np.array_equal(oracle.lora_merge(w, np.zeros_like(b), rng.standard_normal((5, 48)).astype(np.float32),
                                            0.7), w)


def test_exact_small_integers():
    """Small integer factors and a power-of-two scale: every product, partial sum and
    the final add are exact in binary32, so W' equals the exact result."""
    rng = np.random.default_rng(2)
    rows, cols, rank = 33, 80, 24
    w = rng.integers(-100, 100, (rows, cols)).astype(np.float32)
    b = rng.integers(-8, 9, (rows, rank)).astype(np.float32)
    a = rng.integers(-8, 9, (rank, cols)).astype(np.float32)
    exact = w.astype(np.int64) * 4 + (b.astype(np.int64) @ a.astype(np.int64))  # 4 W + B A
    got = oracle.lora_merge(w, b, a, 0.25)
    assert np.array_equal((got.astype(np.float64) * 4).astype(np.int64), exact)


def test_rank_one_is_one_product_and_one_sum():
    """rank 1, scale 1: W' = RN(W + RN(b a)), one binary32 multiply and one add."""
    rng = np.random.default_rng(3)
    w = rng.standard_normal((16, 64)).astype(np.float32)
    b = rng.standard_normal((16, 1)).astype(np.float32)
    a = rng.standard_normal((1, 64)).astype(np.float32)
    ref = w + (b * a).astype(np.float32)  # numpy float32 ops round each result
    assert np.array_equal(oracle.lora_merge(w, b, a, 1.0), ref)


def test_within_the_float_error_bound_of_the_exact_update():
    """|W' - (W + scale B A)| <= (rank + 2) u (|W| + |scale| sum_j |b_j a_j|), u = 2^-24,
    against the float64 product (sequential binary32 summation error)."""
    rng = np.random.default_rng(4)
    rows, cols, rank = 40, 96, 64
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    b = (rng.standard_normal((rows, rank)) * 0.1).astype(np.float32)
    a = (rng.standard_normal((rank, cols)) * 0.1).astype(np.float32)
    scale = np.float32(0.5)
    got = oracle.lora_merge(w, b, a, scale).astype(np.float64)
    exact = w.astype(np.float64) + float(scale) * (b.astype(np.float64) @ a.astype(np.float64))
    mag = np.abs(w.astype(np.float64)) + abs(float(scale)) * (np.abs(b.astype(np.float64)) @ np.abs(a.astype(np.float64)))
    assert np.all(np.abs(got - exact) <= (rank + 2) * 2.0 ** -24 * mag * 1.0001)
    assert np.any(got != exact)  # not trivially exact: the bound is exercised


def test_bf16_weight_equals_its_float_widening():
    w = synth.weights(5, 0, 24, 64)
    b = np.random.default_rng(5).standard_normal((24, 8)).astype(np.float32)
    a = np.random.default_rng(6).standard_normal((8, 64)).astype(np.float32)
    wf = synth.bf16_bits_to_f32(w).astype(np.float32)
    assert np.array_equal(oracle.lora_merge(w, b, a, 0.125), oracle.lora_merge(wf, b, a, 0.125))
