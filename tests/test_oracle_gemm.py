"""Pins of the oracle's GEMM reference: float64 product of the exactly decoded NVFP4
operands, plus the per-element bound sum_k |a_k w_k|.  CPU only.

Source: techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存",
§四 — every matmul of the model runs with 4-bit weights and activations (W4A4)."""
from fractions import Fraction

import numpy as np

import oracle
import synth


def _q(x):
    return oracle.quantize(x)


def _frac_value(code, scale, g):
    mags = [Fraction(m).limit_denominator(4) for m in (0, .5, 1, 1.5, 2, 3, 4, 6)]
    v = mags[code & 7] * Fraction(oracle.e4m3_value(scale)) * Fraction(g)
    return -v if code & 8 else v


def test_tiny_gemm_vs_exact_rationals():
    rng = np.random.default_rng(2)
    M, N, K = 4, 3, 32
    a = (rng.standard_normal((M, K)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    w = (rng.standard_normal((N, K)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    qa, qw = _q(a), _q(w)
    c, bound = oracle.gemm_ref(qa.codes, qa.scales, qa.g, qw.codes, qw.scales, qw.g)
    for m in range(M):
        for n in range(N):
            acc, acc_abs = Fraction(0), Fraction(0)
            for k in range(K):
                ca = (int(qa.codes[m, k // 2]) >> (4 * (k % 2))) & 0xF
                cw = (int(qw.codes[n, k // 2]) >> (4 * (k % 2))) & 0xF
                p = _frac_value(ca, int(qa.scales[m, k // 16]), qa.g) * \
                    _frac_value(cw, int(qw.scales[n, k // 16]), qw.g)
                acc += p
                acc_abs += abs(p)
            assert abs(Fraction(c[m, n]) - acc) <= acc_abs * Fraction(1, 2 ** 50)
            assert abs(Fraction(bound[m, n]) - acc_abs) <= acc_abs * Fraction(1, 2 ** 50)


def test_single_nonzero_product_is_exact():
    a = np.zeros((2, 16), np.uint16)
    w = np.zeros((3, 16), np.uint16)
    a[1, 5] = 0x4128  # 10.5: g = 2^-8 exactly, decodes to 6 * 448 * 2^-8 = 10.5
    w[2, 5] = 0xC128  # -10.5
    qa, qw = _q(a), _q(w)
    c, bound = oracle.gemm_ref(qa.codes, qa.scales, qa.g, qw.codes, qw.scales, qw.g)
    assert c[1, 2] == -110.25 and bound[1, 2] == 110.25
    assert np.count_nonzero(c) == 1
    # a value whose g is not a power of two decodes to 6 * 448 * RN(amax / 2688)
    a[1, 5] = 0x4040  # 3.0
    qa = _q(a)
    c, _ = oracle.gemm_ref(qa.codes, qa.scales, qa.g, qw.codes, qw.scales, qw.g)
    assert c[1, 2] == 6 * 448 * float(np.float32(3.0) / np.float32(2688.0)) * -10.5


def test_selector_weights_pick_decoded_columns():
    x = synth.activations(5, 16, 64)
    qa = _q(x)
    w = np.zeros((4, 64), np.uint16)
    for n, k in enumerate((0, 17, 33, 63)):
        w[n, k] = 0x3F28  # 0.65625 = 10.5 * 2^-4 -> g = 2^-12, decodes to exactly 0.65625
    qw = _q(w)
    c, _ = oracle.gemm_ref(qa.codes, qa.scales, qa.g, qw.codes, qw.scales, qw.g)
    dec = oracle.decode_f64(qa.codes, qa.scales, qa.g)
    wdec = oracle.decode_f64(qw.codes, qw.scales, qw.g)
    assert set(np.unique(wdec)) <= {0.0, 0.65625}
    for n, k in enumerate((0, 17, 33, 63)):
        assert np.array_equal(c[:, n], dec[:, k] * 0.65625)


def test_bound_dominates_and_row_subset():
    a, w = synth.tiny_linear(0)
    qa, qw = _q(a), _q(w)
    c, bound = oracle.gemm_ref(qa.codes, qa.scales, qa.g, qw.codes, qw.scales, qw.g)
    assert np.all(np.abs(c) <= bound)
    rows = np.array([0, 7, 127])
    c2, b2 = oracle.gemm_ref(qa.codes, qa.scales, qa.g, qw.codes, qw.scales, qw.g, rows=rows)
    # same values up to the float64 summation order of the library matmul
    assert np.all(np.abs(c2 - c[rows]) <= 1e-12 * bound[rows])
    assert np.all(np.abs(b2 - bound[rows]) <= 1e-12 * bound[rows])
