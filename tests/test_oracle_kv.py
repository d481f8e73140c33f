"""Pins of the oracle's NVFP4 KV-cache steps: exact per-(head, dim) mean of K,
mean-subtracted K encode, V encode, window dequant, storage size.  CPU only.

Source: techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存",
§四 — K gets a simple mean subtraction and then NVFP4; about 1.125 bytes per value
against 4 in bf16 (read per K+V pair); several chunks are dequantized in one window."""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rn_f32(q: Fraction) -> float:
    """Round a rational to the nearest float32, ties to even, by comparing the
    float32 candidates around float(q) exactly."""
    if q == 0:
        return 0.0
    c = np.float32(float(q))
    cands = {float(c), float(np.nextafter(c, np.float32(np.inf))),
             float(np.nextafter(c, np.float32(-np.inf)))}
    return min(cands, key=lambda f: (abs(Fraction(f) - q),
                                     int(np.float32(f).view(np.uint32)) & 1))


def bits(vals):
    f = np.asarray(vals, dtype=np.float32)
    assert np.all((f.view(np.uint32) & 0xFFFF) == 0)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def exact_mean(col_bits):
    vals = synth.bf16_bits_to_f32(col_bits)
    return rn_f32(sum((Fraction(float(v)) for v in vals), Fraction(0)) / len(vals))


@pytest.mark.parametrize("T", [1, 3, 7, 8, 1000, 8192])
def test_exact_mean_random_columns(T):
    rng = np.random.default_rng(T)
    for trial in range(5):
        col = (rng.standard_normal(T).astype(np.float32) * np.float32(3.0) + np.float32(
            rng.standard_normal()) * 10).view(np.uint32) >> 16
        col = col.astype(np.uint16)
        assert oracle.exact_mean_bf16(col) == exact_mean(col)


def test_exact_mean_adversarial_columns():
    cases = [
        [1.0, 2.0 ** -24] + [0.0] * 6,               # S/8 exactly at a float32 midpoint -> even
        [1.0, 2.0 ** -24, 2.0 ** -60] + [0.0] * 5,   # just above the midpoint -> rounds up
        [1.0, 2.0 ** -24, -(2.0 ** -60)] + [0.0] * 5,
        [2.0 ** 100, 2.0 ** -100, -(2.0 ** 100)],   # cancellation leaves the tiny term
        [3e38, 3e38, -3e38, 1e-38],
        [9.183549615799121e-41, 1.0e-40, 2.0 ** -126],  # bf16 subnormals
        [-1.5, -2.25, -7.0],
        [0.0, -0.0],
    ]
    for vals in cases:
        f = np.asarray(vals, dtype=np.float32)
        col = (f.view(np.uint32) >> 16).astype(np.uint16)
        assert oracle.exact_mean_bf16(col) == exact_mean(col), vals
    # the midpoint case, written out: (1 + 2^-24) / 8 lies halfway between 1/8 and
    # 1/8 + 2^-26, and goes to the even neighbour 1/8
    assert oracle.exact_mean_bf16(bits([1.0, 2.0 ** -24] + [0.0] * 6)) == 0.125
    assert oracle.exact_mean_bf16(bits([1.0, 2.0 ** -24, 2.0 ** -60] + [0.0] * 5)) == 0.125 + 2.0 ** -26


def test_constant_key_columns_give_zero_residual():
    T, H, Dh = 16, 2, 32
    off = np.float32(np.arange(H * Dh) * 0.25 - 3.0)
    k = np.tile(bits(off), (T, 1)).reshape(T, H, Dh)
    v = ((np.linspace(-2, 2, T * H * Dh).astype(np.float32).view(np.uint32) >> 16)
         .astype(np.uint16).reshape(T, H, Dh))
    ch = oracle.kv_append(k, v)
    assert np.array_equal(ch.mu, off)
    assert ch.g_k == 0.0 and ch.amax_k == 0.0
    assert np.all(ch.k_codes == 0) and np.all(ch.k_scales == 0)
    kh, vh = oracle.kv_dequant_chunk(ch)
    assert np.array_equal(kh, k)  # mu is restored exactly


def test_kv_append_matches_plain_quantize_of_parts():
    T, H, Dh = 64, 3, 32
    off = synth.kv_offsets(3, H, Dh)
    k, v = synth.kv_chunk(3, 0, T, H, Dh, off)
    ch = oracle.kv_append(k, v)
    kf = synth.bf16_bits_to_f32(k.reshape(T, H * Dh))
    for c in range(H * Dh):
        assert ch.mu[c] == exact_mean(k.reshape(T, H * Dh)[:, c])
    kp = (kf - ch.mu[None, :]).astype(np.float32)  # RN(k - mu) in float32
    qk = oracle.quantize(kp.reshape(T * H, Dh))
    qv = oracle.quantize(v.reshape(T * H, Dh))
    assert ch.g_k == qk.g and ch.g_v == qv.g
    assert np.array_equal(ch.k_codes.reshape(T * H, -1), qk.codes)
    assert np.array_equal(ch.k_scales.reshape(T * H, -1), qk.scales)
    assert np.array_equal(ch.v_codes.reshape(T * H, -1), qv.codes)
    assert np.array_equal(ch.v_scales.reshape(T * H, -1), qv.scales)
    assert ch.amax_k == float(np.abs(kp).max())


def test_window_dequant_values():
    T, H, Dh = 32, 2, 16
    off = synth.kv_offsets(5, H, Dh)
    k, v = synth.kv_chunk(5, 1, T, H, Dh, off)
    ch = oracle.kv_append(k, v)
    kh, vh = oracle.kv_dequant_chunk(ch)
    # V^ is the plain NVFP4 dequantization of V
    qv = oracle.quantize(v.reshape(T * H, Dh))
    _, vb = oracle.dequantize(qv)
    assert np.array_equal(vh.reshape(T * H, Dh), vb)
    # K^ = bf16(RN(dequant(K') + mu)): dequant in float32, one float32 add, bf16 RNE
    qk = oracle.Quantized(ch.k_codes.reshape(T * H, -1), ch.k_scales.reshape(T * H, -1), ch.g_k,
                          ch.amax_k, T * H, Dh)
    kd, _ = oracle.dequantize(qk)
    s = (kd.reshape(T, H * Dh) + ch.mu[None, :]).astype(np.float32)
    want = np.array([oracle.f32_to_bf16(float(x)) for x in s.ravel()], np.uint16)
    assert np.array_equal(kh.ravel(), want)
    # reconstruction error of K: at most half the largest E2M1 gap (2) times the
    # largest block step D = 448 g_K, plus the bf16 rounding of the result
    kf = synth.bf16_bits_to_f32(k)
    err = np.abs(synth.bf16_bits_to_f32(kh) - kf)
    assert float(err.max()) <= 448 * ch.g_k + 2.0 ** -7 * float(np.abs(kf).max())


def test_kv_storage_bytes_per_pair_matches_page():
    vals = {}
    with open(os.path.join(GOLDEN, "kv_bytes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k_, v_ = line.split()
                vals[k_] = float(v_)
    T, H, Dh = 64, 3, 32
    off = synth.kv_offsets(0, H, Dh)
    k, v = synth.kv_chunk(0, 0, T, H, Dh, off)
    ch = oracle.kv_append(k, v)
    pairs = T * H * Dh
    nbytes = ch.k_codes.nbytes + ch.k_scales.nbytes + ch.v_codes.nbytes + ch.v_scales.nbytes
    assert nbytes / pairs == vals["nvfp4_bytes_per_pair"]
    assert (k.nbytes + v.nbytes) / pairs == vals["bf16_bytes_per_pair"]
    assert round(vals["bf16_bytes_per_pair"] / vals["nvfp4_bytes_per_pair"], 1) == vals["ratio_approx"]


def test_nonfinite_kv_is_an_error():
    k = np.zeros((2, 1, 16), np.uint16)
    v = np.zeros((2, 1, 16), np.uint16)
    v[1, 0, 3] = 0x7FC0
    with pytest.raises(FloatingPointError):
        oracle.kv_append(k, v)
