"""Exact-rational pins of the oracle's decoders: nvfp4 dequantize and the K side of
the KV window, with tensor scales that are not powers of two.  CPU only.

Format source: techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存",
§一 (E2M1 values, one E4M3 scale per 16 values, one FP32 scale per tensor) and §四 (K is
stored after subtracting its mean, which the window adds back).

The decoded value is RN_f32(RN_f32(e2m1 * s) * g); e2m1 * s is exact (at most six
significant bits), so the value equals the single rounding of the exact product
e2m1 * s * g.  The expectations below are computed in exact rationals and rounded
to binary32 and then to bf16 by integer arithmetic written here, so a slip in the
oracle's order of operations (e.g. e2m1 * RN(s * g)) or in its bf16 rounding fails.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle

E2M1 = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]


def e2m1_exact(code: int) -> Fraction:
    m = E2M1[code & 7]
    return -m if code & 8 else m


def e4m3_exact(b: int) -> Fraction:
    """E4M3FN value from the bit fields (bias 7, exponent 0 = subnormal)."""
    e, m = (b >> 3) & 0xF, b & 7
    v = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -v if b & 0x80 else v


def round_binary(q: Fraction, p: int, emin: int) -> Fraction:
    """Nearest number with a p-bit significand and exponent >= emin (subnormals
    below 2^emin), ties to the even significand.  No overflow handling (the cases
    here stay in range)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, emin)                        # exponent of the leading bit (or emin)
    ulp = Fraction(2) ** (e - p + 1)
    n, r = divmod(a, ulp)                   # a = n * ulp + r, 0 <= r < ulp
    n = int(n)
    if r * 2 > ulp or (r * 2 == ulp and n % 2 == 1):
        n += 1
    return sign * n * ulp


def rn_f32(q: Fraction) -> Fraction:
    return round_binary(q, 24, -126)


def rn_bf16(q: Fraction) -> Fraction:
    return round_binary(q, 8, -126)


def bf16_bits(v: Fraction, negative: bool) -> int:
    """bf16 bit pattern of the exact bf16 value v; `negative` gives the sign of a zero
    (IEEE: a product with a negative factor that rounds to zero is -0)."""
    f = np.float32(float(v))
    assert Fraction(float(f)) == v
    b = int(f.view(np.uint32)) >> 16
    return b | 0x8000 if (v == 0 and negative) else b


def all_codes_all_scales():
    """127 rows (one per finite non-negative E4M3 byte) of one 16-value block that
    holds each of the 16 E2M1 codes once."""
    row = np.array([c | ((c + 1) << 4) for c in range(0, 16, 2)], np.uint8)
    codes = np.tile(row, (127, 1))
    scales = np.arange(127, dtype=np.uint8).reshape(127, 1)
    return codes, scales


def tensor_scales():
    """Random float32 tensor scales across 2^-40 .. 2^10 (none a power of two), plus
    values whose products land in the subnormal range and near the rounding ties."""
    rng = np.random.default_rng(2024)
    gs = [np.float32(np.exp2(rng.uniform(-40, 10))) for _ in range(36)]
    gs += [np.float32(1.0 / 3.0), np.float32(0.1), np.float32(2.0 ** -20 * 1.7),
           np.float32(2.0 ** -120 * 1.3), np.float32(1.0000001), np.float32(0.0)]
    return [g for g in gs if float(g) == 0.0 or (int(np.float32(g).view(np.uint32)) & 0x7FFFFF) != 0]


@pytest.mark.parametrize("g", tensor_scales())
def test_dequantize_is_one_rounding_of_the_exact_product(g):
    codes, scales = all_codes_all_scales()
    q = oracle.Quantized(codes, scales, float(g), 0.0, 127, 16)
    y, yb = oracle.dequantize(q)
    G = Fraction(float(g))
    for r in range(127):
        s = e4m3_exact(r)
        for c in range(16):
            v = rn_f32(e2m1_exact(c) * s * G)
            neg = bool(c & 8)
            assert Fraction(float(y[r, c])) == v, (r, c, float(g))
            assert bool(np.signbit(y[r, c])) == (neg if v == 0 else v < 0), (r, c, float(g))
            assert int(yb[r, c]) == bf16_bits(rn_bf16(v), neg), (r, c, float(g))


def test_dequantize_differs_from_rounding_s_times_g_first():
    """The oracle multiplies e2m1 * s first (exact) and rounds once with g; rounding
    s * g first and then multiplying by e2m1 gives different float32 values for some
    of these inputs, so the pin above separates the two orders."""
    codes, scales = all_codes_all_scales()
    differ = 0
    for g in tensor_scales():
        G = Fraction(float(g))
        for r in range(127):
            s = e4m3_exact(r)
            sg = rn_f32(s * G)
            for c in (3, 5):  # magnitudes 1.5 and 3: products with more than one bit
                differ += rn_f32(e2m1_exact(c) * s * G) != rn_f32(e2m1_exact(c) * sg)
    assert differ > 0


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kv_window_k_adds_mu_with_a_separate_rounding(seed):
    """K^ = bf16(RN(RN(e2m1 * s * g_K) + mu)) element by element, for random codes,
    scales, a non-power-of-two g_K and random non-zero mu (float32)."""
    rng = np.random.default_rng(100 + seed)
    T, H, Dh = 8, 2, 32
    kc = rng.integers(0, 256, size=(T, H, Dh // 2), dtype=np.uint8)
    ks = rng.integers(0, 127, size=(T, H, Dh // 16), dtype=np.uint8)
    vc = rng.integers(0, 256, size=(T, H, Dh // 2), dtype=np.uint8)
    vs = rng.integers(0, 127, size=(T, H, Dh // 16), dtype=np.uint8)
    mu = (rng.standard_normal(H * Dh) * 3.0).astype(np.float32)
    g_k = np.float32(np.exp2(rng.uniform(-12, -2)))
    g_v = np.float32(np.exp2(rng.uniform(-12, -2)))
    ch = oracle.KVChunk(mu=mu, g_k=float(g_k), g_v=float(g_v), k_codes=kc, k_scales=ks, v_codes=vc,
                        v_scales=vs, amax_k=0.0, amax_v=0.0, T=T, H=H, Dh=Dh)
    kh, vh = oracle.kv_dequant_chunk(ch)
    GK, GV = Fraction(float(g_k)), Fraction(float(g_v))
    for t in range(T):
        for h in range(H):
            for d in range(Dh):
                byte_k = int(kc[t, h, d // 2])
                code_k = byte_k & 0xF if d % 2 == 0 else byte_k >> 4
                p = rn_f32(e2m1_exact(code_k) * e4m3_exact(int(ks[t, h, d // 16])) * GK)
                m = float(mu[h * Dh + d])
                want_k = rn_bf16(rn_f32(p + Fraction(m)))
                # an exact zero sum is +0 in round-to-nearest unless both addends are -0
                neg_zero = p == 0 and bool(code_k & 8) and m == 0 and np.signbit(np.float32(m))
                assert int(kh[t, h, d]) == bf16_bits(want_k, neg_zero), (t, h, d)
                byte_v = int(vc[t, h, d // 2])
                code_v = byte_v & 0xF if d % 2 == 0 else byte_v >> 4
                want_v = rn_bf16(rn_f32(e2m1_exact(code_v) * e4m3_exact(int(vs[t, h, d // 16])) * GV))
                assert int(vh[t, h, d]) == bf16_bits(want_v, bool(code_v & 8)), (t, h, d)


def test_round_binary_pins():
    """The rounding helper against values fixed by the binary32/bf16 definitions."""
    third = Fraction(1, 3)
    assert rn_f32(third) == Fraction(float(np.float32(1.0 / 3.0)))
    assert rn_f32(Fraction(1) + Fraction(2) ** -24) == 1          # tie -> even
    assert rn_f32(Fraction(1) + 3 * Fraction(2) ** -24) == 1 + Fraction(2) ** -22  # tie -> even (up)
    assert rn_f32(Fraction(2) ** -150) == 0                        # half the smallest subnormal: tie -> 0
    assert rn_f32(3 * Fraction(2) ** -150) == Fraction(2) ** -148  # 1.5 subnormal ulps -> 2 (even)
    assert rn_bf16(Fraction(1) + Fraction(2) ** -8) == 1           # bf16 tie -> even
    assert rn_bf16(Fraction(1) + 3 * Fraction(2) ** -8) == 1 + Fraction(2) ** -6
