"""Pins of the oracle's NVFP4 quantize / dequantize (tensor scale, block scales,
element codes, packing, the tensor-core scale layout).  CPU only.

Format source: techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存",
§一 — E2M1 values, one FP8 (E4M3) scale per 16 values, one FP32 scale per tensor."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth


def bf16(vals):
    f = np.asarray(vals, dtype=np.float32)
    bits = f.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "test values must be exact bf16"
    return (bits >> 16).astype(np.uint16)


def nibbles(codes_row):
    out = []
    for b in codes_row:
        out += [int(b) & 0xF, int(b) >> 4]
    return out


# One row of 48 values = 3 blocks.  Hand derivation:
#   amax = 10.5 -> g = 10.5 / 2688 = 2^-8 exactly; RN(6 g) = 0.0234375.
#   block 1: amax_b = 10.5 -> s_raw = 448 -> s = 0x7E (448), D = 448 * 2^-8 = 1.75.
#     quotients x/D: 0, .25, -.75, 1.25, 1.75, 2.5, 3.5, 5, 6, -6, 1, .5, -.25, 3, 4, 2
#     ties go to the even E2M1 index: .25->0, .75->2(1.0), 1.25->2, 1.75->4(2.0),
#     2.5->4, 3.5->6(4.0), 5->6, -.25 -> -0 (0x8).
#   block 2: amax_b = 1 -> s_raw = RN(1 / 0.0234375) = 42.666668 -> nearest E4M3 is
#     44 (grid step 4 in [32, 64)) = 0x63; D = 44 * 2^-8 = 0.171875.
#     1/D = 5.82 -> 6 (7); .5/D = 2.91 -> 3 (5); -.30078125/D = -1.75 exactly -> tie -> -2
#     (0xC); .25/D = 1.45 -> 1.5 (3); -1 -> 0xF; .75/D = 4.36 -> 4 (6); .125/D = .727 -> .5 (1);
#     -.0625/D = -.364 -> -.5 (9).
#   block 3: all zero -> s = 0x00, codes 0.
BLOCK1 = [0, 0.4375, -1.3125, 2.1875, 3.0625, 4.375, 6.125, 8.75, 10.5, -10.5, 1.75, 0.875,
          -0.4375, 5.25, 7, 3.5]
BLOCK2 = [1, 0.5, -0.30078125, 0.25, 0, -1, 0.75, 0.125] + [0] * 7 + [-0.0625]
CODES1 = [0x0, 0x0, 0xA, 0x2, 0x4, 0x4, 0x6, 0x6, 0x7, 0xF, 0x2, 0x1, 0x8, 0x5, 0x6, 0x4]
CODES2 = [0x7, 0x5, 0xC, 0x3, 0x0, 0xF, 0x6, 0x1] + [0] * 7 + [0x9]
DEQ2 = [1.03125, 0.515625, -0.34375, 0.2578125, 0, -1.03125, 0.6875, 0.0859375] + [0] * 7 + [-0.0859375]


def test_worked_example_48_values():
    x = bf16([BLOCK1 + BLOCK2 + [0] * 16])
    q = oracle.quantize(x)
    assert q.amax == 10.5
    assert q.g == 2.0 ** -8
    assert list(q.scales[0]) == [0x7E, 0x63, 0x00]
    assert nibbles(q.codes[0]) == CODES1 + CODES2 + [0] * 16
    y, yb = oracle.dequantize(q)
    assert list(y[0, 16:32]) == DEQ2
    assert list(y[0, 32:]) == [0.0] * 16


def test_global_scale_closed_form_powers_of_two():
    for k in range(-20, 21):
        x = bf16([[10.5 * 2.0 ** k] + [0.0] * 15])
        q = oracle.quantize(x)
        assert q.g == 2.0 ** (k - 8)
        assert q.scales[0, 0] == 0x7E  # the tensor max maps to s = 448
        assert q.codes[0, 0] & 0xF == 7  # and to E2M1 magnitude 6


def test_global_scale_is_one_division_by_2688():
    rng = np.random.default_rng(0)
    amaxes = rng.uniform(1e-3, 1e3, 200).astype(np.float32)
    for a in (amaxes.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32):
        q = oracle.quantize(bf16([[float(a)] + [0.0] * 15]))
        assert q.g == float(np.float32(a) / np.float32(2688.0))


def test_zero_tensor_and_signed_zero():
    x = bf16([[0.0] * 16 + [-0.0] * 16])
    q = oracle.quantize(x)
    assert q.g == 0.0 and q.amax == 0.0
    assert list(q.scales[0]) == [0, 0]
    assert nibbles(q.codes[0]) == [0] * 16 + [8] * 16
    y, _ = oracle.dequantize(q)
    assert np.all(y == 0)


@pytest.mark.parametrize("v", [1.0, -3.25, 2.0 ** -10 * 1.5, 7 * 2.0 ** 13])
def test_constant_tensor_maps_to_max_code(v):
    x = np.full((3, 32), bf16([v])[0], dtype=np.uint16)
    q = oracle.quantize(x)
    assert np.all(q.scales == 0x7E)
    want = 0xF if v < 0 else 0x7
    assert all(c == want for c in nibbles(q.codes.ravel()))


def test_scale_invariance_by_powers_of_two():
    x = synth.activations(9, 8, 256)
    xf = synth.bf16_bits_to_f32(x)
    q0 = oracle.quantize(x)
    for k in (-6, -1, 1, 5):
        xk = (xf * np.float32(2.0 ** k)).view(np.uint32) >> 16
        qk = oracle.quantize(xk.astype(np.uint16))
        assert qk.g == q0.g * 2.0 ** k
        assert np.array_equal(qk.scales, q0.scales)
        assert np.array_equal(qk.codes, q0.codes)


def test_code_is_within_half_a_gap_of_x():
    """Nearest rounding of |x|/D: | |x| - m D | <= (largest gap next to m) / 2 * D,
    except for saturated elements (|x| > 6 D, magnitude 6)."""
    half_gap = [0.25, 0.25, 0.25, 0.25, 0.5, 0.5, 1.0, 1.0]
    mags = [0, .5, 1, 1.5, 2, 3, 4, 6]
    x = synth.activations(3, 32, 512)
    q = oracle.quantize(x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    checked = 0
    for r in range(x.shape[0]):
        codes = nibbles(q.codes[r])
        for c in range(x.shape[1]):
            s = oracle.e4m3_value(int(q.scales[r, c // 16]))
            D = float(np.float32(np.float32(s) * np.float32(q.g)))
            ax, m = abs(xf[r, c]), codes[c] & 7
            if D == 0 or ax > 6 * D:
                continue
            assert abs(ax - mags[m] * D) <= half_gap[m] * D
            assert (codes[c] >> 3) == (1 if np.signbit(xf[r, c]) else 0)
            checked += 1
    assert checked > 0.9 * x.size


def _brute_block(xs, g):
    """Independent statement of steps 4-5 for one block with exact rationals:
    s = the E4M3 value nearest to RN(amax/RN(6g)) by scanning all codes, then each
    element's nearest E2M1 magnitude to |x|/D by scanning all magnitudes."""
    f32 = np.float32
    amax_b = max(abs(float(v)) for v in xs)
    d6 = f32(f32(6.0) * f32(g))
    if d6 == 0:
        s_code = 0
    else:
        s_raw = Fraction(float(f32(f32(amax_b) / d6)))
        finite = [(b, Fraction(oracle.e4m3_value(b))) for b in range(127)]
        if s_raw >= 448:
            s_code = 0x7E
        else:
            s_code = min(finite, key=lambda bv: (abs(s_raw - bv[1]), bv[0] % 2))[0]
    D = Fraction(float(f32(f32(oracle.e4m3_value(s_code)) * f32(g))))
    mags = [Fraction(m).limit_denominator(4) for m in (0, .5, 1, 1.5, 2, 3, 4, 6)]
    codes = []
    for v in xs:
        if D == 0:
            idx = 0
        else:
            q = abs(Fraction(float(v))) / D
            idx = min(range(8), key=lambda i: (abs(q - mags[i]), i % 2))
        codes.append((8 if np.signbit(v) else 0) | idx)
    return s_code, codes


def test_tiny_tensors_vs_bruteforce():
    rng = np.random.default_rng(1)
    for trial in range(30):
        rows, cols = int(rng.integers(1, 4)), 16 * int(rng.integers(1, 4))
        scale = float(np.exp2(rng.uniform(-30, 30)))
        xf = (rng.standard_t(3, (rows, cols)) * scale).astype(np.float32)
        xb = (xf.view(np.uint32) >> 16).astype(np.uint16)
        xv = synth.bf16_bits_to_f32(xb)
        q = oracle.quantize(xb)
        g = float(np.float32(np.float32(np.abs(xv).max()) / np.float32(2688.0)))
        assert q.g == g
        for r in range(rows):
            row_codes = nibbles(q.codes[r])
            for b in range(cols // 16):
                s_code, codes = _brute_block(xv[r, b * 16:(b + 1) * 16], g)
                assert q.scales[r, b] == s_code
                assert row_codes[b * 16:(b + 1) * 16] == codes


def test_supplied_global_scale_is_used():
    x = synth.activations(4, 4, 64)
    q0 = oracle.quantize(x)
    q1 = oracle.quantize(x, gscale=q0.g)
    assert np.array_equal(q0.codes, q1.codes) and np.array_equal(q0.scales, q1.scales)
    q2 = oracle.quantize(x, gscale=q0.g / 4)  # too small a scale saturates blocks at 448
    assert q2.g == q0.g / 4
    assert q2.scales.max() == 0x7E


def test_nonfinite_input_is_an_error():
    x = bf16([[1.0] * 16])
    x[0, 3] = 0x7F80  # +inf
    assert oracle.quantize_status(x) == oracle.ERR_NONFINITE
    x[0, 3] = 0x7FC0  # nan
    assert oracle.quantize_status(x) == oracle.ERR_NONFINITE


def test_packing_low_nibble_first():
    x = bf16([[6.0, 0.5] + [0.0] * 14])
    q = oracle.quantize(x)
    assert q.codes[0, 0] == (0x7 | (0x1 << 4))


def test_mma_scale_layout_offsets():
    # (row, block, cols) -> byte, written out from the layout definition
    cols = 3072  # 192 blocks -> 48 groups of 4
    assert oracle.sf_mma_offset(0, 0, cols) == 0
    assert oracle.sf_mma_offset(0, 3, cols) == 3
    assert oracle.sf_mma_offset(1, 0, cols) == 16
    assert oracle.sf_mma_offset(31, 0, cols) == 496
    assert oracle.sf_mma_offset(32, 0, cols) == 4
    assert oracle.sf_mma_offset(127, 2, cols) == 31 * 16 + 3 * 4 + 2
    assert oracle.sf_mma_offset(0, 4, cols) == 512
    assert oracle.sf_mma_offset(128, 0, cols) == 48 * 512
    assert oracle.sf_mma_bytes(130, 48) == 256 * 4  # 3 blocks pad to one group of 4
    s = np.arange(200 * 3, dtype=np.uint8).reshape(200, 3)
    buf = oracle.sf_to_mma(s, 48)
    assert np.array_equal(oracle.sf_from_mma(buf, 200, 48), s)
    used = np.zeros(buf.size, bool)
    used[[oracle.sf_mma_offset(r, j, 48) for r in range(200) for j in range(3)]] = True
    assert np.all(buf[~used] == 0)
