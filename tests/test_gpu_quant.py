"""GPU parity of nvfp4_quantize / nvfp4_dequantize against the oracle: codes,
E4M3 scales and the tensor scale bit for bit; dequantized values bit for bit."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle
import synth
from gpu_helpers import (assert_quant_equal, canonical, dev_bf16, device_status, gpu_quantize,
                         host_bits, mma_padding_is_zero)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_MMA])
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (130, 528), (257, 3072), (128, 512)])
def test_quantize_matches_oracle(cuda_dev, layout, shape):
    x = synth.activations(11, *shape)
    q, amax = gpu_quantize(x, layout)
    ref = oracle.quantize(x)
    assert amax == ref.amax
    assert_quant_equal(q, ref)
    if layout == nv.SF_MMA:
        assert mma_padding_is_zero(q)
    assert device_status() == nv.OK


def test_worked_example_on_gpu(cuda_dev):
    from test_oracle_quant import BLOCK1, BLOCK2, CODES1, CODES2, bf16, nibbles

    x = bf16([BLOCK1 + BLOCK2 + [0] * 16])
    q, amax = gpu_quantize(x, nv.SF_ROWMAJOR)
    codes, scales, g = canonical(q)
    assert g == 2.0 ** -8 and amax == 10.5
    assert list(scales[0]) == [0x7E, 0x63, 0]
    assert nibbles(codes[0]) == CODES1 + CODES2 + [0] * 16


def test_midpoints_ties_and_edges(cuda_dev):
    """Values placed exactly on and one bf16 step around every E2M1 midpoint of
    many block scales, plus zeros, -0, subnormals and saturating blocks."""
    rng = np.random.default_rng(0)
    rows = []
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    for _ in range(400):
        D = np.float32(2.0 ** rng.integers(-20, 20)) * np.float32(rng.choice([1.0, 1.25, 1.5, 1.75]))
        vals = np.concatenate([mids * D, [6 * D], rng.choice(mids, 8) * D]).astype(np.float32)
        b = (vals.view(np.uint32) >> 16).astype(np.uint16)
        b = b + rng.integers(-1, 2, b.size).astype(np.uint16) * (rng.random(b.size) < 0.3)
        b ^= (rng.random(b.size) < 0.5).astype(np.uint16) << 15
        rows.append(b[:16])
    x = np.stack(rows).reshape(25, 256)
    x[0, :16] = 0
    x[1, :16] = 0x8000  # -0
    x[2, :16] = np.arange(16, dtype=np.uint16) + 1  # bf16 subnormals
    for layout in (nv.SF_ROWMAJOR, nv.SF_MMA):
        q, _ = gpu_quantize(x, layout)
        assert_quant_equal(q, oracle.quantize(x))


def test_block_scale_rounding_boundaries(cuda_dev):
    """Blocks whose max|x| / RN(6 g) lies exactly on, or one bf16 step either side
    of, an E4M3 rounding boundary (every normal-range midpoint, the subnormal
    midpoints and the saturation edge), with g = 2^-10 supplied so RN(6 g) is exact."""
    rng = np.random.default_rng(7)
    g = 2.0 ** -10
    d6 = 6.0 * g
    targets = [(1.0 + (2 * m + 1) / 16.0) * 2.0 ** e for e in range(-6, 9) for m in range(8)]
    targets += [(j + 0.5) * 2.0 ** -9 for j in range(8)] + [448.0, 464.0, 480.0]
    rows = []
    for t in targets:
        amax_bits = int(np.float32(t * d6).view(np.uint32) >> 16)
        for delta in (-1, 0, 1):
            top = np.array([(amax_bits + delta) << 16], np.uint32).view(np.float32)[0]
            vals = (rng.uniform(-0.9, 0.9, 16) * top).astype(np.float32)
            vals[rng.integers(16)] = top * rng.choice([-1.0, 1.0])
            rows.append((vals.view(np.uint32) >> 16).astype(np.uint16))
    x = np.stack(rows)
    x = np.concatenate([x, np.zeros(((-len(x)) % 8, 16), np.uint16)]).reshape(-1, 128)
    for layout in (nv.SF_ROWMAJOR, nv.SF_MMA):
        q, _ = gpu_quantize(x, layout, gscale=g)
        assert_quant_equal(q, oracle.quantize(x, gscale=g))


@pytest.mark.parametrize("scale", [1e-30, 1e-36, 2.0 ** -133 * 7, 1e30, 3e38])
def test_extreme_magnitudes(cuda_dev, scale):
    x = synth.activations(3, 16, 64)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64) * scale / 30.0
    xf = np.clip(xf, -3.3e38, 3.3e38).astype(np.float32)
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)
    q, _ = gpu_quantize(xb, nv.SF_MMA)
    assert_quant_equal(q, oracle.quantize(xb))


def test_fp32_input(cuda_dev):
    rng = np.random.default_rng(4)
    x = (rng.standard_t(3, (70, 96)) * 0.7).astype(np.float32)
    q, amax = gpu_quantize(x, nv.SF_MMA, fp32=True)
    ref = oracle.quantize(x)
    assert amax == ref.amax
    assert_quant_equal(q, ref)


def test_supplied_gscale_one_pass(cuda_dev):
    x = synth.activations(5, 200, 256)
    g = oracle.quantize(x).g
    for gs in (g, g * 0.37, g * 3.0):
        gs = float(np.float32(gs))
        q, amax = gpu_quantize(x, nv.SF_MMA, gscale=gs)
        ref = oracle.quantize(x, gscale=gs)
        assert amax == ref.amax
        assert_quant_equal(q, ref)


def test_supplied_gscale_huge_block_scales(cuda_dev):
    """A supplied tensor scale large enough that D = s g exceeds 2^125 (so 1/D is
    near the flushed range) with values near the top of the binary32 range."""
    x = synth.activations(6, 64, 128)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64) * (3.0e38 / 30.0)
    xf = np.clip(xf, -3.3e38, 3.3e38).astype(np.float32)
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)
    for gs in (1.0e37, 3.0e36, 2.0 ** 120):
        gs = float(np.float32(gs))
        q, _ = gpu_quantize(xb, nv.SF_MMA, gscale=gs)
        assert_quant_equal(q, oracle.quantize(xb, gscale=gs))


def test_all_zero_and_empty(cuda_dev):
    x = np.zeros((5, 32), np.uint16)
    q, amax = gpu_quantize(x, nv.SF_MMA)
    assert amax == 0.0
    assert_quant_equal(q, oracle.quantize(x))
    e, amax = gpu_quantize(np.zeros((0, 32), np.uint16), nv.SF_MMA)
    assert float(e.gscale.item()) == 0.0 and amax == 0.0


def test_nonfinite_sets_status_and_writes_nothing(cuda_dev):
    x = synth.activations(1, 8, 64)
    x[3, 17] = 0x7FC0  # NaN
    device_status(clear=True)
    xd = dev_bf16(x)
    out = nv.NVFP4Tensor(8, 64, nv.SF_MMA)
    out.codes.fill_(0xAB)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    nv.nvfp4_quantize(xd, out, amax_out=amax)
    assert device_status(clear=True) == nv.ERR_NONFINITE
    assert int((out.codes != 0xAB).sum().item()) == 0
    assert device_status() == nv.OK


@pytest.mark.parametrize("layout", [nv.SF_ROWMAJOR, nv.SF_MMA])
def test_dequantize_matches_oracle(cuda_dev, layout):
    x = synth.activations(7, 300, 1024)
    q, _ = gpu_quantize(x, layout)
    ref = oracle.quantize(x)
    yf, yb = oracle.dequantize(ref)
    out32 = torch.empty((300, 1024), dtype=torch.float32, device="cuda")
    nv.nvfp4_dequantize(q, out32)
    assert np.array_equal(out32.cpu().numpy().view(np.uint32), yf.view(np.uint32))
    out16 = torch.empty((300, 1024), dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_dequantize(q, out16)
    assert np.array_equal(host_bits(out16), yb)


@pytest.mark.slow
def test_full_size_activation_pass(cuda_dev):
    """32768 x 3072 bf16 (0.5 * t3, 31 channels x30): quantize and dequantize, every
    output compared."""
    x = synth.activations(1, 32768, 3072)
    q, amax = gpu_quantize(x, nv.SF_MMA)
    ref = oracle.quantize(x)
    assert amax == ref.amax
    assert_quant_equal(q, ref)
    assert mma_padding_is_zero(q)
    _, yb = oracle.dequantize(ref)
    out16 = torch.empty((32768, 3072), dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_dequantize(q, out16)
    assert np.array_equal(host_bits(out16), yb)
