"""GPU parity of nvfp4_lora_merge (LoRA merged before quantization) against the
oracle, bit for bit, and of the merge -> quantize chain."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle
import synth
from gpu_helpers import assert_quant_equal, dev_bf16, device_status, gpu_quantize

pytestmark = pytest.mark.gpu


def factors(seed, rows, cols, rank, std=0.05):
    rng = np.random.default_rng(seed)
    b = (rng.standard_normal((rows, rank)) * std).astype(np.float32)
    a = (rng.standard_normal((rank, cols)) * std).astype(np.float32)
    return b, a


@pytest.mark.parametrize("rows,cols,rank,bf16", [(256, 512, 16, True), (300, 272, 64, True), (1, 16, 1, False),
                                                (129, 144, 257, False), (64, 3072, 32, True)])
def test_merge_matches_oracle(cuda_dev, rows, cols, rank, bf16):
    w = synth.weights(31, 0, rows, cols)
    if not bf16:
        w = synth.bf16_bits_to_f32(w).astype(np.float32) * np.float32(1.5)
    b, a = factors(32, rows, cols, rank)
    scale = 2.0 / rank
    wd = dev_bf16(w) if bf16 else torch.from_numpy(w).cuda()
    out = torch.full((rows, cols), float("nan"), dtype=torch.float32, device="cuda")
    nv.nvfp4_lora_merge(wd, torch.from_numpy(b).cuda(), torch.from_numpy(a).cuda(), scale, out)
    torch.cuda.synchronize()
    ref = oracle.lora_merge(w, b, a, scale)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert device_status() == nv.OK


def test_merge_then_quantize_chain(cuda_dev):
    """W (3072 x 3072 slice of an FFN weight, bf16) + rank-64 LoRA -> NVFP4."""
    rows, cols, rank = 512, 3072, 64
    w = synth.weights(33, 0, rows, cols)
    b, a = factors(34, rows, cols, rank, std=0.02)
    out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    nv.nvfp4_lora_merge(dev_bf16(w), torch.from_numpy(b).cuda(), torch.from_numpy(a).cuda(), 0.5, out)
    torch.cuda.synchronize()
    merged = oracle.lora_merge(w, b, a, 0.5)
    q, amax = gpu_quantize(out.cpu().numpy(), nv.SF_MMA, fp32=True)
    ref = oracle.quantize(merged)
    assert amax == ref.amax
    assert_quant_equal(q, ref)
