"""Row-sharded quantization on the GPU, its ranks emulated one after another on one
device: nvfp4_amax of each shard, the all-reduce(MAX) over the shards' amax bit
patterns, the one-entry amax history for g, then nvfp4_quantize of every shard with
that g.  Codes, scales and g are bit-identical to one nvfp4_quantize of the whole
tensor and to the oracle (no kernel here waits on another)."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle
import synth
from gpu_helpers import assert_quant_equal, canonical, dev_bf16, device_status
from nvfp4_w4a4_quantized_amax_b200 import sharded

pytestmark = pytest.mark.gpu


class EmulatedGroupOps(sharded.LibraryOps):
    """LibraryOps whose all-reduce is done by the test across the emulated ranks."""

    def all_reduce_max(self, ws):
        pass


@pytest.mark.parametrize("rows,cols,world", [(1000, 3072, 3), (257, 512, 2), (8192, 3072, 8)])
def test_sharded_quantize_matches_whole_tensor(cuda_dev, rows, cols, world):
    x = synth.activations(12, rows, cols)
    xd = dev_bf16(x)
    ops = EmulatedGroupOps()
    shards = [sharded.row_range(rows, r, world) for r in range(world)]
    ws = [sharded.ShardWorkspace.create("cuda") for _ in range(world)]
    outs = [nv.NVFP4Tensor(r1 - r0, cols, nv.SF_ROWMAJOR) for r0, r1 in shards]
    for (r0, r1), w in zip(shards, ws):
        ops.amax(xd[r0:r1], w)
    m = torch.stack([w.amax.view(torch.int32) for w in ws]).amax(dim=0)  # the all-reduce(MAX)
    for w in ws:
        w.amax.view(torch.int32).copy_(m)
    for (r0, r1), w, o in zip(shards, ws, outs):
        ops.tensor_scale(w)
        ops.quantize(xd[r0:r1], o, w)
    torch.cuda.synchronize()
    assert device_status() == nv.OK
    ref = oracle.quantize(x)
    whole = nv.NVFP4Tensor(rows, cols, nv.SF_ROWMAJOR)
    nv.nvfp4_quantize(xd, whole, amax_out=torch.zeros(1, device="cuda"))
    assert_quant_equal(whole, ref)
    for (r0, r1), o in zip(shards, outs):
        codes, scales, g = canonical(o)
        assert g == ref.g
        assert np.array_equal(codes, ref.codes[r0:r1]) and np.array_equal(scales, ref.scales[r0:r1])


def test_amax_entry_point(cuda_dev):
    x = synth.activations(13, 129, 144)
    amax = torch.full((1,), -1.0, device="cuda")
    nv.nvfp4_amax(dev_bf16(x), amax)
    assert amax.item() == oracle.quantize(x).amax
    xf = np.random.default_rng(0).standard_normal((33, 48)).astype(np.float32)
    nv.nvfp4_amax(torch.from_numpy(xf).cuda(), amax)
    assert amax.item() == float(np.abs(xf).max())
    xf[5, 7] = np.inf
    nv.nvfp4_amax(torch.from_numpy(xf).cuda(), amax)
    assert amax.item() == float("inf")
    nv.nvfp4_amax(torch.empty((0, 16), dtype=torch.bfloat16, device="cuda"), amax)
    assert amax.item() == 0.0
    assert device_status() == nv.OK
