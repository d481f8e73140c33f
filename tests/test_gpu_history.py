"""GPU parity of nvfp4_amax_history_push against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle
from gpu_helpers import device_status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("length", [1, 3, 16, 1024])
def test_history_pushes_match_oracle(cuda_dev, length):
    rng = np.random.default_rng(length)
    hist = torch.zeros(length, dtype=torch.float32, device="cuda")
    ref = np.zeros(length, np.float32)
    new = torch.zeros(1, dtype=torch.float32, device="cuda")
    g = torch.zeros(1, dtype=torch.float32, device="cuda")
    for step in range(40):
        a = np.float32(np.exp(rng.normal(0, 3)))
        new.fill_(float(a))
        nv.nvfp4_amax_history_push(hist, new, g)
        ref, gref = oracle.amax_history_push(ref, a)
        torch.cuda.synchronize()
        assert np.array_equal(hist.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        assert g.item() == gref
    assert device_status() == nv.OK


def test_nonfinite_push_changes_nothing(cuda_dev):
    hist = torch.tensor([3.0, 2.0, 1.0], dtype=torch.float32, device="cuda")
    g = torch.tensor([0.125], dtype=torch.float32, device="cuda")
    device_status(clear=True)
    nv.nvfp4_amax_history_push(hist, torch.tensor([float("nan")], device="cuda"), g)
    assert device_status(clear=True) == nv.ERR_NONFINITE
    assert hist.cpu().tolist() == [3.0, 2.0, 1.0] and g.item() == 0.125
    assert device_status() == nv.OK
