"""Bounded waits: with the test hook that makes every CTA's GEMM producer skip its
first pipeline stage, or the one that makes the grid barrier of the one-launch
quantize wait for more CTAs than the grid has, the waits run out,
the call reports NVFP4_ERR_TIMEOUT in the device status word, returns in bounded
time, and the context stays usable (the next call is correct)."""
import time

import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle
import synth
from gpu_helpers import assert_quant_equal, canonical, dev_bf16, device_status, gpu_quantize

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (256, 256, 256)])  # single-CTA and CTA-pair kernels
def test_gemm_wait_timeout_is_reported_and_the_context_survives(cuda_dev, M, N, K):
    qa, _ = gpu_quantize(synth.activations(41, M, K), nv.SF_MMA)
    qw, _ = gpu_quantize(synth.weights(41, 0, N, K), nv.SF_MMA)
    c = torch.empty((M, N), dtype=torch.float32, device="cuda")
    assert device_status(clear=True) == nv.OK
    nv.debug_gemm_fault(True, 20_000_000)  # 20 ms per wait
    try:
        t0 = time.time()
        nv.nvfp4_gemm(qa, qw, c)
        torch.cuda.synchronize()
        elapsed = time.time() - t0
    finally:
        nv.debug_gemm_fault(False, 0)
    assert device_status(clear=True) == nv.ERR_TIMEOUT
    assert elapsed < 5.0
    # the same GEMM again, without the hook: correct and no error
    nv.nvfp4_gemm(qa, qw, c)
    torch.cuda.synchronize()
    assert device_status() == nv.OK
    ac, asc, ag = canonical(qa)
    wc, wsc, wg = canonical(qw)
    ref, bound = oracle.gemm_ref(ac, asc, ag, wc, wsc, wg)
    assert np.all(np.abs(c.cpu().numpy().astype(np.float64) - ref) <= 1e-5 * bound)


def test_grid_barrier_timeout_in_one_launch_quantize(cuda_dev):
    x = synth.activations(42, 512, 1024)  # small: the one-launch path
    assert device_status(clear=True) == nv.OK
    nv.debug_grid_barrier(1, 20_000_000)  # one CTA more than the grid has, 20 ms
    try:
        t0 = time.time()
        gpu_quantize(x, nv.SF_MMA)
        elapsed = time.time() - t0
    finally:
        nv.debug_grid_barrier(0, 0)
    assert device_status(clear=True) == nv.ERR_TIMEOUT
    assert elapsed < 5.0
    q, _ = gpu_quantize(x, nv.SF_MMA)
    assert device_status() == nv.OK
    assert_quant_equal(q, oracle.quantize(x))
