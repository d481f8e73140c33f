"""Shared helpers of the GPU parity tests: move synthetic inputs to the device,
run the library through its binding, and bring results back as numpy arrays in
the oracle's canonical layouts."""
import numpy as np
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bits (numpy) -> bf16 CUDA tensor with the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.to("cuda").view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> uint16 numpy bits."""
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def gpu_quantize(x: np.ndarray, layout=nv.SF_MMA, gscale=None, fp32=False):
    """Quantize on the GPU; returns (NVFP4Tensor, amax float)."""
    if fp32:
        xd = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    else:
        xd = dev_bf16(x)
    rows, cols = x.shape
    out = nv.NVFP4Tensor(rows, cols, layout)
    amax = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    gin = None if gscale is None else torch.tensor([gscale], dtype=torch.float32, device="cuda")
    nv.nvfp4_quantize(xd, out, gscale_in=gin, amax_out=amax)
    torch.cuda.synchronize()
    return out, float(amax.item())


def canonical(t: nv.NVFP4Tensor):
    """(codes [rows, cols/2], scales [rows, cols/16], g) in the oracle's layout."""
    codes = t.codes.cpu().numpy()[:, : t.cols // 2]
    raw = t.scales.cpu().numpy()
    if t.sf_layout == nv.SF_MMA:
        scales = oracle.sf_from_mma(raw, t.rows, t.cols)
    else:
        scales = raw.reshape(t.rows, t.cols // 16)
    return codes, scales, float(t.gscale.item())


def mma_padding_is_zero(t: nv.NVFP4Tensor) -> bool:
    raw = t.scales.cpu().numpy()
    used = np.zeros(raw.size, bool)
    nb = t.cols // 16
    r = np.arange(t.rows)[:, None]
    j = np.arange(nb)[None, :]
    groups = (nb + 3) // 4
    off = ((r // 128) * groups + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)
    used[off.ravel()] = True
    return bool(np.all(raw[~used] == 0))


def assert_quant_equal(gpu: nv.NVFP4Tensor, ref: oracle.Quantized):
    codes, scales, g = canonical(gpu)
    assert g == ref.g, (g, ref.g)
    bad_s = np.argwhere(scales != ref.scales)
    assert bad_s.size == 0, f"{len(bad_s)} scale mismatches, first {bad_s[:3].tolist()}"
    bad_c = np.argwhere(codes != ref.codes)
    assert bad_c.size == 0, f"{len(bad_c)} code-byte mismatches, first {bad_c[:3].tolist()}"


def device_status(clear=True) -> int:
    return nv.get_device_status(torch.cuda.current_device(), clear=clear)
