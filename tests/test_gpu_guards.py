"""Guard-byte canaries around every output buffer (no kernel writes outside its
output), and bit-determinism (every call run twice gives identical bytes)."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import synth
from gpu_helpers import dev_bf16, device_status

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """A device byte buffer with GUARD bytes of PATTERN on both sides of `nbytes`."""

    def __init__(self, nbytes):
        self.full = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.body = self.full[GUARD:GUARD + nbytes]

    def view(self, dtype, shape):
        return self.body.view(dtype).view(shape)

    def intact(self):
        f = self.full.cpu().numpy()
        return bool(np.all(f[:GUARD] == PATTERN) and np.all(f[-GUARD:] == PATTERN))


def guarded_nvfp4(rows, cols, layout=nv.SF_MMA):
    ld = ((cols // 2 + 15) // 16) * 16
    codes = Guarded(rows * ld)
    scales = Guarded(nv.scales_bytes(rows, cols, layout))
    g = Guarded(4)
    t = nv.NVFP4Tensor(rows, cols, layout, codes=codes.view(torch.uint8, (rows, ld)), scales=scales.body,
                       gscale=g.view(torch.float32, (1,)))
    return t, (codes, scales, g)


@pytest.mark.parametrize("rows,cols,layout", [(130, 528, nv.SF_MMA), (77, 48, nv.SF_ROWMAJOR), (1, 16, nv.SF_MMA)])
def test_quantize_dequantize_stay_inside_and_repeat(cuda_dev, rows, cols, layout):
    x = dev_bf16(synth.activations(51, rows, cols))
    t, guards = guarded_nvfp4(rows, cols, layout)
    amax = Guarded(4)
    outs = []
    for _ in range(2):
        nv.nvfp4_quantize(x, t, amax_out=amax.view(torch.float32, (1,)))
        torch.cuda.synchronize()
        outs.append((t.codes.cpu().numpy().copy(), t.scales.cpu().numpy().copy()))
    assert all(g.intact() for g in guards) and amax.intact()
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    y = Guarded(rows * cols * 2)
    nv.nvfp4_dequantize(t, y.view(torch.bfloat16, (rows, cols)))
    torch.cuda.synchronize()
    assert y.intact()
    assert device_status() == nv.OK


@pytest.mark.parametrize("M,N,K,fused", [(300, 272, 400, False), (129, 144, 1040, False), (513, 256, 256, False),
                                         (300, 512, 384, True), (100, 192, 256, True)])
def test_gemm_stays_inside_and_repeats(cuda_dev, M, N, K, fused):
    qa, _ = guarded_nvfp4(M, K)
    qw, _ = guarded_nvfp4(N, K)
    am = torch.zeros(2, dtype=torch.float32, device="cuda")
    nv.nvfp4_quantize(dev_bf16(synth.activations(52, M, K)), qa, amax_out=am[0:1])
    nv.nvfp4_quantize(dev_bf16(synth.weights(52, 0, N, K)), qw, amax_out=am[1:2])
    c = Guarded(M * N * 4)
    cv = c.view(torch.float32, (M, N))
    results = []
    for _ in range(2):
        if fused:
            qh, hg = guarded_nvfp4(M, N)
            h = Guarded(M * N * 4)
            amax = Guarded(4)
            gin = torch.tensor([0.01], dtype=torch.float32, device="cuda")
            nv.nvfp4_gemm(qa, qw, cv, act=nv.ACT_GELU_TANH, q_out=qh, q_gscale_in=gin,
                          q_amax_out=amax.view(torch.float32, (1,)), h_out=h.view(torch.float32, (M, N)))
            torch.cuda.synchronize()
            assert all(g.intact() for g in hg) and h.intact() and amax.intact()
            results.append((cv.cpu().numpy().copy(), qh.codes.cpu().numpy().copy(), qh.scales.cpu().numpy().copy()))
        else:
            nv.nvfp4_gemm(qa, qw, cv)
            torch.cuda.synchronize()
            results.append((cv.cpu().numpy().copy(),))
        assert c.intact()
    for a, b in zip(results[0], results[1]):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))
    assert device_status() == nv.OK


def test_kv_window_and_lora_stay_inside_and_repeat(cuda_dev):
    heads, hd, T = 3, 48, 200
    off = synth.kv_offsets(53, heads, hd)
    cache = nv.KVCache(heads, hd, T, 3)
    for s, n in enumerate((T, 37, T)):
        k, v = synth.kv_chunk(53, s, T, heads, hd, off)
        nv.kv_quant_append(cache, dev_bf16(k[:n].copy()), dev_bf16(v[:n].copy()), s)
    slots, toks = [2, 1, 0], [T, 37, T]
    total = sum(toks)
    outs = []
    for _ in range(2):
        ko, vo = Guarded(total * heads * hd * 2), Guarded(total * heads * hd * 2)
        nv.kv_dequant_window_tokens(cache, slots, toks, ko.view(torch.bfloat16, (total, heads, hd)),
                                    vo.view(torch.bfloat16, (total, heads, hd)))
        torch.cuda.synchronize()
        assert ko.intact() and vo.intact()
        outs.append((ko.body.cpu().numpy(), vo.body.cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    rows, cols, rank = 37, 80, 9
    rng = np.random.default_rng(54)
    w = torch.from_numpy(rng.standard_normal((rows, cols)).astype(np.float32)).cuda()
    lb = torch.from_numpy(rng.standard_normal((rows, rank)).astype(np.float32)).cuda()
    la = torch.from_numpy(rng.standard_normal((rank, cols)).astype(np.float32)).cuda()
    o = Guarded(rows * cols * 4)
    nv.nvfp4_lora_merge(w, lb, la, 0.3, o.view(torch.float32, (rows, cols)))
    torch.cuda.synchronize()
    assert o.intact()
    assert device_status() == nv.OK
