"""GPU parity of kv_window_scores (attention scores with K read from the NVFP4 cache
inside the kernel) against the oracle: the float64 product of the queries with the
oracle's dequantized K of the window (techwalker.com, "NVIDIA研究团队打造全球首个FP4视频
生成系统，速度提升两倍还省一半内存", §四: the window's cache chunks are dequantized
together for attention).  Every score within 1e-5 of sum_d |q_d k_d| (times |scale|)
of the exact value; bf16 outputs add half a bf16 ulp."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle
import synth
from gpu_helpers import dev_bf16, device_status

pytestmark = pytest.mark.gpu

TOL = 1e-5


def build_cache(heads, chunk, fills, seed):
    """A cache whose slot s holds fills[s] tokens; the oracle's K^ of each slot."""
    D = 128
    off = synth.kv_offsets(seed, heads, D)
    cache = nv.KVCache(heads, D, chunk, len(fills))
    khat = []
    for s, n in enumerate(fills):
        k, v = synth.kv_chunk(seed, s, chunk, heads, D, off)
        k, v = k[:n].copy(), v[:n].copy()
        nv.kv_quant_append(cache, dev_bf16(k), dev_bf16(v), s)
        khat.append(oracle.kv_dequant_chunk(oracle.kv_append(k, v))[0])
    torch.cuda.synchronize()
    return cache, khat


def reference(q_bits, khat, slots, tokens, scale):
    """Exact scores in float64 (bf16 x bf16 products are exact) and sum |q k|."""
    keys = np.concatenate([khat[s][:t] for s, t in zip(slots, tokens)])  # [Tk, H, D] bf16 bits
    qf = synth.bf16_bits_to_f32(q_bits).astype(np.float64)      # [Tq, H, D]
    kf = synth.bf16_bits_to_f32(keys).astype(np.float64)        # [Tk, H, D]
    s = np.einsum("ihd,jhd->hij", qf, kf) * scale
    b = np.einsum("ihd,jhd->hij", np.abs(qf), np.abs(kf)) * abs(scale)
    return s, b


def queries(seed, tq, heads):
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal((tq, heads, 128)) * 1.5).astype(np.float32)
    return (q.view(np.uint32) >> 16).astype(np.uint16)  # truncation to bf16 bits is fine for inputs


def run_scores(cache, khat, slots, tokens, tq, heads, out_dtype, scale, seed, pad=16):
    q = queries(seed, tq, heads)
    tk = int(sum(tokens))
    ld = (tk + pad + 7) // 8 * 8  # 16-byte row pitch for FP32 and bf16
    s_out = torch.full((heads, tq, ld), float("nan"), dtype=out_dtype, device="cuda")
    nv.kv_window_scores(cache, slots, tokens, dev_bf16(q), scale, s_out)
    torch.cuda.synchronize()
    got = s_out.float().cpu().numpy().astype(np.float64)
    ref, bound = reference(q, khat, slots, tokens, scale)
    return got, ref, bound, tk


def assert_scores(got, ref, bound, tk, extra_rel=0.0, esz=4):
    g = got[:, :, :tk]
    err = np.abs(g - ref)
    lim = TOL * bound + extra_rel * np.abs(ref)
    assert np.all(err <= lim), f"{int(np.sum(err > lim))} scores outside the bound"
    pad_end = (tk * esz + 15) // 16 * 16 // esz  # the row's next 16-byte boundary
    assert np.all(got[:, :, tk:pad_end] == 0), "the padding up to the 16-byte boundary holds zeros"
    assert np.all(np.isnan(got[:, :, pad_end:])), "columns beyond the padding were written"


@pytest.mark.parametrize("tq", [1, 128, 200])
def test_ragged_window_fp32(cuda_dev, tq):
    """Three slots, partial fills, listed out of order: 77 + 256 + 200 = 533 keys
    (four full 128-key tiles and a ragged one, two of them straddling slots)."""
    cache, khat = build_cache(heads=2, chunk=256, fills=[256, 200, 77], seed=5)
    slots, tokens = [2, 0, 1], [77, 256, 200]
    got, ref, bound, tk = run_scores(cache, khat, slots, tokens, tq, 2, torch.float32, 1.0 / np.sqrt(128.0), 9)
    assert_scores(got, ref, bound, tk)
    assert device_status() == nv.OK


def test_bf16_output_and_repeated_slots(cuda_dev):
    cache, khat = build_cache(heads=3, chunk=192, fills=[192, 192], seed=6)
    slots, tokens = [1, 0, 1], [192, 192, 192]
    got, ref, bound, tk = run_scores(cache, khat, slots, tokens, 300, 3, torch.bfloat16, 0.125, 10)
    assert_scores(got, ref, bound, tk, extra_rel=2.0 ** -8, esz=2)
    assert device_status() == nv.OK


def test_matches_the_window_dequant_then_float64_product(cuda_dev):
    """The kernel's K^ is the window's: the same scores from the GPU's own
    kv_dequant_window_tokens output (bit-identical to the oracle's K^)."""
    cache, khat = build_cache(heads=2, chunk=256, fills=[256, 130], seed=7)
    slots, tokens = [1, 0], [130, 256]
    ko = torch.empty((386, 2, 128), dtype=torch.bfloat16, device="cuda")
    nv.kv_dequant_window_tokens(cache, slots, tokens, ko, torch.empty_like(ko))
    torch.cuda.synchronize()
    kh = ko.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(kh, np.concatenate([khat[1][:130], khat[0][:256]]))
    got, ref, bound, tk = run_scores(cache, khat, slots, tokens, 64, 2, torch.float32, -0.5, 11)
    assert_scores(got, ref, bound, tk)


def test_wrong_token_count_sets_shape_status(cuda_dev):
    cache, _ = build_cache(heads=1, chunk=128, fills=[128, 100], seed=8)
    q = dev_bf16(queries(12, 16, 1))
    s_out = torch.zeros((1, 16, 256), dtype=torch.float32, device="cuda")
    device_status(clear=True)
    nv.kv_window_scores(cache, [0, 1], [128, 128], q, 1.0, s_out)  # slot 1 holds 100 tokens
    torch.cuda.synchronize()
    assert device_status() == nv.ERR_SHAPE


def test_host_checks(cuda_dev):
    cache = nv.KVCache(2, 64, 64, 1)  # head_dim 64: not supported by the scores kernel
    q = torch.zeros((4, 2, 64), dtype=torch.bfloat16, device="cuda")
    s_out = torch.zeros((2, 4, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.kv_window_scores(cache, [0], [64], q, 1.0, s_out)
    assert e.value.status == nv.ERR_SHAPE


@pytest.mark.slow
def test_full_size_window_sampled_heads(cuda_dev):
    """24 heads x 128, four chunks of 8192 tokens (32768 keys), 256 queries, FP32
    scores: heads 0, 11 and 23 checked against the oracle's K^ in full."""
    heads, chunk = 24, 8192
    off = synth.kv_offsets(3, heads, 128)
    cache = nv.KVCache(heads, 128, chunk, 4)
    khat = []
    for s in range(4):
        k, v = synth.kv_chunk(3, s, chunk, heads, 128, off)
        nv.kv_quant_append(cache, dev_bf16(k), dev_bf16(v), s)
        khat.append(oracle.kv_dequant_chunk(oracle.kv_append(k, v))[0])
    q = queries(13, 256, heads)
    s_out = torch.empty((heads, 256, 4 * chunk), dtype=torch.float32, device="cuda")
    nv.kv_window_scores(cache, [0, 1, 2, 3], [chunk] * 4, dev_bf16(q), 1.0 / np.sqrt(128.0), s_out)
    torch.cuda.synchronize()
    assert device_status() == nv.OK
    for h in (0, 11, 23):
        keys = np.concatenate(khat)[:, h]
        qf = synth.bf16_bits_to_f32(q[:, h]).astype(np.float64)
        kf = synth.bf16_bits_to_f32(keys).astype(np.float64)
        ref = (qf @ kf.T) / np.sqrt(128.0)
        bound = (np.abs(qf) @ np.abs(kf).T) / np.sqrt(128.0)
        got = s_out[h].cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= TOL * bound), f"head {h}"
