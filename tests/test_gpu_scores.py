"""GPU parity of the attention-side consumers of the NVFP4 KV cache against the
oracle (techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存",
§四: the window's cache chunks are dequantized together for attention):
kv_window_scores (K read from the cache inside the kernel) against the float64
product of the queries with the oracle's dequantized K, and kv_window_context (V read
from the cache inside the kernel) against the float64 product of the weights with the
oracle's dequantized V.  Every output within 1e-5 of the sum of the absolute products
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


def build_cache(heads, chunk, fills, seed, with_v=False):
    """A cache whose slot s holds fills[s] tokens; the oracle's K^ (and V^) of each slot."""
    D = 128
    off = synth.kv_offsets(seed, heads, D)
    cache = nv.KVCache(heads, D, chunk, len(fills))
    khat, vhat = [], []
    for s, n in enumerate(fills):
        k, v = synth.kv_chunk(seed, s, chunk, heads, D, off)
        k, v = k[:n].copy(), v[:n].copy()
        nv.kv_quant_append(cache, dev_bf16(k), dev_bf16(v), s)
        kh, vh = oracle.kv_dequant_chunk(oracle.kv_append(k, v))
        khat.append(kh)
        vhat.append(vh)
    torch.cuda.synchronize()
    return (cache, khat, vhat) if with_v else (cache, khat)


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


# ------------------------------------------------------------------ the V side

def weights(seed, heads, tq, ld):
    """bf16 weights in [0, 1) with a ragged row pitch beyond the window (NaN there:
    the kernel must not read past Tk)."""
    rng = np.random.default_rng(seed)
    w = rng.random((heads, tq, ld)).astype(np.float32)
    bits = (w.view(np.uint32) >> 16).astype(np.uint16)
    return bits


def run_context(cache, vhat, slots, tokens, tq, heads, out_dtype, seed):
    tk = int(sum(tokens))
    ld = (tk + 16 + 7) // 8 * 8
    pb = weights(seed, heads, tq, ld)
    pb[:, :, tk:] = 0x7FC0  # NaN beyond the window
    o = torch.full((tq, heads, 128), float("nan"), dtype=out_dtype, device="cuda")
    nv.kv_window_context(cache, slots, tokens, dev_bf16(pb), o)
    torch.cuda.synchronize()
    vals = np.concatenate([vhat[s][:t] for s, t in zip(slots, tokens)])     # [Tk, H, D]
    pf = synth.bf16_bits_to_f32(pb[:, :, :tk]).astype(np.float64)            # [H, Tq, Tk]
    vf = synth.bf16_bits_to_f32(vals).astype(np.float64)
    ref = np.einsum("hij,jhd->ihd", pf, vf)
    bound = np.einsum("hij,jhd->ihd", np.abs(pf), np.abs(vf))
    return o.float().cpu().numpy().astype(np.float64), ref, bound


@pytest.mark.parametrize("tq", [1, 130])
def test_context_ragged_window(cuda_dev, tq):
    cache, _, vhat = build_cache(heads=2, chunk=256, fills=[256, 200, 77], seed=15, with_v=True)
    got, ref, bound = run_context(cache, vhat, [2, 0, 1], [77, 256, 200], tq, 2, torch.float32, 16)
    assert np.all(np.abs(got - ref) <= TOL * bound), float(np.max(np.abs(got - ref) / np.maximum(bound, 1e-300)))
    assert device_status() == nv.OK


def test_context_bf16_output_repeated_slots(cuda_dev):
    cache, _, vhat = build_cache(heads=3, chunk=192, fills=[192, 192], seed=17, with_v=True)
    got, ref, bound = run_context(cache, vhat, [1, 0, 1], [192, 192, 192], 200, 3, torch.bfloat16, 18)
    assert np.all(np.abs(got - ref) <= TOL * bound + 2.0 ** -8 * np.abs(ref))
    assert device_status() == nv.OK


@pytest.mark.parametrize("heads,chunk,fills,slots,tokens,tq,dtype", [
    # 16 key tiles: the keys of each (query tile, head) split over a cluster of two CTAs
    (2, 1024, [1024, 1000], [1, 0], [1000, 1024], 130, torch.float32),
    # 72 key tiles (slot boundaries inside tiles): eight CTAs, the last range ragged
    (1, 4096, [4096, 4096, 900], [2, 0, 1], [900, 4096, 4096], 70, torch.bfloat16),
])
def test_context_keys_split_across_a_cluster(cuda_dev, heads, chunk, fills, slots, tokens, tq, dtype):
    """Few query tiles against many keys: the partial outputs of the CTAs of a cluster are
    summed over distributed shared memory; the result stays within the FP32 bound."""
    cache, _, vhat = build_cache(heads=heads, chunk=chunk, fills=fills, seed=23, with_v=True)
    device_status(clear=True)
    got, ref, bound = run_context(cache, vhat, slots, tokens, tq, heads, dtype, 24)
    extra = 2.0 ** -8 * np.abs(ref) if dtype == torch.bfloat16 else 0.0
    assert np.all(np.abs(got - ref) <= TOL * bound + extra)
    assert device_status() == nv.OK


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_context_many_query_tiles_one_key_tile(cuda_dev, dtype):
    """60 keys (one 64-key tile, so no key split) against 12763 queries of 4 heads: the
    grid no longer fits one wave, so each CTA takes several query tiles (three; the last
    group one, the last tile ragged) and writes its accumulators straight out."""
    heads, tq = 4, 12763
    cache, _, vhat = build_cache(heads=heads, chunk=64, fills=[60], seed=31, with_v=True)
    device_status(clear=True)
    got, ref, bound = run_context(cache, vhat, [0], [60], tq, heads, dtype, 32)
    extra = 2.0 ** -8 * np.abs(ref) if dtype == torch.bfloat16 else 0.0
    assert np.all(np.abs(got - ref) <= TOL * bound + extra)
    assert device_status() == nv.OK


def test_context_wrong_token_count_sets_shape_status(cuda_dev):
    cache, _, _ = build_cache(heads=1, chunk=2048, fills=[2048, 100], seed=25, with_v=True)
    p = torch.zeros((1, 8, 4096), dtype=torch.bfloat16, device="cuda")
    o = torch.empty((8, 1, 128), dtype=torch.float32, device="cuda")
    device_status(clear=True)
    nv.kv_window_context(cache, [0, 1], [2048, 2048], p, o)  # slot 1 holds 100 tokens
    torch.cuda.synchronize()
    assert device_status() == nv.ERR_SHAPE
    assert torch.all(o == 0)  # its keys are read as zeros


def test_many_tiny_slots_scores_and_context(cuda_dev):
    """40 slots of 1..8 tokens listed out of order: every key tile straddles many slots
    (the decoders' slot tracking, the per-slot g and mu); the output's 3 key tiles of
    64 go to a cluster of three CTAs with an uneven row split."""
    rng = np.random.default_rng(27)
    fills = [int(x) for x in rng.integers(1, 9, size=40)]
    cache, khat, vhat = build_cache(heads=3, chunk=8, fills=fills, seed=28, with_v=True)
    order = [int(x) for x in rng.permutation(40)]
    tokens = [fills[i] for i in order]
    device_status(clear=True)
    got, ref, bound, tk = run_scores(cache, khat, order, tokens, 150, 3, torch.float32, 0.125, 29)
    assert_scores(got, ref, bound, tk)
    got, ref, bound = run_context(cache, vhat, order, tokens, 150, 3, torch.float32, 30)
    assert np.all(np.abs(got - ref) <= TOL * bound)
    assert device_status() == nv.OK


def test_attention_from_the_cache_end_to_end(cuda_dev):
    """scores -> softmax (torch, FP32, then bf16 weights) -> context, against attention in
    float64 on the oracle's K^ and V^: the bf16 weights bound the error (2^-8 of sum p|v|)."""
    heads, tq = 2, 96
    cache, khat, vhat = build_cache(heads=heads, chunk=256, fills=[256, 150], seed=19, with_v=True)
    slots, tokens = [0, 1], [256, 150]
    tk = 406
    q = queries(20, tq, heads)
    scale = 1.0 / np.sqrt(128.0)
    s_out = torch.empty((heads, tq, 408), dtype=torch.float32, device="cuda")
    nv.kv_window_scores(cache, slots, tokens, dev_bf16(q), scale, s_out)
    p = torch.softmax(s_out[:, :, :tk], dim=-1).to(torch.bfloat16)
    p_full = torch.zeros((heads, tq, 408), dtype=torch.bfloat16, device="cuda")
    p_full[:, :, :tk] = p
    o = torch.empty((tq, heads, 128), dtype=torch.float32, device="cuda")
    nv.kv_window_context(cache, slots, tokens, p_full, o)
    torch.cuda.synchronize()
    assert device_status() == nv.OK
    sref, _ = reference(q, khat, slots, tokens, scale)
    pref = np.exp(sref - sref.max(axis=-1, keepdims=True))
    pref /= pref.sum(axis=-1, keepdims=True)
    vals = synth.bf16_bits_to_f32(np.concatenate([vhat[s][:t] for s, t in zip(slots, tokens)])).astype(np.float64)
    oref = np.einsum("hij,jhd->ihd", pref, vals)
    bound = np.einsum("hij,jhd->ihd", pref, np.abs(vals))
    assert np.all(np.abs(o.cpu().numpy() - oref) <= 2.0 ** -8 * bound + 1e-6)


@pytest.mark.slow
def test_context_full_size_window_sampled_heads(cuda_dev):
    """24 heads x 128, four chunks of 8192 tokens (32768 keys), 256 queries, FP32 out:
    heads 0, 11 and 23 checked against the oracle's V^ in full."""
    heads, chunk = 24, 8192
    off = synth.kv_offsets(21, heads, 128)
    cache = nv.KVCache(heads, 128, chunk, 4)
    vhat = []
    for s in range(4):
        k, v = synth.kv_chunk(21, s, chunk, heads, 128, off)
        nv.kv_quant_append(cache, dev_bf16(k), dev_bf16(v), s)
        vhat.append(oracle.kv_dequant_chunk(oracle.kv_append(k, v))[1])
    tk = 4 * chunk
    pb = weights(22, heads, 256, tk)
    o = torch.empty((256, heads, 128), dtype=torch.float32, device="cuda")
    nv.kv_window_context(cache, [0, 1, 2, 3], [chunk] * 4, dev_bf16(pb), o)
    torch.cuda.synchronize()
    assert device_status() == nv.OK
    vals = np.concatenate(vhat)
    got = o.cpu().numpy().astype(np.float64)
    for h in (0, 11, 23):
        pf = synth.bf16_bits_to_f32(pb[h]).astype(np.float64)
        vf = synth.bf16_bits_to_f32(vals[:, h]).astype(np.float64)
        ref = pf @ vf
        bound = pf @ np.abs(vf)
        assert np.all(np.abs(got[:, h] - ref) <= TOL * bound), f"head {h}"
