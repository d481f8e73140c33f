"""GPU parity of the NVFP4 KV cache against the oracle: per-(head, dim) mean,
tensor scales, codes and scales of K' and V bit for bit after each append, and the
multi-chunk window dequantization bit for bit."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle
import synth
from gpu_helpers import dev_bf16, device_status, host_bits

pytestmark = pytest.mark.gpu


def check_slot(cache, slot, ref):
    kc, ks, vc, vs, mu, g = cache.slot_views(slot)
    T, H, Dh = ref.T, ref.H, ref.Dh
    assert np.array_equal(mu.cpu().numpy().view(np.uint32), ref.mu.view(np.uint32)), "mu"
    gk, gv = g.cpu().numpy().tolist()
    assert gk == ref.g_k and gv == ref.g_v
    assert np.array_equal(ks.cpu().numpy(), ref.k_scales.ravel()), "K scales"
    assert np.array_equal(kc.cpu().numpy(), ref.k_codes.ravel()), "K codes"
    assert np.array_equal(vs.cpu().numpy(), ref.v_scales.ravel()), "V scales"
    assert np.array_equal(vc.cpu().numpy(), ref.v_codes.ravel()), "V codes"


def run_cache(heads, head_dim, T, chunks, window, seed, full_window_check=True, plant=None):
    off = synth.kv_offsets(seed, heads, head_dim)
    cache = nv.KVCache(heads, head_dim, T, chunks)
    refs = []
    for c in range(chunks):
        k, v = synth.kv_chunk(seed, c, T, heads, head_dim, off)
        if plant is not None:
            plant(c, k, v)
        nv.kv_quant_append(cache, dev_bf16(k), dev_bf16(v), c)
        ref = oracle.kv_append(k, v)
        torch.cuda.synchronize()
        check_slot(cache, c, ref)
        refs.append(ref)
    assert device_status() == nv.OK
    slots = list(range(chunks - window, chunks))
    C = heads * head_dim
    ko = torch.empty((window * T, heads, head_dim), dtype=torch.bfloat16, device="cuda")
    vo = torch.empty_like(ko)
    nv.kv_dequant_window(cache, slots, ko, vo)
    kh, vh = host_bits(ko), host_bits(vo)
    for i, s in enumerate(slots if full_window_check else slots[-1:]):
        i = slots.index(s)
        rk, rv = oracle.kv_dequant_chunk(refs[s])
        assert np.array_equal(kh[i * T:(i + 1) * T], rk), f"K^ window entry {i}"
        assert np.array_equal(vh[i * T:(i + 1) * T], rv), f"V^ window entry {i}"
    return cache, refs


def test_small_cache_ragged_geometry(cuda_dev):
    # C = 144 columns (not a multiple of the 256-column stats tile), T = 1000 tokens
    # (not a power of two: the mean needs a correctly rounded division)
    run_cache(heads=3, head_dim=48, T=1000, chunks=3, window=2, seed=3)


def test_window_order_repeats_and_any_slot_list(cuda_dev):
    cache, refs = run_cache(heads=2, head_dim=64, T=256, chunks=4, window=4, seed=8)
    slots = [3, 0, 0, 2, 1]
    T = 256
    ko = torch.empty((len(slots) * T, 2, 64), dtype=torch.bfloat16, device="cuda")
    vo = torch.empty_like(ko)
    nv.kv_dequant_window(cache, slots, ko, vo)
    kh, vh = host_bits(ko), host_bits(vo)
    for i, s in enumerate(slots):
        rk, rv = oracle.kv_dequant_chunk(refs[s])
        assert np.array_equal(kh[i * T:(i + 1) * T], rk)
        assert np.array_equal(vh[i * T:(i + 1) * T], rv)


def test_wide_range_columns_take_the_exact_path(cuda_dev):
    """Columns whose magnitudes span more binades than a double sum can hold exactly:
    the mean must still equal the exactly rounded one."""
    def plant(c, k, v):
        flat = k.reshape(k.shape[0], -1)
        flat[5, 7] = 0x7E80       # 8.5e37
        flat[9, 7] = 0x0001       # smallest bf16 subnormal
        flat[11, 7] = 0xFE80      # -8.5e37: cancels, leaving tiny terms
        flat[3, 33] = 0x4F00      # 2^31
        flat[4, 33] = 0x2F80      # 2^-32
        flat[:, 40] = 0           # an all-zero column
        flat[:, 41] = 0x3F80      # a constant column
    run_cache(heads=2, head_dim=32, T=64, chunks=2, window=2, seed=4, plant=plant)


@pytest.mark.parametrize("where,bits", [("v", 0x7F80), ("v", 0xFF80), ("v", 0x7FC0),
                                        ("k", 0x7F80), ("k", 0xFF80), ("k", 0x7FC0), ("k", 0xFFC1)])
def test_nonfinite_chunk_leaves_slot_unchanged(cuda_dev, where, bits):
    """+-inf and +-NaN in K or V: NONFINITE in the device status, the slot keeps its
    previous contents."""
    heads, dh, T = 2, 32, 64
    off = synth.kv_offsets(1, heads, dh)
    cache = nv.KVCache(heads, dh, T, 2)
    k, v = synth.kv_chunk(1, 0, T, heads, dh, off)
    nv.kv_quant_append(cache, dev_bf16(k), dev_bf16(v), 0)
    ref = oracle.kv_append(k, v)
    device_status(clear=True)
    k2, v2 = synth.kv_chunk(1, 1, T, heads, dh, off)
    (v2 if where == "v" else k2)[7, 1, 3] = bits
    with pytest.raises(FloatingPointError):  # the oracle rejects the chunk too
        oracle.kv_append(k2, v2)
    nv.kv_quant_append(cache, dev_bf16(k2), dev_bf16(v2), 0)
    assert device_status(clear=True) == nv.ERR_NONFINITE
    check_slot(cache, 0, ref)


def test_signed_zero_and_one_signed_columns(cuda_dev):
    """Columns of -0 only, of +0 and -0, of negative values only, of positive values
    only, and of subnormals only: max, min, mean and the smallest nonzero magnitude
    of every column as the oracle has them."""
    def plant(c, k, v):
        flat = k.reshape(k.shape[0], -1)
        flat[:, 50] = 0x8000                 # -0 everywhere
        flat[:, 51] = 0x8000
        flat[::2, 51] = 0x0000               # +0 and -0
        flat[:, 52] = 0xBF80                 # -1 ...
        flat[::3, 52] = 0xC040               # ... and -3
        flat[:, 53] = 0x3F80                 # +1 ...
        flat[1::4, 53] = 0x4100              # ... and +8
        flat[:, 54] = 0x0003                 # subnormals ...
        flat[::5, 54] = 0x8005               # ... of both signs
    run_cache(heads=2, head_dim=32, T=64, chunks=2, window=2, seed=6, plant=plant)


@pytest.mark.slow
def test_full_size_cache_24x128_8192_tokens(cuda_dev):
    """24 heads x 128, chunks of 8192 tokens: 5 appends (every slot checked) and a
    4-chunk window of 32768 tokens, all values compared."""
    run_cache(heads=24, head_dim=128, T=8192, chunks=5, window=4, seed=3)


def check_slot_prefix(cache, slot, ref):
    """A slot holding ref.T tokens (possibly fewer than chunk_tokens): its first tokens."""
    kc, ks, vc, vs, mu, g = cache.slot_views(slot)
    C = ref.H * ref.Dh
    nc, ns = ref.T * C // 2, ref.T * C // 16
    assert cache.slot_tokens(slot) == ref.T
    assert np.array_equal(mu.cpu().numpy().view(np.uint32), ref.mu.view(np.uint32)), "mu"
    gk, gv = g.cpu().numpy().tolist()
    assert gk == ref.g_k and gv == ref.g_v
    assert np.array_equal(kc[:nc].cpu().numpy(), ref.k_codes.ravel()), "K codes"
    assert np.array_equal(ks[:ns].cpu().numpy(), ref.k_scales.ravel()), "K scales"
    assert np.array_equal(vc[:nc].cpu().numpy(), ref.v_codes.ravel()), "V codes"
    assert np.array_equal(vs[:ns].cpu().numpy(), ref.v_scales.ravel()), "V scales"


def test_partial_chunks_and_sink_aware_window(cuda_dev):
    """Slots holding 17, 1, 1000, 333 and all 2048 tokens; a sink-aware window lists a
    sink slot, a shot-sink slot, the sliding slots (one partial) and a repeat."""
    heads, hd, T = 4, 64, 2048
    off = synth.kv_offsets(9, heads, hd)
    cache = nv.KVCache(heads, hd, T, 6)
    fills = {0: 17, 1: T, 2: 1, 3: 1000, 4: T, 5: 333}
    refs = {}
    for slot, n in fills.items():
        k, v = synth.kv_chunk(9, slot, T, heads, hd, off)
        k, v = np.ascontiguousarray(k[:n]), np.ascontiguousarray(v[:n])
        nv.kv_quant_append(cache, dev_bf16(k), dev_bf16(v), slot)
        refs[slot] = oracle.kv_append(k, v)
        torch.cuda.synchronize()
        check_slot_prefix(cache, slot, refs[slot])
    slots = [0, 2, 3, 4, 5, 1, 3]
    toks = [fills[s] for s in slots]
    ko = torch.full((sum(toks), heads, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    vo = torch.full_like(ko, float("nan"))
    nv.kv_dequant_window_tokens(cache, slots, toks, ko, vo)
    kh, vh = host_bits(ko), host_bits(vo)
    row = 0
    for s, n in zip(slots, toks):
        rk, rv = oracle.kv_dequant_chunk(refs[s])
        assert np.array_equal(kh[row:row + n], rk), f"K^ slot {s}"
        assert np.array_equal(vh[row:row + n], rv), f"V^ slot {s}"
        row += n
    assert device_status() == nv.OK


def test_window_token_count_mismatch_sets_status_and_skips_the_slot(cuda_dev):
    heads, hd, T = 2, 32, 256
    off = synth.kv_offsets(10, heads, hd)
    cache = nv.KVCache(heads, hd, T, 2)
    k, v = synth.kv_chunk(10, 0, T, heads, hd, off)
    nv.kv_quant_append(cache, dev_bf16(k[:100].copy()), dev_bf16(v[:100].copy()), 0)
    nv.kv_quant_append(cache, dev_bf16(k), dev_bf16(v), 1)
    ref1 = oracle.kv_append(k, v)
    torch.cuda.synchronize()
    assert device_status(clear=True) == nv.OK
    sentinel = 0x7F7F
    ko = torch.full((T + 99, heads, hd), 0, dtype=torch.int16, device="cuda").fill_(sentinel).view(torch.bfloat16)
    vo = torch.full((T + 99, heads, hd), 0, dtype=torch.int16, device="cuda").fill_(sentinel).view(torch.bfloat16)
    nv.kv_dequant_window_tokens(cache, [1, 0], [T, 99], ko, vo)  # slot 0 holds 100, not 99
    assert device_status(clear=True) == nv.ERR_SHAPE
    kh, vh = host_bits(ko), host_bits(vo)
    rk, rv = oracle.kv_dequant_chunk(ref1)
    assert np.array_equal(kh[:T], rk) and np.array_equal(vh[:T], rv)
    assert np.all(kh[T:] == sentinel) and np.all(vh[T:] == sentinel)
    # the full-chunk window reports a partial slot the same way
    k2 = torch.empty((T, heads, hd), dtype=torch.bfloat16, device="cuda")
    nv.kv_dequant_window(cache, [0], k2, torch.empty_like(k2))
    assert device_status(clear=True) == nv.ERR_SHAPE
    assert device_status() == nv.OK
