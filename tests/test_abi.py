"""The C-ABI library: it loads, exports every entry point that include/nvfp4.h
declares, and rejects bad arguments on the host before touching a device.  CPU only
(no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

import nvfp4_w4a4_quantized_amax_b200 as nv

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvfp4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for n in ["nvfp4_quantize", "nvfp4_dequantize", "nvfp4_gemm", "kv_quant_append",
              "kv_dequant_window"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = nv.library()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(declared_functions()) == sorted(nv.EXPORTS)


def test_version_and_status_strings():
    lib = nv.library()
    assert lib.nvfp4_version() >> 16 == 1
    assert nv.status_string(nv.OK) == "ok"
    assert "non-finite" in nv.status_string(nv.ERR_NONFINITE)


def test_scale_sizes():
    assert nv.scales_bytes(128, 512, nv.SF_ROWMAJOR) == 128 * 32
    assert nv.scales_bytes(130, 48, nv.SF_MMA) == 256 * 4
    assert nv.scales_bytes(8192, 3072, nv.SF_MMA) == 8192 * 192
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.scales_bytes(4, 24, nv.SF_MMA)
    assert e.value.status == nv.ERR_SHAPE


def test_kv_cache_geometry_matches_storage_claim():
    heads, dh, T, chunks = 24, 128, 8192, 16
    nbytes = nv.kv_cache_bytes(heads, dh, T, chunks)
    pairs = heads * dh * T * chunks
    codes_and_scales = 2 * (pairs // 2 + pairs // 16)
    assert codes_and_scales / pairs == 1.125
    assert nbytes >= codes_and_scales
    # the per-chunk mean, scales and scratch add well under 1% on top
    assert nbytes < codes_and_scales * 1.01
    with pytest.raises(nv.Nvfp4Error):
        nv.kv_cache_bytes(24, 120, 8192, 16)  # head_dim % 16


def _fake_tensor(rows, cols, layout=nv.SF_MMA, ptr=4096):
    return nv.nvfp4_tensor(ptr, ptr, ptr, rows, cols, ((cols // 2 + 15) // 16) * 16,
                           cols // 16 if layout == nv.SF_ROWMAJOR else 0, layout, 0)


def test_host_argument_checks_return_before_any_device_work():
    lib = nv.library()
    t = _fake_tensor(16, 64)
    # NULL input
    assert lib.nvfp4_quantize(None, nv.BF16, 16, 64, 64, None, ctypes.byref(t), ctypes.c_void_p(4096),
                              None) == nv.ERR_INVALID_ARG
    # cols not a multiple of 16
    bad = _fake_tensor(16, 64)
    bad.cols = 40
    assert lib.nvfp4_quantize(ctypes.c_void_p(4096), nv.BF16, 16, 40, 40, None, ctypes.byref(bad),
                              ctypes.c_void_p(4096), None) == nv.ERR_SHAPE
    # misaligned input pointer
    assert lib.nvfp4_quantize(ctypes.c_void_p(4098), nv.BF16, 16, 64, 64, None, ctypes.byref(t),
                              ctypes.c_void_p(4096), None) == nv.ERR_ALIGNMENT
    # two-pass mode needs amax_out
    assert lib.nvfp4_quantize(ctypes.c_void_p(4096), nv.BF16, 16, 64, 64, None, ctypes.byref(t), None,
                              None) == nv.ERR_INVALID_ARG
    # GEMM needs the tensor-core scale layout and matching K
    a = _fake_tensor(16, 64, nv.SF_ROWMAJOR)
    w = _fake_tensor(32, 64)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(w), ctypes.c_void_p(4096), nv.FP32, 32, None,
                          None) == nv.ERR_INVALID_ARG
    a = _fake_tensor(16, 64)
    w = _fake_tensor(32, 128)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(w), ctypes.c_void_p(4096), nv.FP32, 32, None,
                          None) == nv.ERR_SHAPE
    # KV cache init: misaligned memory, too small
    h = nv.nvfp4_kv_cache()
    assert lib.nvfp4_kv_cache_init(ctypes.c_void_p(4097), 1 << 30, 2, 16, 64, 2, ctypes.byref(h)) == \
        nv.ERR_ALIGNMENT
    assert lib.nvfp4_kv_cache_init(ctypes.c_void_p(4096), 16, 2, 16, 64, 2, ctypes.byref(h)) == nv.ERR_SHAPE
    assert lib.nvfp4_kv_cache_init(ctypes.c_void_p(4096), 1 << 30, 2, 16, 64, 2, ctypes.byref(h)) == nv.OK
    # append: token count outside 1..chunk_tokens, slot out of range; window: empty list
    for bad_tokens in (0, 65, -1):
        assert lib.kv_quant_append(ctypes.byref(h), ctypes.c_void_p(4096), ctypes.c_void_p(4096), bad_tokens,
                                   0, None) == nv.ERR_SHAPE
    assert lib.kv_quant_append(ctypes.byref(h), ctypes.c_void_p(4096), ctypes.c_void_p(4096), 64, 2,
                               None) == nv.ERR_INVALID_ARG
    slots = (ctypes.c_int32 * 1)(5)
    assert lib.kv_dequant_window(ctypes.byref(h), slots, 1, ctypes.c_void_p(4096),
                                 ctypes.c_void_p(4096), None) == nv.ERR_INVALID_ARG
    assert lib.kv_dequant_window(ctypes.byref(h), slots, 0, ctypes.c_void_p(4096),
                                 ctypes.c_void_p(4096), None) == nv.ERR_INVALID_ARG
    # token windows: missing counts, counts outside 1..chunk_tokens, bad slot, too many slots
    ok_slots = (ctypes.c_int32 * 2)(0, 1)
    W = lib.kv_dequant_window_tokens
    out = ctypes.c_void_p(4096)
    assert W(ctypes.byref(h), ok_slots, None, 2, out, out, None) == nv.ERR_INVALID_ARG
    for bad in ((0, 64), (64, 65), (-3, 1)):
        toks = (ctypes.c_int32 * 2)(*bad)
        assert W(ctypes.byref(h), ok_slots, toks, 2, out, out, None) == nv.ERR_SHAPE
    toks = (ctypes.c_int32 * 2)(64, 17)
    assert W(ctypes.byref(h), (ctypes.c_int32 * 2)(0, 2), toks, 2, out, out, None) == nv.ERR_INVALID_ARG
    many = (ctypes.c_int32 * 65)(*([0] * 65))
    assert W(ctypes.byref(h), many, many, 65, out, out, None) == nv.ERR_INVALID_ARG
    # LoRA merge: rank outside 1..4096, NULL factors, pitch below cols; empty is a no-op
    L = lib.nvfp4_lora_merge
    p = ctypes.c_void_p(4096)
    assert L(p, nv.BF16, 4, 32, 32, p, p, 0, 1.0, p, 32, None) == nv.ERR_INVALID_ARG
    assert L(p, nv.BF16, 4, 32, 32, p, p, 4097, 1.0, p, 32, None) == nv.ERR_INVALID_ARG
    assert L(p, nv.BF16, 4, 32, 32, None, p, 8, 1.0, p, 32, None) == nv.ERR_INVALID_ARG
    assert L(p, nv.BF16, 4, 32, 16, p, p, 8, 1.0, p, 32, None) == nv.ERR_SHAPE
    assert L(p, 7, 4, 32, 32, p, p, 8, 1.0, p, 32, None) == nv.ERR_INVALID_ARG
    assert L(None, nv.BF16, 0, 32, 32, None, None, 8, 1.0, None, 32, None) == nv.OK
    # amax history: NULL pointers, length outside 1..1024
    Hp = lib.nvfp4_amax_history_push
    assert Hp(None, 4, p, p, None) == nv.ERR_INVALID_ARG
    assert Hp(p, 0, p, p, None) == nv.ERR_SHAPE
    assert Hp(p, 1025, p, p, None) == nv.ERR_SHAPE


def test_dequantize_and_gemm_epilogue_host_checks():
    """The argument rules of nvfp4_dequantize and of the GEMM epilogue, each checked on
    the host (no device is touched: every call returns before the device lookup)."""
    lib = nv.library()
    p = ctypes.c_void_p(4096)
    t = _fake_tensor(16, 64)
    D = lib.nvfp4_dequantize
    assert D(ctypes.byref(t), None, nv.BF16, 64, None) == nv.ERR_INVALID_ARG      # no output
    assert D(ctypes.byref(t), p, 7, 64, None) == nv.ERR_INVALID_ARG                # output dtype
    assert D(ctypes.byref(t), p, nv.BF16, 48, None) == nv.ERR_SHAPE                # ldy < cols
    assert D(ctypes.byref(t), ctypes.c_void_p(4100), nv.FP32, 64, None) == nv.ERR_ALIGNMENT
    assert D(ctypes.byref(t), p, nv.BF16, 68, None) == nv.ERR_ALIGNMENT           # row pitch 136 B

    G = lib.nvfp4_gemm
    a = _fake_tensor(64, 64)
    w = _fake_tensor(128, 64)
    w40 = _fake_tensor(40, 64)
    ok = lambda ep, c=p, ct=nv.FP32, ldc=128, W=w: G(ctypes.byref(a), ctypes.byref(W), c, ct, ldc,  # noqa: E731
                                                     None if ep is None else ctypes.byref(ep), None)
    assert ok(None, W=w40, ldc=40) == nv.ERR_SHAPE                  # N % 16 != 0
    assert ok(None, ldc=120) == nv.ERR_SHAPE                         # ldc < N
    assert ok(None, c=ctypes.c_void_p(4104)) == nv.ERR_ALIGNMENT     # C not 16-byte aligned
    assert ok(None, ct=9) == nv.ERR_INVALID_ARG                      # C dtype
    assert ok(None, c=None) == nv.ERR_INVALID_ARG                    # no output at all
    ep = nv.nvfp4_epilogue(5, 0, None, None, None, None)
    assert ok(ep) == nv.ERR_INVALID_ARG                              # unknown activation
    ep = nv.nvfp4_epilogue(nv.ACT_GELU_TANH, 1, None, None, None, None)
    assert ok(ep) == nv.ERR_INVALID_ARG                              # reserved field set
    q = _fake_tensor(64, 128)
    ep = nv.nvfp4_epilogue(nv.ACT_GELU_TANH, 0, ctypes.pointer(q), None, None, None)
    assert ok(ep, c=None) == nv.ERR_INVALID_ARG                      # q_out without its scale
    qr = _fake_tensor(64, 128, nv.SF_ROWMAJOR)
    ep = nv.nvfp4_epilogue(nv.ACT_GELU_TANH, 0, ctypes.pointer(qr), p, None, None)
    assert ok(ep, c=None) == nv.ERR_INVALID_ARG                      # q_out must use the MMA layout
    q_small = _fake_tensor(32, 128)
    ep = nv.nvfp4_epilogue(nv.ACT_GELU_TANH, 0, ctypes.pointer(q_small), p, None, None)
    assert ok(ep, c=None) == nv.ERR_SHAPE                            # q_out is not [M, N]
    w48 = _fake_tensor(48, 64)
    q48 = _fake_tensor(64, 48)
    ep = nv.nvfp4_epilogue(nv.ACT_GELU_TANH, 0, ctypes.pointer(q48), p, None, None)
    assert ok(ep, c=None, W=w48, ldc=48) == nv.ERR_SHAPE             # requantization needs N % 64 == 0
    ep = nv.nvfp4_epilogue(nv.ACT_GELU_TANH, 0, None, None, None, ctypes.c_void_p(4098))
    assert ok(ep, c=None) == nv.ERR_ALIGNMENT                        # h_out not 16-byte aligned


def test_noalloc_cache_may_end_at_the_scratch_region():
    """A cache laid out without the append scratch: accepted by the no-alloc append
    (which then fails later, here on a misaligned K, i.e. after the cache check) and
    refused by kv_quant_append, which needs that scratch.  Host checks only."""
    lib = nv.library()
    h = nv.nvfp4_kv_cache()
    full = ctypes.c_size_t()
    assert lib.nvfp4_kv_cache_bytes(2, 16, 64, 2, ctypes.byref(full)) == nv.OK
    assert lib.nvfp4_kv_cache_init(ctypes.c_void_p(4096), full.value, 2, 16, 64, 2, ctypes.byref(h)) == nv.OK
    short = h.off_scratch
    assert 0 < short < full.value
    assert lib.nvfp4_kv_cache_init(ctypes.c_void_p(4096), short - 1, 2, 16, 64, 2, ctypes.byref(h)) == nv.ERR_SHAPE
    assert lib.nvfp4_kv_cache_init(ctypes.c_void_p(4096), short, 2, 16, 64, 2, ctypes.byref(h)) == nv.OK
    k = ctypes.c_void_p(4097)
    assert lib.kv_quant_append(ctypes.byref(h), k, k, 64, 0, None) == nv.ERR_INVALID_ARG
    assert lib.kv_quant_append_noalloc(ctypes.byref(h), k, k, 64, 0, None) == nv.ERR_ALIGNMENT


def test_attention_side_host_checks():
    """kv_window_scores / kv_window_context: head_dim, window, pitch, alignment and size
    rules, each rejected on the host before the device lookup."""
    lib = nv.library()
    h = nv.nvfp4_kv_cache()
    nbytes = ctypes.c_size_t()
    assert lib.nvfp4_kv_cache_bytes(2, 128, 64, 2, ctypes.byref(nbytes)) == nv.OK
    assert lib.nvfp4_kv_cache_init(ctypes.c_void_p(4096), nbytes.value, 2, 128, 64, 2, ctypes.byref(h)) == nv.OK
    slots = (ctypes.c_int32 * 2)(0, 1)
    toks = (ctypes.c_int32 * 2)(64, 30)                 # Tk = 94
    p = ctypes.c_void_p(1 << 20)
    S = lib.kv_window_scores
    sc = ctypes.c_float(0.125)
    ok_s = lambda tq=16, ldq=256, ld_s=96, out=p, st=nv.FP32, q=p, n=2, t=toks: S(  # noqa: E731
        ctypes.byref(h), slots, t, n, q, tq, ldq, sc, out, st, ld_s, None)
    assert ok_s(ld_s=92) == nv.ERR_SHAPE                           # ld_s < Tk
    assert ok_s(ldq=200) == nv.ERR_SHAPE                           # ldq < heads * 128
    assert ok_s(ld_s=98) == nv.ERR_ALIGNMENT                       # score rows not 16-byte multiples
    assert ok_s(out=ctypes.c_void_p((1 << 20) + 4)) == nv.ERR_ALIGNMENT
    assert ok_s(st=7) == nv.ERR_INVALID_ARG                        # output dtype
    assert ok_s(n=0) == nv.ERR_INVALID_ARG                         # empty window
    assert ok_s(t=(ctypes.c_int32 * 2)(64, 65)) == nv.ERR_SHAPE    # more tokens than a chunk holds
    C = lib.kv_window_context
    ok_c = lambda tq=16, ld_p=96, ldo=256, out=p, ot=nv.FP32: C(  # noqa: E731
        ctypes.byref(h), slots, toks, 2, p, tq, ld_p, out, ot, ldo, None)
    assert ok_c(ld_p=88) == nv.ERR_SHAPE                           # ld_p < Tk
    assert ok_c(ldo=128) == nv.ERR_SHAPE                           # ldo < heads * 128
    assert ok_c(ld_p=100) == nv.ERR_ALIGNMENT                      # weight rows not 16-byte multiples
    assert ok_c(out=ctypes.c_void_p((1 << 20) + 8)) == nv.ERR_ALIGNMENT
    assert ok_c(tq=65535 * 512 + 1) == nv.ERR_SHAPE                # more than 65535 groups of 4 query tiles
    assert ok_c(tq=-1) == nv.ERR_SHAPE
    h64 = nv.nvfp4_kv_cache()
    assert lib.nvfp4_kv_cache_bytes(2, 64, 64, 2, ctypes.byref(nbytes)) == nv.OK
    assert lib.nvfp4_kv_cache_init(ctypes.c_void_p(4096), nbytes.value, 2, 64, 64, 2, ctypes.byref(h64)) == nv.OK
    assert C(ctypes.byref(h64), slots, toks, 2, p, 16, 96, p, nv.FP32, 128, None) == nv.ERR_SHAPE  # head_dim 64


def test_binding_refuses_host_tensors_and_foreign_layouts():
    """The Python binding passes device addresses only: a host tensor, or a layout the C
    call cannot express with its row pitch, is refused before the library is called."""
    import torch

    x = torch.zeros(4, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        nv.nvfp4_amax(x, torch.zeros(1))
    with pytest.raises(ValueError, match="CUDA"):
        nv.nvfp4_lora_merge(torch.zeros(4, 32), torch.zeros(4, 2), torch.zeros(2, 32), 1.0, torch.zeros(4, 32))
    with pytest.raises(ValueError, match="contiguous rows"):
        nv.nvfp4_amax(x.t(), torch.zeros(1))
    with pytest.raises(ValueError, match="contiguous"):
        nv.nvfp4_lora_merge(torch.zeros(4, 32), torch.zeros(2, 4).t(), torch.zeros(2, 32), 1.0, torch.zeros(4, 32))
