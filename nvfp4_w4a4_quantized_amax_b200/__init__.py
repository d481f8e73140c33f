"""Python binding of libnvfp4 (C ABI in include/nvfp4.h).

Argument marshalling only: torch tensors provide device memory and streams, and
every step runs in the CUDA library.  The functions keep the C names:
``nvfp4_quantize``, ``nvfp4_dequantize``, ``nvfp4_gemm``, ``kv_quant_append``,
``kv_dequant_window`` (plus the cache and status helpers).  A missing library is
an ImportError: there is no fallback implementation.

NVFP4 buffers are raw bytes (uint8) plus one float32 tensor scale; they are never
cast to another dtype (news.ainew.jp copy of the LongLive 2.0 README, "Quick
Start / NVFP4": a dtype cast of the pipeline would corrupt the quantized buffers).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGNMENT, ERR_NONFINITE, ERR_TIMEOUT, ERR_CUDA, \
    ERR_UNSUPPORTED_DEVICE = range(8)
BF16, FP32 = 0, 1
SF_ROWMAJOR, SF_MMA = 0, 1
ACT_NONE, ACT_GELU_TANH = 0, 1

_lock = threading.Lock()
_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == ERR_CUDA:
            detail = ": " + library().nvfp4_last_cuda_error_string().decode()
        super().__init__(f"{where}: {status_string(status)} (status {status}){detail}")


class nvfp4_tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("gscale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("ld_codes", ctypes.c_int64),
                ("ld_scales", ctypes.c_int64), ("sf_layout", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class nvfp4_epilogue(ctypes.Structure):
    _fields_ = [("act", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("q_out", ctypes.POINTER(nvfp4_tensor)), ("q_gscale_in", ctypes.c_void_p),
                ("q_amax_out", ctypes.c_void_p), ("h_out", ctypes.c_void_p)]


class nvfp4_kv_cache(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("bytes", ctypes.c_size_t), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("chunk_tokens", ctypes.c_int64),
                ("max_chunks", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("off_k_codes", ctypes.c_int64), ("off_v_codes", ctypes.c_int64),
                ("off_k_scales", ctypes.c_int64), ("off_v_scales", ctypes.c_int64),
                ("off_mu", ctypes.c_int64), ("off_gscale", ctypes.c_int64),
                ("off_tokens", ctypes.c_int64), ("off_scratch", ctypes.c_int64),
                ("slot_codes_bytes", ctypes.c_int64),
                ("slot_scales_bytes", ctypes.c_int64)]


EXPORTS = ["nvfp4_version", "nvfp4_status_string", "nvfp4_scales_bytes", "nvfp4_quantize", "nvfp4_amax",
           "nvfp4_dequantize", "nvfp4_gemm", "nvfp4_kv_cache_bytes", "nvfp4_kv_cache_init",
           "kv_quant_append", "kv_quant_append_noalloc", "kv_dequant_window", "kv_dequant_window_tokens",
           "kv_window_scores", "kv_window_context",
           "nvfp4_lora_merge", "nvfp4_amax_history_push", "nvfp4_last_cuda_error_string",
           "nvfp4_debug_gemm_fault", "nvfp4_debug_grid_barrier",
           "nvfp4_get_device_status"]


def library():
    """Load libnvfp4.so (raises ImportError when it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"libnvfp4.so not built ({LIB_PATH}); run "
                                  "python -m nvfp4_w4a4_quantized_amax_b200.build")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
            T = ctypes.POINTER(nvfp4_tensor)
            KV = ctypes.POINTER(nvfp4_kv_cache)
            lib.nvfp4_version.restype = i32
            lib.nvfp4_status_string.restype = ctypes.c_char_p
            lib.nvfp4_status_string.argtypes = [i32]
            lib.nvfp4_debug_grid_barrier.restype = i32
            lib.nvfp4_debug_grid_barrier.argtypes = [ctypes.c_uint32, ctypes.c_uint64]
            lib.nvfp4_debug_gemm_fault.restype = i32
            lib.nvfp4_debug_gemm_fault.argtypes = [i32, ctypes.c_uint64]
            lib.nvfp4_last_cuda_error_string.restype = ctypes.c_char_p
            lib.nvfp4_last_cuda_error_string.argtypes = []
            lib.nvfp4_scales_bytes.restype = i32
            lib.nvfp4_scales_bytes.argtypes = [i64, i64, i32, ctypes.POINTER(ctypes.c_size_t)]
            lib.nvfp4_quantize.restype = i32
            lib.nvfp4_quantize.argtypes = [vp, i32, i64, i64, i64, vp, T, vp, vp]
            lib.nvfp4_amax.restype = i32
            lib.nvfp4_amax.argtypes = [vp, i32, i64, i64, i64, vp, vp]
            lib.nvfp4_dequantize.restype = i32
            lib.nvfp4_dequantize.argtypes = [T, vp, i32, i64, vp]
            lib.nvfp4_gemm.restype = i32
            lib.nvfp4_gemm.argtypes = [T, T, vp, i32, i64, ctypes.POINTER(nvfp4_epilogue), vp]
            lib.nvfp4_kv_cache_bytes.restype = i32
            lib.nvfp4_kv_cache_bytes.argtypes = [i32, i32, i64, i32, ctypes.POINTER(ctypes.c_size_t)]
            lib.nvfp4_kv_cache_init.restype = i32
            lib.nvfp4_kv_cache_init.argtypes = [vp, ctypes.c_size_t, i32, i32, i64, i32, KV]
            lib.kv_quant_append.restype = i32
            lib.kv_quant_append.argtypes = [KV, vp, vp, i64, i32, vp]
            lib.kv_quant_append_noalloc.restype = i32
            lib.kv_quant_append_noalloc.argtypes = [KV, vp, vp, i64, i32, vp]
            lib.kv_dequant_window.restype = i32
            lib.kv_dequant_window.argtypes = [KV, ctypes.POINTER(ctypes.c_int32), i32, vp, vp, vp]
            lib.kv_dequant_window_tokens.restype = i32
            lib.kv_dequant_window_tokens.argtypes = [KV, ctypes.POINTER(ctypes.c_int32),
                                                     ctypes.POINTER(ctypes.c_int32), i32, vp, vp, vp]
            lib.kv_window_scores.restype = i32
            lib.kv_window_scores.argtypes = [KV, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32), i32,
                                             vp, i64, i64, ctypes.c_float, vp, i32, i64, vp]
            lib.kv_window_context.restype = i32
            lib.kv_window_context.argtypes = [KV, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32), i32,
                                              vp, i64, i64, vp, i32, i64, vp]
            lib.nvfp4_lora_merge.restype = i32
            lib.nvfp4_lora_merge.argtypes = [vp, i32, i64, i64, i64, vp, vp, i32, ctypes.c_float, vp, i64, vp]
            lib.nvfp4_amax_history_push.restype = i32
            lib.nvfp4_amax_history_push.argtypes = [vp, i32, vp, vp, vp]
            lib.nvfp4_get_device_status.restype = i32
            lib.nvfp4_get_device_status.argtypes = [i32, ctypes.POINTER(ctypes.c_int32), i32]
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().nvfp4_status_string(status).decode()


def _check(status: int, where: str):
    if status != OK:
        raise Nvfp4Error(status, where)


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t) -> Optional[ctypes.c_void_p]:
    """Device address of a CUDA tensor (None stays NULL).  A host tensor is refused here:
    its address would reach a kernel."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"a CUDA tensor is required, got one on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


def _rows(t, name: str):
    """t is [rows, cols] with unit stride along the row (the C calls take a row pitch);
    an empty tensor's strides mean nothing and pass."""
    if t.dim() != 2 or (t.numel() > 0 and t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name}: a 2-D tensor with contiguous rows is required")


def _dense(t, name: str):
    if t.numel() > 0 and not t.is_contiguous():
        raise ValueError(f"{name}: a contiguous tensor is required")


def _bf16(t, name: str):
    import torch

    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name}: bf16 is required, got {t.dtype}")


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def scales_bytes(rows: int, cols: int, sf_layout: int) -> int:
    n = ctypes.c_size_t()
    _check(library().nvfp4_scales_bytes(rows, cols, sf_layout, ctypes.byref(n)), "nvfp4_scales_bytes")
    return n.value


class NVFP4Tensor:
    """Device buffers of one NVFP4 tensor [rows, cols]: codes (uint8 [rows, ld_codes]),
    scales (uint8, row-major or tensor-core layout) and the FP32 tensor scale."""

    def __init__(self, rows: int, cols: int, sf_layout: int = SF_MMA, device=None,
                 codes=None, scales=None, gscale=None):
        import torch

        device = device or torch.device("cuda")
        self.rows, self.cols, self.sf_layout = rows, cols, sf_layout
        self.ld_codes = ((cols // 2 + 15) // 16) * 16
        self.ld_scales = cols // 16 if sf_layout == SF_ROWMAJOR else 0
        self.codes = codes if codes is not None else torch.empty(
            (rows, self.ld_codes), dtype=torch.uint8, device=device)
        self.scales = scales if scales is not None else torch.empty(
            scales_bytes(rows, cols, sf_layout), dtype=torch.uint8, device=device)
        self.gscale = gscale if gscale is not None else torch.zeros(1, dtype=torch.float32,
                                                                     device=device)
        self._c = nvfp4_tensor(self.codes.data_ptr(), self.scales.data_ptr(), self.gscale.data_ptr(),
                               rows, cols, self.ld_codes, self.ld_scales, sf_layout, 0)

    @property
    def c(self) -> nvfp4_tensor:
        return self._c


def nvfp4_quantize(x, out: NVFP4Tensor, gscale_in=None, amax_out=None, stream=None):
    """Quantize x [rows, cols] (bf16 or fp32, CUDA) into `out`."""
    _rows(x, "x")
    rows, cols = x.shape
    _check(library().nvfp4_quantize(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), _ptr(gscale_in),
                                    ctypes.byref(out.c), _ptr(amax_out), _stream(stream)),
           "nvfp4_quantize")


def nvfp4_amax(x, amax_out, stream=None):
    """max|x| of x [rows, cols] (bf16 or fp32, CUDA) into amax_out (fp32 [1], CUDA)."""
    _rows(x, "x")
    rows, cols = x.shape
    _check(library().nvfp4_amax(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), _ptr(amax_out),
                                _stream(stream)), "nvfp4_amax")


def nvfp4_dequantize(t: NVFP4Tensor, y, stream=None):
    _rows(y, "y")
    _check(library().nvfp4_dequantize(ctypes.byref(t.c), _ptr(y), _dtype_code(y), y.stride(0),
                                      _stream(stream)), "nvfp4_dequantize")


def nvfp4_gemm(a: NVFP4Tensor, w: NVFP4Tensor, c=None, act: int = ACT_NONE,
               q_out: Optional[NVFP4Tensor] = None, q_gscale_in=None, q_amax_out=None, h_out=None,
               stream=None):
    """C = A W^T (+ optional GELU and fused NVFP4 requantization into q_out)."""
    ep = None
    if act != ACT_NONE or q_out is not None or q_amax_out is not None or h_out is not None:
        ep = nvfp4_epilogue(act, 0, ctypes.pointer(q_out.c) if q_out is not None else None,
                            _ptr(q_gscale_in), _ptr(q_amax_out), _ptr(h_out))
    if c is not None:
        _rows(c, "c")
    ct = _dtype_code(c) if c is not None else FP32
    ldc = c.stride(0) if c is not None else 0
    _check(library().nvfp4_gemm(ctypes.byref(a.c), ctypes.byref(w.c), _ptr(c), ct, ldc,
                                ctypes.byref(ep) if ep is not None else None, _stream(stream)),
           "nvfp4_gemm")


def kv_cache_bytes(heads: int, head_dim: int, chunk_tokens: int, max_chunks: int) -> int:
    n = ctypes.c_size_t()
    _check(library().nvfp4_kv_cache_bytes(heads, head_dim, chunk_tokens, max_chunks, ctypes.byref(n)),
           "nvfp4_kv_cache_bytes")
    return n.value


class KVCache:
    """An NVFP4 KV cache laid out by the library in one device allocation."""

    def __init__(self, heads: int, head_dim: int, chunk_tokens: int, max_chunks: int, device=None,
                 buffer=None):
        import torch

        device = device or torch.device("cuda")
        nbytes = kv_cache_bytes(heads, head_dim, chunk_tokens, max_chunks)
        self.buffer = buffer if buffer is not None else torch.empty(nbytes, dtype=torch.uint8,
                                                                    device=device)
        self.handle = nvfp4_kv_cache()
        _check(library().nvfp4_kv_cache_init(self.buffer.data_ptr(), self.buffer.numel(), heads,
                                             head_dim, chunk_tokens, max_chunks,
                                             ctypes.byref(self.handle)), "nvfp4_kv_cache_init")
        self.heads, self.head_dim, self.chunk_tokens, self.max_chunks = (heads, head_dim,
                                                                         chunk_tokens, max_chunks)

    def _view(self, off: int, nbytes: int):
        return self.buffer[off:off + nbytes]

    def slot_views(self, slot: int):
        """(k_codes, k_scales, v_codes, v_scales, mu (float32), gscale (float32 [2])) of a slot."""
        import torch

        h = self.handle
        c = self.heads * self.head_dim
        kc = self._view(h.off_k_codes + slot * h.slot_codes_bytes, h.slot_codes_bytes)
        vc = self._view(h.off_v_codes + slot * h.slot_codes_bytes, h.slot_codes_bytes)
        ks = self._view(h.off_k_scales + slot * h.slot_scales_bytes, h.slot_scales_bytes)
        vs = self._view(h.off_v_scales + slot * h.slot_scales_bytes, h.slot_scales_bytes)
        mu = self._view(h.off_mu + slot * c * 4, c * 4).view(torch.float32)
        g = self._view(h.off_gscale + slot * 8, 8).view(torch.float32)
        return kc, ks, vc, vs, mu, g

    def slot_tokens(self, slot: int) -> int:
        """Tokens recorded for `slot` by its last append (reads the device)."""
        import torch

        return int(self._view(self.handle.off_tokens + slot * 4, 4).view(torch.int32).item())


def kv_quant_append(cache: KVCache, k, v, slot: int, stream=None):
    """Quantize one chunk (bf16 [tokens, heads, head_dim], 1 <= tokens <= chunk_tokens)
    of K and V into `slot`."""
    _dense(k, "k")
    _dense(v, "v")
    _check(library().kv_quant_append(ctypes.byref(cache.handle), _ptr(k), _ptr(v), k.shape[0], slot,
                                     _stream(stream)), "kv_quant_append")


def kv_quant_append_noalloc(cache: KVCache, k, v, slot: int, stream=None):
    """kv_quant_append without any caller-provided scratch: the library's static
    per-device array holds the column statistics (heads * head_dim <= 4096).
    For callers that may not allocate device memory; calls racing on the GPU
    share that array, so issue them on one stream."""
    _dense(k, "k")
    _dense(v, "v")
    _check(library().kv_quant_append_noalloc(ctypes.byref(cache.handle), _ptr(k), _ptr(v), k.shape[0],
                                             slot, _stream(stream)), "kv_quant_append_noalloc")


def kv_dequant_window(cache: KVCache, slots: Sequence[int], k_out, v_out, stream=None):
    _dense(k_out, "k_out")
    _dense(v_out, "v_out")
    arr = (ctypes.c_int32 * len(slots))(*slots)
    _check(library().kv_dequant_window(ctypes.byref(cache.handle), arr, len(slots), _ptr(k_out),
                                       _ptr(v_out), _stream(stream)), "kv_dequant_window")


def kv_dequant_window_tokens(cache: KVCache, slots: Sequence[int], tokens: Sequence[int], k_out, v_out,
                             stream=None):
    """Window over slots holding tokens[i] tokens each; output rows sum(tokens), in list order."""
    if len(tokens) != len(slots):
        raise ValueError("one token count per slot")
    _dense(k_out, "k_out")
    _dense(v_out, "v_out")
    sarr = (ctypes.c_int32 * len(slots))(*slots)
    tarr = (ctypes.c_int32 * len(tokens))(*tokens)
    _check(library().kv_dequant_window_tokens(ctypes.byref(cache.handle), sarr, tarr, len(slots), _ptr(k_out),
                                              _ptr(v_out), _stream(stream)), "kv_dequant_window_tokens")


def kv_window_scores(cache: KVCache, slots: Sequence[int], tokens: Sequence[int], q, scale: float, s_out,
                     stream=None):
    """Scores of q (bf16 [tq, heads, head_dim]) against the window's keys, K read
    from the NVFP4 cache inside the kernel; s_out (fp32 or bf16 [heads, tq, >= Tk])."""
    if len(tokens) != len(slots):
        raise ValueError("one token count per slot")
    _bf16(q, "q")
    if q.dim() != 3 or q.shape[1] != cache.heads or (q.numel() > 0 and (q.stride(2) != 1 or q.stride(1) != q.shape[2])):
        raise ValueError("q: [tq, heads, head_dim] with contiguous heads and dims is required")
    tq = q.shape[0]
    if s_out.dim() != 3 or s_out.shape[0] != cache.heads or s_out.shape[1] != tq or (
            s_out.numel() > 0 and (s_out.stride(2) != 1 or s_out.stride(0) != tq * s_out.stride(1))):
        raise ValueError("s_out: [heads, tq, ld_s] with rows ld_s apart and heads tq * ld_s apart is required")
    sarr = (ctypes.c_int32 * len(slots))(*slots)
    tarr = (ctypes.c_int32 * len(tokens))(*tokens)
    _check(library().kv_window_scores(ctypes.byref(cache.handle), sarr, tarr, len(slots), _ptr(q), tq,
                                      q.stride(0), float(scale), _ptr(s_out), _dtype_code(s_out),
                                      s_out.stride(1), _stream(stream)), "kv_window_scores")


def kv_window_context(cache: KVCache, slots: Sequence[int], tokens: Sequence[int], p, o_out, stream=None):
    """O = P V^ over the window's keys, V read from the NVFP4 cache inside the kernel:
    p bf16 [heads, tq, >= Tk]; o_out (fp32 or bf16) [tq, heads, head_dim]."""
    if len(tokens) != len(slots):
        raise ValueError("one token count per slot")
    _bf16(p, "p")
    if p.dim() != 3 or p.shape[0] != cache.heads or (
            p.numel() > 0 and (p.stride(2) != 1 or p.stride(0) != p.shape[1] * p.stride(1))):
        raise ValueError("p: [heads, tq, ld_p] with rows ld_p apart and heads tq * ld_p apart is required")
    if o_out.dim() != 3 or o_out.shape[0] != p.shape[1] or o_out.shape[1] != cache.heads or (
            o_out.numel() > 0 and (o_out.stride(2) != 1 or o_out.stride(1) != o_out.shape[2])):
        raise ValueError("o_out: [tq, heads, head_dim] with contiguous heads and dims is required")
    sarr = (ctypes.c_int32 * len(slots))(*slots)
    tarr = (ctypes.c_int32 * len(tokens))(*tokens)
    _check(library().kv_window_context(ctypes.byref(cache.handle), sarr, tarr, len(slots), _ptr(p), p.shape[1],
                                       p.stride(1), _ptr(o_out), _dtype_code(o_out), o_out.stride(0),
                                       _stream(stream)), "kv_window_context")


def nvfp4_lora_merge(w, lora_b, lora_a, scale: float, out, stream=None):
    """out = W + scale * (B A) in binary32 with the library's fixed order (LoRA merged
    before quantization).  w: bf16 or fp32 [rows, cols]; lora_b fp32 [rows, rank];
    lora_a fp32 [rank, cols]; out fp32 [rows, cols]."""
    _rows(w, "w")
    _rows(out, "out")
    _dense(lora_b, "lora_b")
    _dense(lora_a, "lora_a")
    rows, cols = w.shape
    rank = lora_b.shape[1]
    _check(library().nvfp4_lora_merge(_ptr(w), _dtype_code(w), rows, cols, w.stride(0), _ptr(lora_b),
                                      _ptr(lora_a), rank, float(scale), _ptr(out), out.stride(0),
                                      _stream(stream)), "nvfp4_lora_merge")


def nvfp4_amax_history_push(history, amax_new, gscale_out, stream=None):
    """Shift amax_new (device fp32 [1]) into history (device fp32 [len]) and write the
    next supplied tensor scale RN(max(history) / 2688) to gscale_out."""
    _check(library().nvfp4_amax_history_push(_ptr(history), history.numel(), _ptr(amax_new), _ptr(gscale_out),
                                             _stream(stream)), "nvfp4_amax_history_push")


def debug_gemm_fault(drop_first_stage: bool, wait_limit_ns: int = 0):
    """Test hook of the GEMM's bounded waits (see nvfp4_debug_gemm_fault)."""
    _check(library().nvfp4_debug_gemm_fault(1 if drop_first_stage else 0, wait_limit_ns), "nvfp4_debug_gemm_fault")


def debug_grid_barrier(extra_arrivals: int, wait_limit_ns: int = 0):
    """Test hook of the one-launch quantization's grid barrier (see nvfp4_debug_grid_barrier)."""
    _check(library().nvfp4_debug_grid_barrier(extra_arrivals, wait_limit_ns), "nvfp4_debug_grid_barrier")


def get_device_status(device: int = 0, clear: bool = False) -> int:
    v = ctypes.c_int32()
    _check(library().nvfp4_get_device_status(device, ctypes.byref(v), 1 if clear else 0),
           "nvfp4_get_device_status")
    return v.value
