"""ORACLE — plain CPU statement of the NVFP4 hot path.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  It shares no code with the CUDA library
(``nvfp4_w4a4_quantized_amax_b200``) and neither imports the other.

The bit-level steps (E2M1/E4M3 encoding, block and tensor scales, the exact mean
of K, the KV chunk encode and window dequant) live in ``nvfp4_oracle.c`` (plain C,
no FMA contraction, no flush-to-zero).  The GEMM reference is a float64 matrix
product of the exactly decoded operands (a library matmul used as one step).

Sources (web pages about LongLive-2.0):
  [TW §一] techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存",
           §一 — the two-level NVFP4 format (E2M1 values, FP8 scale per 16, FP32 per tensor).
  [TW §四] same page, §四 — W4A4 matmuls; mean-subtracted K in an NVFP4 KV cache.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_NONFINITE = 4


def build(force: bool = False) -> str:
    """Compile liboracle.so (plain C: -O2, no FP contraction, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            i64, vp, f32, dbl, u8 = (ctypes.c_int64, ctypes.c_void_p, ctypes.c_float,
                                     ctypes.c_double, ctypes.c_uint8)
            lib.oracle_e2m1_value.restype = dbl
            lib.oracle_e2m1_value.argtypes = [u8]
            lib.oracle_e2m1_index_exact.restype = ctypes.c_int
            lib.oracle_e2m1_index_exact.argtypes = [f32, f32]
            lib.oracle_e4m3_value.restype = dbl
            lib.oracle_e4m3_value.argtypes = [u8]
            lib.oracle_e4m3_encode.restype = u8
            lib.oracle_e4m3_encode.argtypes = [f32]
            lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
            lib.oracle_f32_to_bf16.argtypes = [f32]
            lib.oracle_quantize.restype = ctypes.c_int
            lib.oracle_quantize.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, vp, vp, vp, vp]
            lib.oracle_dequantize.argtypes = [vp, vp, f32, i64, i64, vp, vp]
            lib.oracle_decode_f64.argtypes = [vp, vp, f32, i64, i64, vp]
            lib.oracle_sf_mma_offset.restype = i64
            lib.oracle_sf_mma_offset.argtypes = [i64, i64, i64]
            lib.oracle_exact_mean_bf16.restype = f32
            lib.oracle_exact_mean_bf16.argtypes = [vp, i64, i64]
            lib.oracle_kv_append.restype = ctypes.c_int
            lib.oracle_kv_append.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp,
                                             vp, vp]
            lib.oracle_kv_dequant_chunk.argtypes = [vp, vp, vp, vp, vp, f32, f32, i64, i64, i64,
                                                    vp, vp]
            lib.oracle_gelu_tanh.restype = dbl
            lib.oracle_gelu_tanh.argtypes = [dbl]
            lib.oracle_gelu_tanh_array.argtypes = [vp, i64, vp]
            lib.oracle_amax_history_push.restype = ctypes.c_int
            lib.oracle_amax_history_push.argtypes = [vp, i64, f32, vp]
            lib.oracle_lora_merge.restype = None
            lib.oracle_lora_merge.argtypes = [vp, ctypes.c_int, i64, i64, i64, vp, vp, i64, f32, vp, i64]
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


# ------------------------------------------------------------------ scalars

def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(code)


def e2m1_index_exact(ax: float, d: float) -> int:
    return _load().oracle_e2m1_index_exact(ax, d)


def e4m3_value(b: int) -> float:
    return _load().oracle_e4m3_value(b)


def e4m3_encode(s: float) -> int:
    return _load().oracle_e4m3_encode(s)


def f32_to_bf16(f: float) -> int:
    return _load().oracle_f32_to_bf16(f)


# ------------------------------------------------------------------ tensors

class Quantized:
    """Canonical (row-major) NVFP4 tensor as produced by the oracle."""

    def __init__(self, codes, scales, g, amax, rows, cols):
        self.codes, self.scales, self.g, self.amax = codes, scales, g, amax
        self.rows, self.cols = rows, cols


def quantize(x: np.ndarray, gscale: float | None = None) -> Quantized:
    """x: uint16 (bf16 bits) or float32 array [rows, cols].  Raises on non-finite input."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    xt = 0 if x.dtype == np.uint16 else 1
    if xt == 1:
        x = x.astype(np.float32, copy=False)
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    amax = np.zeros(1, dtype=np.float32)
    gin = None if gscale is None else np.array([gscale], dtype=np.float32)
    rc = _load().oracle_quantize(_p(x), xt, rows, cols, cols, _p(gin), _p(codes), _p(scales),
                                 _p(g), _p(amax))
    if rc != OK:
        raise FloatingPointError(f"oracle_quantize status {rc}")
    return Quantized(codes, scales, float(g[0]), float(amax[0]), rows, cols)


def quantize_status(x: np.ndarray) -> int:
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    xt = 0 if x.dtype == np.uint16 else 1
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros((rows, cols // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    amax = np.zeros(1, dtype=np.float32)
    return _load().oracle_quantize(_p(x), xt, rows, cols, cols, None, _p(codes), _p(scales),
                                   _p(g), _p(amax))


def dequantize(q: Quantized):
    """(float32 values, bf16 bits) of RN(RN(e2m1 * s) * g)."""
    y = np.zeros((q.rows, q.cols), dtype=np.float32)
    yb = np.zeros((q.rows, q.cols), dtype=np.uint16)
    _load().oracle_dequantize(_p(q.codes), _p(q.scales), q.g, q.rows, q.cols, _p(y), _p(yb))
    return y, yb


def decode_f64(codes: np.ndarray, scales: np.ndarray, g: float) -> np.ndarray:
    """Exact operand values e2m1 * s * g (float64) of a canonical NVFP4 tensor."""
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    rows, half = codes.shape
    out = np.zeros((rows, 2 * half), dtype=np.float64)
    _load().oracle_decode_f64(_p(codes), _p(scales), g, rows, 2 * half, _p(out))
    return out


def gemm_ref(a_codes, a_scales, a_g, w_codes, w_scales, w_g, rows=None):
    """C_ref = A_hat W_hat^T in float64 and the bound sum_k |a_k w_k| per element.
    `rows` (optional index array) restricts the product to those rows of A."""
    if rows is not None:
        a_codes, a_scales = a_codes[rows], a_scales[rows]
    a = decode_f64(a_codes, a_scales, a_g)
    w = decode_f64(w_codes, w_scales, w_g)
    return a @ w.T, np.abs(a) @ np.abs(w).T


def sf_mma_offset(r: int, j: int, cols: int) -> int:
    return _load().oracle_sf_mma_offset(r, j, cols)


def sf_mma_bytes(rows: int, cols: int) -> int:
    return ((rows + 127) // 128) * 128 * (((cols // 16) + 3) // 4) * 4


def sf_to_mma(scales: np.ndarray, cols: int) -> np.ndarray:
    """Place canonical row-major scales [rows, cols/16] into the tensor-core layout
    (padding bytes 0), using the oracle's offset function row by row."""
    rows, nb = scales.shape
    out = np.zeros(sf_mma_bytes(rows, cols), dtype=np.uint8)
    lib = _load()
    offs = np.array([[lib.oracle_sf_mma_offset(r, j, cols) for j in range(nb)] for r in range(min(rows, 128))],
                    dtype=np.int64) if rows else np.zeros((0, nb), np.int64)
    # the offset is affine in the row tile: rows r and r + 128 differ by one atom row
    groups = ((cols // 16) + 3) // 4
    for r0 in range(0, rows, 128):
        n = min(128, rows - r0)
        out[offs[:n] + (r0 // 128) * groups * 512] = scales[r0:r0 + n]
    return out


def sf_from_mma(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Inverse of sf_to_mma (ignores padding)."""
    nb = cols // 16
    lib = _load()
    offs = np.array([[lib.oracle_sf_mma_offset(r, j, cols) for j in range(nb)] for r in range(min(rows, 128))],
                    dtype=np.int64) if rows else np.zeros((0, nb), np.int64)
    groups = ((cols // 16) + 3) // 4
    out = np.zeros((rows, nb), dtype=np.uint8)
    for r0 in range(0, rows, 128):
        n = min(128, rows - r0)
        out[r0:r0 + n] = buf[offs[:n] + (r0 // 128) * groups * 512]
    return out


def exact_mean_bf16(col: np.ndarray) -> float:
    col = np.ascontiguousarray(col, dtype=np.uint16)
    return float(_load().oracle_exact_mean_bf16(_p(col), col.size, 1))


class KVChunk:
    def __init__(self, **kw):
        self.__dict__.update(kw)


def kv_append(k: np.ndarray, v: np.ndarray) -> KVChunk:
    """k, v: uint16 (bf16 bits) [T, H, Dh]."""
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    T, H, Dh = k.shape
    mu = np.zeros(H * Dh, dtype=np.float32)
    gk = np.zeros(1, np.float32)
    gv = np.zeros(1, np.float32)
    ak = np.zeros(1, np.float32)
    av = np.zeros(1, np.float32)
    kc = np.zeros((T, H, Dh // 2), np.uint8)
    ks = np.zeros((T, H, Dh // 16), np.uint8)
    vc = np.zeros((T, H, Dh // 2), np.uint8)
    vs = np.zeros((T, H, Dh // 16), np.uint8)
    rc = _load().oracle_kv_append(_p(k), _p(v), T, H, Dh, _p(mu), _p(gk), _p(gv), _p(kc), _p(ks),
                                  _p(vc), _p(vs), _p(ak), _p(av))
    if rc != OK:
        raise FloatingPointError(f"oracle_kv_append status {rc}")
    return KVChunk(mu=mu, g_k=float(gk[0]), g_v=float(gv[0]), k_codes=kc, k_scales=ks,
                   v_codes=vc, v_scales=vs, amax_k=float(ak[0]), amax_v=float(av[0]),
                   T=T, H=H, Dh=Dh)


def kv_dequant_chunk(ch: KVChunk):
    """(K^, V^) bf16 bits [T, H, Dh] of one appended chunk."""
    ko = np.zeros((ch.T, ch.H, ch.Dh), np.uint16)
    vo = np.zeros((ch.T, ch.H, ch.Dh), np.uint16)
    _load().oracle_kv_dequant_chunk(_p(ch.k_codes), _p(ch.k_scales), _p(ch.v_codes),
                                    _p(ch.v_scales), _p(ch.mu), ch.g_k, ch.g_v, ch.T, ch.H, ch.Dh,
                                    _p(ko), _p(vo))
    return ko, vo


def gelu_tanh(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.float32)
    out = np.zeros(c.shape, dtype=np.float64)
    _load().oracle_gelu_tanh_array(_p(c), c.size, _p(out))
    return out


def lora_merge(w: np.ndarray, b: np.ndarray, a: np.ndarray, scale: float) -> np.ndarray:
    """W' = W + scale * (B A) in binary32 with the oracle's fixed order (see
    oracle_lora_merge).  w: uint16 (bf16 bits) or float32 [rows, cols];
    b: float32 [rows, rank]; a: float32 [rank, cols].  Returns float32 [rows, cols]."""
    w = np.ascontiguousarray(w)
    wt = 0 if w.dtype == np.uint16 else 1
    if wt == 1:
        w = w.astype(np.float32, copy=False)
    b = np.ascontiguousarray(b, dtype=np.float32)
    a = np.ascontiguousarray(a, dtype=np.float32)
    rows, cols = w.shape
    rank = b.shape[1]
    assert b.shape == (rows, rank) and a.shape == (rank, cols)
    out = np.zeros((rows, cols), np.float32)
    _load().oracle_lora_merge(_p(w), wt, rows, cols, cols, _p(b), _p(a), rank, float(np.float32(scale)), _p(out),
                              cols)
    return out


def amax_history_push(history: np.ndarray, amax_new: float):
    """(updated history, g) after pushing amax_new (see oracle_amax_history_push);
    raises on a non-finite amax_new."""
    h = np.ascontiguousarray(history, dtype=np.float32).copy()
    g = np.zeros(1, np.float32)
    st = _load().oracle_amax_history_push(_p(h), h.size, float(np.float32(amax_new)), _p(g))
    if st != 0:
        raise ValueError("non-finite amax")
    return h, float(g[0])
