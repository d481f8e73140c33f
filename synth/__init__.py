"""Seeded synthetic inputs for the NVFP4 hot path (tests, smoke check, benchmark).

The arrays are produced by ``synth.c`` (splitmix64 counter generator, Box-Muller
normals, Student-t with 3 degrees of freedom) and returned as numpy arrays; bf16
tensors are returned as ``uint16`` bit patterns.  Nothing here performs any NVFP4
arithmetic.

Workload recipes (shapes follow one 8-frame chunk of a 5B video DiT block):
  * ``tiny_linear``   A [128, 512] ~ N(0,1) with 4 picked columns x20,
                      W [256, 512] ~ N(0, 0.02), seed 0.
  * ``activations``   X [rows, cols] = 0.5 * t3, with ceil(1% of cols) picked
                      columns x30 (seed 1 for the 32768 x 3072 pass, 2 for the
                      GEMM block, 4 for the fused FFN).
  * ``weights``       W [N, K] ~ N(0, 0.02).
  * ``kv``            per (head, dim) K offset ~ N(0, 3) drawn once; per chunk
                      K = N(0,1) + offset, V = N(0,1); 24 heads x 128, 8192 tokens.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_SRC = os.path.join(_HERE, "synth.c")
_lock = threading.Lock()
_lib = None

# stream ids (one independent random stream per tensor role)
S_TINY_A, S_TINY_A_PICK, S_TINY_W = 1, 2, 3
S_ACT, S_ACT_PICK = 10, 11
S_WEIGHT0 = 20
S_KV_OFFSET, S_KV_K, S_KV_V = 30, 31, 32


def build(force: bool = False) -> str:
    """Compile libsynth.so next to this file (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.synth_u64.restype = u64
            lib.synth_u64.argtypes = [u64, u64, u64]
            lib.synth_splitmix64_at.restype = u64
            lib.synth_splitmix64_at.argtypes = [u64, u64]
            lib.synth_uniform.restype = dbl
            lib.synth_uniform.argtypes = [u64, u64, u64]
            lib.synth_normal_bf16.argtypes = [u64, u64, u64, i64, dbl, dbl, vp]
            lib.synth_normal_f32.argtypes = [u64, u64, u64, i64, dbl, dbl, vp]
            lib.synth_t3_matrix_bf16.argtypes = [u64, u64, i64, i64, dbl, vp, dbl, vp]
            lib.synth_normal_matrix_bf16.argtypes = [u64, u64, i64, i64, dbl, vp, dbl, vp]
            lib.synth_kv_chunk_bf16.argtypes = [u64, u64, i64, i64, i64, vp, vp]
            lib.synth_distinct_picks.argtypes = [u64, u64, i64, i64, vp]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def u64(seed: int, stream: int, i: int) -> int:
    return int(_load().synth_u64(seed, stream, i))


def splitmix64_at(state: int, i: int) -> int:
    return int(_load().synth_splitmix64_at(state, i))


def uniform(seed: int, stream: int, i: int) -> float:
    return float(_load().synth_uniform(seed, stream, i))


def picks(seed: int, stream: int, n: int, count: int) -> np.ndarray:
    """First `count` distinct draws of floor(u * n)."""
    out = np.zeros(count, dtype=np.int64)
    _load().synth_distinct_picks(seed, stream, n, count, _ptr(out))
    return out


def normal_bf16(seed: int, stream: int, n: int, mean: float = 0.0, std: float = 1.0,
                first: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    _load().synth_normal_bf16(seed, stream, first, n, mean, std, _ptr(out))
    return out


def normal_f32(seed: int, stream: int, n: int, mean: float = 0.0, std: float = 1.0,
               first: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _load().synth_normal_f32(seed, stream, first, n, mean, std, _ptr(out))
    return out


def outlier_mask(seed: int, stream: int, cols: int, count: int) -> np.ndarray:
    mask = np.zeros(cols, dtype=np.uint8)
    if count > 0:
        mask[picks(seed, stream, cols, count)] = 1
    return mask


def activations(seed: int, rows: int, cols: int, outlier_frac: float = 0.01,
                factor: float = 30.0, scale: float = 0.5) -> np.ndarray:
    """bf16 bits [rows, cols]: 0.5 * Student-t(3), ceil(1% of cols) picked columns x30."""
    count = int(math.ceil(outlier_frac * cols - 1e-9))
    mask = outlier_mask(seed, S_ACT_PICK, cols, count)
    out = np.empty((rows, cols), dtype=np.uint16)
    _load().synth_t3_matrix_bf16(seed, S_ACT, rows, cols, scale, _ptr(mask), factor, _ptr(out))
    return out


def weights(seed: int, index: int, n: int, k: int, std: float = 0.02) -> np.ndarray:
    """bf16 bits [n, k] ~ N(0, std); `index` separates the weights of one workload."""
    out = np.empty((n, k), dtype=np.uint16)
    _load().synth_normal_matrix_bf16(seed, S_WEIGHT0 + index, n, k, std, None, 1.0, _ptr(out))
    return out


def tiny_linear(seed: int = 0):
    """A [128, 512] ~ N(0,1) with 4 picked columns x20; W [256, 512] ~ N(0, 0.02)."""
    mask = outlier_mask(seed, S_TINY_A_PICK, 512, 4)
    a = np.empty((128, 512), dtype=np.uint16)
    _load().synth_normal_matrix_bf16(seed, S_TINY_A, 128, 512, 1.0, _ptr(mask), 20.0, _ptr(a))
    w = np.empty((256, 512), dtype=np.uint16)
    _load().synth_normal_matrix_bf16(seed, S_TINY_W, 256, 512, 0.02, None, 1.0, _ptr(w))
    return a, w


def kv_offsets(seed: int, heads: int, head_dim: int, std: float = 3.0) -> np.ndarray:
    return normal_f32(seed, S_KV_OFFSET, heads * head_dim, 0.0, std)


def kv_chunk(seed: int, chunk: int, tokens: int, heads: int, head_dim: int,
             offsets: np.ndarray | None):
    """(K, V) bf16 bits [tokens, heads, head_dim] of chunk number `chunk`."""
    c = heads * head_dim
    k = np.empty((tokens, heads, head_dim), dtype=np.uint16)
    v = np.empty((tokens, heads, head_dim), dtype=np.uint16)
    off_arr = None if offsets is None else np.ascontiguousarray(offsets, dtype=np.float32)
    off = None if off_arr is None else _ptr(off_arr)
    _load().synth_kv_chunk_bf16(seed, S_KV_K, chunk * tokens, tokens, c, off, _ptr(k))
    _load().synth_kv_chunk_bf16(seed, S_KV_V, chunk * tokens, tokens, c, None, _ptr(v))
    return k, v


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)
