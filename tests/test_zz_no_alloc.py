"""kv_quant_append_noalloc: the KV append for callers that may not allocate device
memory (a framework that owns every device allocation through its own pool, a
real-time loop that must not stall on cudaMalloc/cudaFree, a plugin that only
receives its input and output buffers).  It keeps its per-chunk statistics in a
static device array of the library instead of the cache's scratch region.  Called
through the C ABI and compared with kv_quant_append bit for bit (the tolerance of
every KV test) on two calls in a row.  This file is collected last."""
import ctypes

import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import synth
from gpu_helpers import dev_bf16, device_status

pytestmark = pytest.mark.gpu


def _stream_ptr():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_noalloc_append_equals_append_on_two_calls(cuda_dev):
    heads, dh, T = 24, 128, 1024  # 3072 columns, within the 4096-column limit
    off = synth.kv_offsets(7, heads, dh)
    ref = nv.KVCache(heads, dh, T, 2)
    got = nv.KVCache(heads, dh, T, 2)
    lib = nv.library()
    device_status(clear=True)
    for call, slot in enumerate([0, 1]):
        k, v = synth.kv_chunk(7, call, T, heads, dh, off)
        if call == 1:  # one wide-range column: the exact-sum path also runs on the static array
            k.reshape(T, -1)[3, 5] = 0x7E80
            k.reshape(T, -1)[4, 5] = 0x0001
        kd, vd = dev_bf16(k), dev_bf16(v)
        nv.kv_quant_append(ref, kd, vd, slot)
        st = lib.kv_quant_append_noalloc(ctypes.byref(got.handle), ctypes.c_void_p(kd.data_ptr()),
                                         ctypes.c_void_p(vd.data_ptr()), T, slot, _stream_ptr())
        assert st == nv.OK, nv.status_string(st)
        torch.cuda.synchronize()
        names = ["K codes", "K scales", "V codes", "V scales", "mu", "g"]
        for name, a, b in zip(names, ref.slot_views(slot), got.slot_views(slot)):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f"call {call}: {name} differs"
    assert device_status() == nv.OK


def test_noalloc_rejects_geometry_beyond_the_static_array(cuda_dev):
    cache = nv.KVCache(40, 128, 16, 1)  # 5120 columns > 4096
    k = torch.zeros((16, 40, 128), dtype=torch.bfloat16, device="cuda")
    st = nv.library().kv_quant_append_noalloc(ctypes.byref(cache.handle), ctypes.c_void_p(k.data_ptr()),
                                              ctypes.c_void_p(k.data_ptr()), 16, 0, _stream_ptr())
    assert st == nv.ERR_SHAPE
