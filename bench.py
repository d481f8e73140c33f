"""Benchmark of the NVFP4 hot path on B200.

One step = one pass of every hot-path step over one batch of synthetic inputs, at
full size:
  * activation pass      X [32768, 3072] bf16: quantize (amax + encode), dequantize to bf16
  * DiT block GEMMs      M = 8192 tokens: quantize the activations [8192, 3072] and
                         [8192, 14336], then the four W4A4 GEMMs (3072->3072,
                         3072->9216 QKV, 3072->14336 FFN up, 14336->3072 FFN down), FP32 out
  * KV cache             append one 8192-token chunk of K, V [8192, 24, 128] into the next
                         of 16 slots, dequantize the latest 4-chunk window (32768 tokens)
  * fused FFN chunk      quantize X [8192, 3072] -> GEMM to 14336 with GELU and NVFP4
                         requantization in the epilogue -> GEMM to 3072, bf16 out
Weights are quantized once before timing ("weight materialization").  The step's
working set (about 2 GB) is far larger than the 126 MB L2, so no flush is added.

value = W4A4 GEMM FLOPs of the step / step time (TFLOP/s, all GPUs); the per-kernel
breakdown carries the GB/s of the memory-bound kernels and every roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: launched with torch.distributed.run, one process per GPU; each rank runs
the same step on its own inputs (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

M_TOK = 8192
HEADS, HEAD_DIM, CHUNK, SLOTS, WINDOW = 24, 128, 8192, 16, 4
ACT_ROWS, ACT_COLS = 32768, 3072
BLOCK_GEMMS = [(3072, 3072), (3072, 9216), (3072, 14336), (14336, 3072)]  # (K, N)
FFN = (3072, 14336)
SCORES_TQ = 1024  # queries scored against the 4-chunk window by the attention-side consumer
METRIC = "W4A4 GEMM TFLOPS; NVFP4 quant/KV-dequant GB/s; % of B200 roofline"
WORKLOAD = ("longlive_dit_block_chunk: act quant/dequant 32768x3072; GEMMs M=8192 "
            "(3072->3072, 3072->9216, 3072->14336, 14336->3072); KV 24x128 append 8192 tok + "
            "4-chunk window; fused FFN 8192x3072->14336(GELU+NVFP4)->3072")


def gemm_flops() -> float:
    f = sum(2.0 * M_TOK * n * k for k, n in BLOCK_GEMMS)
    f += 2.0 * M_TOK * FFN[1] * FFN[0] * 2
    return f


def alg_bytes():
    """Algorithmic bytes per call of each memory-bound kernel group."""
    x = ACT_ROWS * ACT_COLS
    kv = CHUNK * HEADS * HEAD_DIM

    def quant(n):  # two reads of the bf16 input, codes and scales written
        return 2 * 2 * n + n // 2 + n // 16

    return {
        "quantize_32768x3072": quant(x),
        "quantize_8192x3072": quant(M_TOK * 3072),
        "quantize_8192x14336": quant(M_TOK * 14336),
        "quantize_8192x3072_ffn": quant(M_TOK * 3072),
        "dequantize_32768x3072": x // 2 + x // 16 + 2 * x,        # codes + scales in, bf16 out
        "kv_append_8192": 2 * (2 * 2 * kv) + 2 * (kv // 2 + kv // 16),
        "kv_window_4x8192": WINDOW * 2 * (kv // 2 + kv // 16) + WINDOW * 2 * 2 * kv,
    }


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"nvfp4_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- our arm
def rank_seed_offset(rank: int) -> int:
    """Each rank is an independent replica: its synthetic chunk uses its own seeds."""
    return 1000 * rank


def max_over_ranks(values, dist, device):
    """Element-wise max of per-rank timings (the slowest rank sets the job's time);
    identity without a process group."""
    if dist is None:
        return list(values)
    import torch

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


class StepOutputs:
    """Every result one step writes (device).  The end-to-end loop keeps two sets so
    that step i + 1 computes while step i's results travel back to the host."""

    def __init__(self, nv, torch, dev):
        self.qx2 = nv.NVFP4Tensor(ACT_ROWS, ACT_COLS, nv.SF_MMA, dev)
        self.y2 = torch.empty((ACT_ROWS, ACT_COLS), dtype=torch.bfloat16, device=dev)
        self.qa3 = nv.NVFP4Tensor(M_TOK, 3072, nv.SF_MMA, dev)
        self.qa3b = nv.NVFP4Tensor(M_TOK, 14336, nv.SF_MMA, dev)
        self.cs = [torch.empty((M_TOK, n), dtype=torch.float32, device=dev) for _, n in BLOCK_GEMMS]
        self.ko = torch.empty((WINDOW * CHUNK, HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev)
        self.vo = torch.empty_like(self.ko)
        self.qx5 = nv.NVFP4Tensor(M_TOK, FFN[0], nv.SF_MMA, dev)
        self.qh = nv.NVFP4Tensor(M_TOK, FFN[1], nv.SF_MMA, dev)
        self.y5 = torch.empty((M_TOK, FFN[0]), dtype=torch.bfloat16, device=dev)
        self.amax = torch.zeros(8, dtype=torch.float32, device=dev)

    def results(self):
        """The step's results, in a fixed order (the KV slot written is added by the caller)."""
        out = []
        for q in (self.qx2, self.qa3, self.qa3b, self.qx5, self.qh):
            out += [q.codes, q.scales, q.gscale]
        return out + [self.y2, *self.cs, self.ko, self.vo, self.y5, self.amax]


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch

    import nvfp4_w4a4_quantized_amax_b200 as nv

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    seed_off = rank_seed_offset(rank)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    def pinned(bits):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
        return t.pin_memory()

    # ---- inputs (host, then device)
    h_x2 = synth.activations(1 + seed_off, ACT_ROWS, ACT_COLS)
    h_a3 = synth.activations(2 + seed_off, M_TOK, 3072)
    h_a3b = synth.activations(2 + seed_off, M_TOK, 14336)
    h_x5 = synth.activations(4 + seed_off, M_TOK, 3072)
    off = synth.kv_offsets(3 + seed_off, HEADS, HEAD_DIM)
    kv_chunks = [synth.kv_chunk(3 + seed_off, c, CHUNK, HEADS, HEAD_DIM, off) for c in range(2)]

    x2, a3, a3b, x5 = to_dev(h_x2), to_dev(h_a3), to_dev(h_a3b), to_dev(h_x5)
    kvd = [(to_dev(k), to_dev(v)) for k, v in kv_chunks]

    # ---- weights, quantized once (not timed)
    amax_tmp = torch.zeros(1, dtype=torch.float32, device=dev)
    wq = []
    for i, (k, n) in enumerate(BLOCK_GEMMS):
        w = to_dev(synth.weights(2 + seed_off, i, n, k))
        q = nv.NVFP4Tensor(n, k, nv.SF_MMA, dev)
        nv.nvfp4_quantize(w, q, amax_out=amax_tmp)
        wq.append(q)
        del w
    w1 = to_dev(synth.weights(4 + seed_off, 0, FFN[1], FFN[0]))
    w2 = to_dev(synth.weights(4 + seed_off, 1, FFN[0], FFN[1]))
    q1 = nv.NVFP4Tensor(FFN[1], FFN[0], nv.SF_MMA, dev)
    q2 = nv.NVFP4Tensor(FFN[0], FFN[1], nv.SF_MMA, dev)
    nv.nvfp4_quantize(w1, q1, amax_out=amax_tmp)
    nv.nvfp4_quantize(w2, q2, amax_out=amax_tmp)
    del w1, w2

    # ---- outputs (two sets for the end-to-end loop) and the KV cache (state)
    outs = [StepOutputs(nv, torch, dev), StepOutputs(nv, torch, dev)]
    cache = nv.KVCache(HEADS, HEAD_DIM, CHUNK, SLOTS, dev)

    # supplied tensor scale of the fused FFN's requantization: an amax history of
    # the FFN-up output (16 chunks), started by one calibration chunk and updated
    # by every step with that step's max|h|
    o0 = outs[0]
    nv.nvfp4_quantize(x5, o0.qx5, amax_out=o0.amax[4:5])
    nv.nvfp4_gemm(o0.qx5, q1, None, act=nv.ACT_GELU_TANH, q_amax_out=o0.amax[5:6])
    hist = torch.zeros(16, dtype=torch.float32, device=dev)
    g_h = torch.zeros(1, dtype=torch.float32, device=dev)
    nv.nvfp4_amax_history_push(hist, o0.amax[5:6], g_h)
    for s in range(SLOTS):  # fill the cache
        k, v = kvd[s % 2]
        nv.kv_quant_append(cache, k, v, s)
    torch.cuda.synchronize()

    kernels = {}
    launches = [0]

    def timed(name, fn, n_kernels, events):
        if events is not None:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            events.append((name, e0, e1))
        else:
            fn()
        launches[0] += n_kernels

    slot_counter = [0]

    def step(events=None, inputs=None, o=None):
        """One pass of the whole path; returns the KV slot it appended."""
        o = o if o is not None else outs[0]
        X2, A3, A3B, X5, KVK, KVV = inputs if inputs is not None else (
            x2, a3, a3b, x5, kvd[slot_counter[0] % 2][0], kvd[slot_counter[0] % 2][1])
        am = o.amax
        # Order: a kernel inherits the dirty L2 lines of the one before it and pays for
        # their write-back.  The KV append, whose two passes are bound by latency and
        # issue rather than DRAM, takes what the previous step's GEMMs left; the other
        # memory-bound kernels with small outputs follow (each behind a small writer),
        # the two big writers (dequantize 201 MB, KV window 403 MB) last among them, then
        # the GEMMs, which read from L2 and leave DRAM time for the write-back they inherit.
        slot = slot_counter[0] % SLOTS
        timed("kv_append_8192", lambda: nv.kv_quant_append(cache, KVK, KVV, slot), 4, events)
        timed("quantize_8192x3072_ffn", lambda: nv.nvfp4_quantize(X5, o.qx5, amax_out=am[3:4]), 3, events)
        timed("quantize_8192x3072", lambda: nv.nvfp4_quantize(A3, o.qa3, amax_out=am[1:2]), 3, events)
        timed("quantize_8192x14336", lambda: nv.nvfp4_quantize(A3B, o.qa3b, amax_out=am[2:3]), 3, events)
        timed("quantize_32768x3072", lambda: nv.nvfp4_quantize(X2, o.qx2, amax_out=am[0:1]), 3, events)
        timed("dequantize_32768x3072", lambda: nv.nvfp4_dequantize(o.qx2, o.y2), 1, events)
        win = [(slot - WINDOW + 1 + j) % SLOTS for j in range(WINDOW)]
        timed("kv_window_4x8192", lambda: nv.kv_dequant_window(cache, win, o.ko, o.vo), 1, events)
        slot_counter[0] += 1
        for i, (k, n) in enumerate(BLOCK_GEMMS):
            a = o.qa3 if k == 3072 else o.qa3b
            timed(f"gemm_{k}x{n}", lambda a=a, i=i: nv.nvfp4_gemm(a, wq[i], o.cs[i]), 1, events)
        timed("gemm_ffn_up_gelu_requant", lambda: nv.nvfp4_gemm(o.qx5, q1, None, act=nv.ACT_GELU_TANH,
                                                                q_out=o.qh, q_gscale_in=g_h,
                                                                q_amax_out=am[6:7]), 2, events)
        timed("amax_history_push", lambda: nv.nvfp4_amax_history_push(hist, am[6:7], g_h), 1, events)
        timed("gemm_ffn_down_bf16", lambda: nv.nvfp4_gemm(o.qh, q2, o.y5), 1, events)
        return slot

    dist = None
    if world > 1:
        import torch.distributed as dist  # noqa: F811

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    if nv.get_device_status(local_rank) != nv.OK:
        raise RuntimeError("device status after warm-up: " + nv.status_string(nv.get_device_status(local_rank)))

    # ---- timed region: K steps, device-timed
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    launches[0] = 0
    barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    barrier()
    elapsed_ms = t0.elapsed_time(t1)
    clocks = sampler.stop()
    n_launch = launches[0]

    # ---- per-kernel breakdown (separate pass, events around each call)
    evs_all = []
    for _ in range(max(3, min(args.steps, 10))):
        evs = []
        step(evs)
        evs_all.append(evs)
    torch.cuda.synchronize()
    for evs in evs_all:
        for name, e0, e1 in evs:
            kernels.setdefault(name, []).append(e0.elapsed_time(e1))

    # ---- end to end through the C ABI: pinned host inputs in, every result of the
    # step back to pinned host memory.  Two input sets and two output sets on the
    # device: a copy stream brings step i+1's inputs in and another takes step i-1's
    # results out while step i computes; every copy of every timed step ends inside
    # the timed region.
    hp = [pinned(h_x2), pinned(h_a3), pinned(h_a3b), pinned(h_x5), pinned(kv_chunks[0][0]),
          pinned(kv_chunks[0][1])]
    dsets = [[torch.empty(t.shape, dtype=t.dtype, device=dev) for t in hp] for _ in range(2)]
    n_res = len(outs[0].results())
    res_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs[0].results()]
    slot_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in cache.slot_views(0)]
    h2d = sum(t.numel() * t.element_size() for t in hp)
    d2h = sum(t.numel() * t.element_size() for t in res_host + slot_host)
    e2e_steps = max(2, min(args.steps, 10))
    in_stream = torch.cuda.Stream(device=dev)
    out_stream = torch.cuda.Stream(device=dev)
    ready = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    returned = [torch.cuda.Event() for _ in range(2)]
    barrier()
    t2 = torch.cuda.Event(enable_timing=True)
    t3 = torch.cuda.Event(enable_timing=True)
    t2.record(stream)
    in_stream.wait_event(t2)
    for i in range(e2e_steps):
        b = i % 2
        with torch.cuda.stream(in_stream):
            if i >= 2:
                in_stream.wait_event(consumed[b])  # step i-2 has finished reading this input set
            for d, h in zip(dsets[b], hp):
                d.copy_(h, non_blocking=True)
            ready[b].record(in_stream)
        stream.wait_event(ready[b])
        if i >= 2:
            stream.wait_event(returned[b])  # step i-2's results have left this output set
        slot = step(inputs=tuple(dsets[b]), o=outs[b])
        consumed[b].record(stream)
        out_stream.wait_event(consumed[b])
        with torch.cuda.stream(out_stream):
            for h, d in zip(res_host + slot_host, outs[b].results() + list(cache.slot_views(slot))):
                h.copy_(d, non_blocking=True)
            returned[b].record(out_stream)
    for b in range(2):
        stream.wait_event(returned[b])
    t3.record(stream)
    barrier()
    assert len(res_host) == n_res
    e2e_ms = t2.elapsed_time(t3) / e2e_steps
    status = nv.get_device_status(local_rank)
    if status != nv.OK:
        raise RuntimeError("device status: " + nv.status_string(status))

    # ---- the attention-side consumer of the cache (a "next" row, outside the step):
    # scores of SCORES_TQ queries against the latest 4-chunk window with K read from
    # the NVFP4 cache inside the kernel, against the window dequant to bf16 followed
    # by a bf16 batched GEMM (cuBLAS through torch.bmm) on the dequantized keys
    win = [(slot_counter[0] - WINDOW + j) % SLOTS for j in range(WINDOW)]
    q = to_dev(synth.activations(5 + seed_off, SCORES_TQ, HEADS * HEAD_DIM)).view(SCORES_TQ, HEADS, HEAD_DIM)
    s_fused = torch.empty((HEADS, SCORES_TQ, WINDOW * CHUNK), dtype=torch.bfloat16, device=dev)
    s_pair = torch.empty_like(s_fused)
    ko, vo = outs[0].ko, outs[0].vo

    o_fused = torch.empty((SCORES_TQ, HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev)
    o_pair = torch.empty((HEADS, SCORES_TQ, HEAD_DIM), dtype=torch.bfloat16, device=dev)

    def fused():
        nv.kv_window_scores(cache, win, [CHUNK] * WINDOW, q, 1.0, s_fused)

    def pair():
        nv.kv_dequant_window(cache, win, ko, vo)
        torch.bmm(q.transpose(0, 1), ko.permute(1, 2, 0), out=s_pair)

    def ctx_fused():  # the V side: weights (here the bf16 scores buffer) times V^ from the cache
        nv.kv_window_context(cache, win, [CHUNK] * WINDOW, s_fused, o_fused)

    def ctx_pair():
        nv.kv_dequant_window(cache, win, ko, vo)
        torch.bmm(s_pair, vo.transpose(0, 1), out=o_pair)

    scores = {}
    for name, fn in (("kv_window_scores", fused), ("window_then_bmm", pair), ("kv_window_context", ctx_fused),
                     ("window_then_bmm_v", ctx_pair)):
        for _ in range(3):
            fn()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(10):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        scores[name] = e0.elapsed_time(e1) / 10
    del s_fused, s_pair, o_fused, o_pair
    status = nv.get_device_status(local_rank)
    if status != nv.OK:
        raise RuntimeError("device status: " + nv.status_string(status))

    # ---- max over ranks
    ms_per_step, e2e_ms = max_over_ranks([elapsed_ms / args.steps, e2e_ms], dist, dev)
    return {"ms_per_step": ms_per_step, "e2e_ms": e2e_ms, "kernels": kernels, "clocks": clocks,
            "launches": n_launch, "h2d": h2d, "d2h": d2h, "scores": scores}


def scores_summary(t, peaks):
    """Scores of SCORES_TQ queries x 24 heads against the 32768-key window, bf16 out:
    algorithmic bytes = K codes and scales read + queries read + scores written."""
    keys = WINDOW * CHUNK
    c = HEADS * HEAD_DIM
    fused_bytes = keys * c // 2 + keys * c // 16 + SCORES_TQ * c * 2 + HEADS * SCORES_TQ * keys * 2
    pair_bytes = (WINDOW * 2 * (CHUNK * c // 2 + CHUNK * c // 16) + WINDOW * 2 * 2 * CHUNK * c  # window
                  + keys * c * 2 + SCORES_TQ * c * 2 + HEADS * SCORES_TQ * keys * 2)             # bmm
    gbs = fused_bytes / (t["kv_window_scores"] * 1e-3) / 1e9
    # V side: weights [24, tq, keys] bf16 read, V codes and scales read, O written
    ctx_bytes = HEADS * SCORES_TQ * keys * 2 + keys * c // 2 + keys * c // 16 + SCORES_TQ * c * 2
    ctx_gbs = ctx_bytes / (t["kv_window_context"] * 1e-3) / 1e9
    return {"workload": f"{SCORES_TQ} queries x {HEADS} heads x 128 against {keys} window keys, bf16 in/out",
            "kv_window_scores_ms": round(t["kv_window_scores"], 4),
            "window_then_bmm_ms": round(t["window_then_bmm"], 4),
            "speedup": round(t["window_then_bmm"] / t["kv_window_scores"], 3),
            "fused_alg_bytes": fused_bytes, "pair_alg_bytes": pair_bytes,
            "fused_gbs": round(gbs, 1), "fused_frac_hbm": round(gbs / peaks["hbm_gbs"], 3),
            "kv_window_context_ms": round(t["kv_window_context"], 4),
            "window_then_bmm_v_ms": round(t["window_then_bmm_v"], 4),
            "context_speedup": round(t["window_then_bmm_v"] / t["kv_window_context"], 3),
            "context_alg_bytes": ctx_bytes, "context_gbs": round(ctx_gbs, 1),
            "context_frac_hbm": round(ctx_gbs / peaks["hbm_gbs"], 3),
            "flops": 2.0 * HEADS * SCORES_TQ * keys * HEAD_DIM}


# Datasheet figures of one B200 (dense, no sparsity), reported beside the measured ones.
DATASHEET_FP4_TFLOPS = 9000.0
DATASHEET_HBM_GBS = 8000.0


def summarize(res, args, world):
    peaks = read_peaks()
    flops = gemm_flops()
    ab = alg_bytes()
    # Dense FP4 = 4 x dense bf16 (nominal ratio of the datasheet).  The GEMMs are timed
    # inside a ~1.5 ms step at full clock, so the burst bf16 figure is the one that
    # applies (the sustained one was taken seconds into a power-capped loop).
    fp4_peak = peaks["bf16_tflops"] * 4.0
    ktab = {}
    for name, ts in res["kernels"].items():
        avg = statistics.mean(ts)
        entry = {"ms": round(avg, 4)}
        if name.startswith("gemm"):
            if name == "gemm_ffn_up_gelu_requant":
                f = 2.0 * M_TOK * FFN[1] * FFN[0]
            elif name == "gemm_ffn_down_bf16":
                f = 2.0 * M_TOK * FFN[0] * FFN[1]
            else:
                k, n = (int(v) for v in name.split("_")[1].split("x"))
                f = 2.0 * M_TOK * n * k
            entry["tflops"] = round(f / (avg * 1e-3) / 1e12, 1)
            entry["frac_fp4_peak"] = round(entry["tflops"] / fp4_peak, 3)
            entry["frac_fp4_datasheet"] = round(entry["tflops"] / DATASHEET_FP4_TFLOPS, 3)
        else:
            if name in ab:
                gbs = ab[name] / (avg * 1e-3) / 1e9
                entry["gbs"] = round(gbs, 1)
                entry["frac_hbm"] = round(gbs / peaks["hbm_gbs"], 3)
                entry["frac_hbm_datasheet"] = round(gbs / DATASHEET_HBM_GBS, 3)
        ktab[name] = entry
    gemm_names = [n for n in ktab if n.startswith("gemm")]
    gemm_ms = sum(ktab[n]["ms"] for n in gemm_names)
    all_gemm = flops / (gemm_ms * 1e-3) / 1e12
    # the dominant launch: the FFN-up-shaped block GEMM, 8192 x 14336 x 3072, FP32 out
    dom = ktab["gemm_3072x14336"]
    dom_flops = 2.0 * M_TOK * 14336 * 3072
    achieved = dom_flops / (dom["ms"] * 1e-3) / 1e12
    step_ms = res["ms_per_step"]
    value = world * flops / (step_ms * 1e-3) / 1e12
    e2e_value = world * flops / (res["e2e_ms"] * 1e-3) / 1e12
    traffic = None
    prof = os.path.join(ROOT, "profiles", "gemm_pair_kernel_8192x14336x3072_traffic.json")
    if os.path.exists(prof):
        with open(prof) as f:
            traffic = json.load(f).get("dram_bytes_per_launch")
    return {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3 products, f32 accumulate); f32/bf16 scale math",
        "data": "synthetic (seeded splitmix64: 0.5*t3 activations with 1% channels x30, N(0,0.02) weights, N(0,1)+N(0,3)-offset K/V)",
        "config": {"workload": WORKLOAD, "tokens_per_chunk": M_TOK, "l2": "working set ~2 GB > 126 MB L2; no flush",
                   "parallelism": f"replica x{world} (independent chunks per GPU)"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(fp4_peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / fp4_peak, 4), "traffic": traffic,
                     "kernel": "gemm_pair_kernel, one 8192x14336x3072 launch (FP32 out), CUDA events",
                     "peak_source": f"{peaks['source']} bf16 burst x4 (dense FP4/BF16 nominal ratio)",
                     "peak_datasheet": DATASHEET_FP4_TFLOPS,
                     "frac_datasheet": round(achieved / DATASHEET_FP4_TFLOPS, 4),
                     "all_gemm_time_weighted": {"achieved": round(all_gemm, 1),
                                                "frac": round(all_gemm / fp4_peak, 4),
                                                "frac_datasheet": round(all_gemm / DATASHEET_FP4_TFLOPS, 4)}},
        "kernels": ktab,
        "kernels_note": ("CUDA events around each call in a separate pass; bracketing serialises the "
                         "programmatic dependent launches, so these are upper bounds"),
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
        "next_rows": {"attention_side_dequant": scores_summary(res["scores"], peaks)},
    }


# ----------------------------------------------------------------- CPU oracle arm
# The oracle (plain C + a float64 numpy matmul for the GEMM) timed per kernel on a
# bounded sample of the step's workload, in worker processes started with `spawn`:
# one worker = the single-threaded oracle (BLAS limited to one thread); W workers =
# the same sample in W processes at once (one per host core), whose throughput is
# W samples over the slowest worker's time.  The step-level figure scales each
# kernel's sample throughput to its full work in one step.

# per-sample work of each oracle kernel (rows / tokens of the step's inputs)
CPU_SAMPLE = {"quantize_rows": 1024, "dequantize_rows": 1024, "kv_tokens": 512, "window_tokens": 1024,
              "gemm_rows": 128, "gemm_cols": 896}


def cpu_step_work():
    """Full work of one step per oracle kernel: bytes for the memory-bound kernels
    (the GPU's algorithmic counts), FLOPs for the GEMMs."""
    quant_elems = ACT_ROWS * ACT_COLS + M_TOK * 3072 * 2 + M_TOK * 14336 * 2  # incl. the FFN requant of h
    pair = HEADS * HEAD_DIM
    return {"quantize": quant_elems * 4.5625, "dequantize": ACT_ROWS * ACT_COLS * 2.5625,
            "kv_append": CHUNK * pair * 9.125, "kv_window": WINDOW * CHUNK * pair * 5.125,
            "gemm": gemm_flops()}


def _cpu_worker(idx, barrier, tasks, results):
    """One oracle worker: builds its sample inputs, then for every task waits at the
    barrier with the other workers and times each kernel on its sample."""
    import threadpoolctl

    import oracle

    threadpoolctl.threadpool_limits(1)
    sd = 7 + idx
    x = synth.activations(sd, CPU_SAMPLE["quantize_rows"], ACT_COLS)
    qd = oracle.quantize(synth.activations(sd, CPU_SAMPLE["dequantize_rows"], ACT_COLS))
    off = synth.kv_offsets(3, HEADS, HEAD_DIM)
    k, v = synth.kv_chunk(sd, 0, CPU_SAMPLE["kv_tokens"], HEADS, HEAD_DIM, off)
    kw, vw = synth.kv_chunk(sd, 1, CPU_SAMPLE["window_tokens"], HEADS, HEAD_DIM, off)
    ch = oracle.kv_append(kw, vw)
    qa = oracle.quantize(synth.activations(sd, CPU_SAMPLE["gemm_rows"], 3072))
    qw = oracle.quantize(synth.weights(sd, 2, CPU_SAMPLE["gemm_cols"], 3072))
    pair = HEADS * HEAD_DIM
    work = {"quantize": x.size * 4.5625, "dequantize": qd.rows * qd.cols * 2.5625,
            "kv_append": CPU_SAMPLE["kv_tokens"] * pair * 9.125,
            "kv_window": CPU_SAMPLE["window_tokens"] * pair * 5.125,
            "gemm": 2.0 * CPU_SAMPLE["gemm_rows"] * CPU_SAMPLE["gemm_cols"] * 3072}
    runs = {"quantize": lambda: oracle.quantize(x), "dequantize": lambda: oracle.dequantize(qd),
            "kv_append": lambda: oracle.kv_append(k, v), "kv_window": lambda: oracle.kv_dequant_chunk(ch),
            "gemm": lambda: oracle.gemm_ref(qa.codes, qa.scales, qa.g, qw.codes, qw.scales, qw.g)}
    results.put(("ready", idx, None))
    while True:
        t = tasks.get()
        if t is None:
            return
        out = {}
        for name, fn in runs.items():
            barrier.wait()
            t0 = time.perf_counter()
            fn()
            out[name] = (time.perf_counter() - t0, work[name])
        results.put(("done", idx, out))


class OracleCPU:
    """`workers` oracle processes (spawned, so safe after CUDA has been initialised)."""

    def __init__(self, workers: int):
        import multiprocessing as mp

        ctx = mp.get_context("spawn")
        self.n = workers
        self.barrier = ctx.Barrier(workers)
        self.tasks = [ctx.Queue() for _ in range(workers)]
        self.results = ctx.Queue()
        self.procs = [ctx.Process(target=_cpu_worker, args=(i, self.barrier, self.tasks[i], self.results),
                                  daemon=True) for i in range(workers)]
        for pr in self.procs:
            pr.start()
        for _ in range(workers):
            self.results.get(timeout=600)

    def pass_(self):
        """One timed pass over every kernel: {kernel: (seconds, work per second)},
        seconds = the slowest worker's time, throughput = all workers' work / it."""
        for q in self.tasks:
            q.put("run")
        outs = [self.results.get(timeout=600)[2] for _ in range(self.n)]
        res = {}
        for name in outs[0]:
            secs = max(o[name][0] for o in outs)
            res[name] = (secs, sum(o[name][1] for o in outs) / secs)
        return res

    def close(self):
        for q in self.tasks:
            q.put(None)
        for pr in self.procs:
            pr.join(timeout=30)


def cpu_summary(per_kernel):
    """Per-kernel throughputs and the step-level GEMM TFLOP/s they imply: each
    kernel's full work in one step divided by its sample throughput, summed."""
    full = cpu_step_work()
    step_s = sum(full[k] / per_kernel[k][1] for k in full)
    table = {k: ({"tflops": per_kernel[k][1] / 1e12} if k == "gemm" else {"gbs": per_kernel[k][1] / 1e9})
             for k in full}
    return gemm_flops() / step_s / 1e12, step_s, table


CPU_SAMPLE_TEXT = ("per kernel, per worker: quantize 1024x3072 activation rows, dequantize 1024x3072, KV append "
                   "512 tokens x 24 x 128, KV window 1024 tokens, GEMM 128 rows x 896 weight rows x K 3072; "
                   "each kernel's throughput scaled to its full work in one step; inputs built before timing")


def host_cores() -> int:
    """Host cores this process may run on, at most 32 (one oracle worker each)."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, 32))


def cpu_baseline_line():
    """The cpu_baseline object: the oracle single-threaded and on the host's cores."""
    cores = host_cores()
    one = OracleCPU(1)
    try:
        v1, s1, t1 = cpu_summary(one.pass_())
    finally:
        one.close()
    allc = OracleCPU(cores)
    try:
        va, sa, ta = cpu_summary(allc.pass_())
    finally:
        allc.close()
    return {"value": va, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": CPU_SAMPLE_TEXT,
            "step_s": sa, "per_kernel": ta,
            "single_thread": {"value": v1, "cores": 1, "step_s": s1, "per_kernel": t1}}


def run_reference(args, rank, world):
    """The oracle arm: every step is one pass of the per-kernel samples on all host
    cores (one worker process each); rank 0 only."""
    if rank != 0:
        return None
    cores = host_cores()
    pool = OracleCPU(cores)
    try:
        for _ in range(args.warmup):
            pool.pass_()
        steps = [cpu_summary(pool.pass_()) for _ in range(args.steps)]
    finally:
        pool.close()
    step_s = statistics.mean(s for _, s, _ in steps)
    value = gemm_flops() / step_s / 1e12
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64/f32 (CPU oracle)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": CPU_SAMPLE_TEXT},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": CPU_SAMPLE_TEXT, "per_kernel": steps[-1][2]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def run_single_kernel(args):
    """A small case of one kernel, launched `--iters` times after its inputs are
    prepared (for profilers: few launches, a few hundred MB on the device)."""
    import torch

    import nvfp4_w4a4_quantized_amax_b200 as nv

    dev = torch.device("cuda", 0)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    amax = torch.zeros(4, dtype=torch.float32, device=dev)
    if args.kernel.startswith("gemm"):
        M, N, K = (int(v) for v in args.shape.split(","))
        qa = nv.NVFP4Tensor(M, K, nv.SF_MMA, dev)
        qw = nv.NVFP4Tensor(N, K, nv.SF_MMA, dev)
        nv.nvfp4_quantize(to_dev(synth.activations(2, M, K)), qa, amax_out=amax[0:1])
        nv.nvfp4_quantize(to_dev(synth.weights(2, 0, N, K)), qw, amax_out=amax[1:2])
        if args.kernel == "gemm_fused":
            qh = nv.NVFP4Tensor(M, N, nv.SF_MMA, dev)
            g = torch.tensor([0.01], dtype=torch.float32, device=dev)
            fn = lambda: nv.nvfp4_gemm(qa, qw, None, act=nv.ACT_GELU_TANH, q_out=qh, q_gscale_in=g)  # noqa: E731
        else:
            c = torch.empty((M, N), dtype=torch.float32, device=dev)
            fn = lambda: nv.nvfp4_gemm(qa, qw, c)  # noqa: E731
    elif args.kernel in ("quantize", "dequantize"):
        R, C = (int(v) for v in args.shape.split(","))
        x = to_dev(synth.activations(1, R, C))
        q = nv.NVFP4Tensor(R, C, nv.SF_MMA, dev)
        nv.nvfp4_quantize(x, q, amax_out=amax[0:1])
        y = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
        fn = (lambda: nv.nvfp4_quantize(x, q, amax_out=amax[0:1])) if args.kernel == "quantize" else \
            (lambda: nv.nvfp4_dequantize(q, y))
    elif args.kernel == "lora_merge":
        # FFN-up weight 14336 x 3072 (bf16) + rank-64 LoRA -> FP32 W' (then quantized offline)
        rows, cols, rank = 14336, 3072, 64
        rng = np.random.default_rng(7)
        w = to_dev(synth.weights(2, 2, rows, cols))
        lb = torch.from_numpy((rng.standard_normal((rows, rank)) * 0.02).astype(np.float32)).to(dev)
        la = torch.from_numpy((rng.standard_normal((rank, cols)) * 0.02).astype(np.float32)).to(dev)
        out = torch.empty((rows, cols), dtype=torch.float32, device=dev)
        fn = lambda: nv.nvfp4_lora_merge(w, lb, la, 2.0 / rank, out)  # noqa: E731
    elif args.kernel == "kv_window_sink":
        # sink-aware window: a 1024-token sink slot, a 4096-token shot-sink slot, three
        # full sliding slots and the newest, partial slot (3000 tokens): 32696 tokens
        off = synth.kv_offsets(3, HEADS, HEAD_DIM)
        k, v = synth.kv_chunk(3, 0, CHUNK, HEADS, HEAD_DIM, off)
        kd, vd = to_dev(k), to_dev(v)
        cache = nv.KVCache(HEADS, HEAD_DIM, CHUNK, 6, dev)
        fills = [1024, 4096, CHUNK, CHUNK, CHUNK, 3000]
        for sl, n in enumerate(fills):
            nv.kv_quant_append(cache, kd[:n], vd[:n], sl)
        ko = torch.empty((sum(fills), HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev)
        vo = torch.empty_like(ko)
        fn = lambda: nv.kv_dequant_window_tokens(cache, list(range(6)), fills, ko, vo)  # noqa: E731
    elif args.kernel in ("kv_scores", "kv_context"):
        # attention scores (or outputs) of SCORES_TQ queries x 24 heads against a 4-chunk
        # window, bf16 out: the workload of the attention-side measurement of the step run
        off = synth.kv_offsets(3, HEADS, HEAD_DIM)
        k, v = synth.kv_chunk(3, 0, CHUNK, HEADS, HEAD_DIM, off)
        kd, vd = to_dev(k), to_dev(v)
        cache = nv.KVCache(HEADS, HEAD_DIM, CHUNK, WINDOW, dev)
        for sl in range(WINDOW):
            nv.kv_quant_append(cache, kd, vd, sl)
        tq = args.tq
        q = to_dev(synth.activations(5, tq, HEADS * HEAD_DIM)).view(tq, HEADS, HEAD_DIM)
        s_out = torch.empty((HEADS, tq, WINDOW * CHUNK), dtype=torch.bfloat16, device=dev)
        win = list(range(WINDOW))
        fn = lambda: nv.kv_window_scores(cache, win, [CHUNK] * WINDOW, q, 1.0, s_out)  # noqa: E731
        # the same result through the window dequant to bf16 and a cuBLAS batched GEMM
        ko = torch.empty((WINDOW * CHUNK, HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev)
        vo = torch.empty_like(ko)
        s_pair = torch.empty_like(s_out)

        def pair_fn():
            nv.kv_dequant_window(cache, win, ko, vo)
            torch.bmm(q.transpose(0, 1), ko.permute(1, 2, 0), out=s_pair)
        if args.kernel == "kv_context":
            nv.kv_window_scores(cache, win, [CHUNK] * WINDOW, q, 1.0 / 128.0, s_out)
            o = torch.empty((tq, HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev)
            o_pair = torch.empty((HEADS, tq, HEAD_DIM), dtype=torch.bfloat16, device=dev)
            fn = lambda: nv.kv_window_context(cache, win, [CHUNK] * WINDOW, s_out, o)  # noqa: E731

            def pair_fn():
                nv.kv_dequant_window(cache, win, ko, vo)
                torch.bmm(s_out, vo.transpose(0, 1), out=o_pair)
    elif args.kernel in ("kv_append", "kv_window"):
        off = synth.kv_offsets(3, HEADS, HEAD_DIM)
        k, v = synth.kv_chunk(3, 0, CHUNK, HEADS, HEAD_DIM, off)
        kd, vd = to_dev(k), to_dev(v)
        cache = nv.KVCache(HEADS, HEAD_DIM, CHUNK, WINDOW, dev)
        for sl in range(WINDOW):
            nv.kv_quant_append(cache, kd, vd, sl)
        ko = torch.empty((WINDOW * CHUNK, HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev)
        vo = torch.empty_like(ko)
        fn = (lambda: nv.kv_quant_append(cache, kd, vd, 0)) if args.kernel == "kv_append" else \
            (lambda: nv.kv_dequant_window(cache, list(range(WINDOW)), ko, vo))
    else:
        raise SystemExit(f"unknown kernel {args.kernel}")
    for _ in range(args.kernel_warmup):  # one-time launch setup stays out of the timed calls
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    st = nv.get_device_status(0)
    line = {"kernel": args.kernel, "shape": args.shape, "iters": args.iters,
            "ms_per_call": e0.elapsed_time(e1) / args.iters, "status": st}
    if args.kernel in ("kv_scores", "kv_context"):
        line["shape"] = f"{args.tq} queries x {HEADS} heads x {HEAD_DIM} against {WINDOW * CHUNK} keys"
        for _ in range(args.kernel_warmup):
            pair_fn()
        e0.record()
        for _ in range(args.iters):
            pair_fn()
        e1.record()
        torch.cuda.synchronize()
        line["window_then_bmm_ms"] = e0.elapsed_time(e1) / args.iters
    print(json.dumps(line))
    if st != nv.OK:
        raise SystemExit(1)


def free_port() -> int:
    import socket

    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def relaunch(n: int) -> int:
    """Start this command again under torch.distributed.run with n processes (one per
    GPU) and return its exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.abspath(__file__),
           *sys.argv[1:]]
    print(f"bench.py: --gpus {n}: starting {n} ranks under torch.distributed.run", file=sys.stderr, flush=True)
    return subprocess.call(cmd)


def world_from_env(gpus: int):
    """(world, rank, local_rank) from the launcher's environment; --gpus must match it."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != gpus:
        raise SystemExit(f"bench.py: --gpus {gpus} but WORLD_SIZE={world}: launch one process per GPU "
                         f"(or leave WORLD_SIZE unset and let bench.py start them)")
    return world, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", default=None,
                    help="profiling mode: gemm | gemm_fused | quantize | dequantize | kv_append | kv_window | kv_window_sink | "
                         "kv_scores | kv_context | lora_merge")
    ap.add_argument("--shape", default="8192,14336,3072", help="M,N,K for gemm; rows,cols for (de)quantize")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--tq", type=int, default=SCORES_TQ, help="queries for --kernel kv_scores / kv_context")
    ap.add_argument("--kernel-warmup", type=int, default=1,
                    help="untimed calls before the timed ones in --kernel mode")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.kernel:
        run_single_kernel(args)
        return
    if args.gpus < 1:
        raise SystemExit("bench.py: --gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch(args.gpus))
    world, rank, local_rank = world_from_env(args.gpus)

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line))
        return

    import torch

    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        probe = torch.ones(1, device="cuda")
        dist.all_reduce(probe)  # the communicator is built here
        print(f"bench.py: rank {rank}/{world} on cuda:{local_rank}: NCCL {'.'.join(map(str, torch.cuda.nccl.version()))} "
              f"communicator ready (all_reduce of ones = {int(probe.item())})", file=sys.stderr, flush=True)
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            line = summarize(res, args, world)
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline_line()
            print(json.dumps(line))
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
