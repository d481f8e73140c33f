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

    # ---- outputs and intermediates
    qx2 = nv.NVFP4Tensor(ACT_ROWS, ACT_COLS, nv.SF_MMA, dev)
    y2 = torch.empty((ACT_ROWS, ACT_COLS), dtype=torch.bfloat16, device=dev)
    qa3 = nv.NVFP4Tensor(M_TOK, 3072, nv.SF_MMA, dev)
    qa3b = nv.NVFP4Tensor(M_TOK, 14336, nv.SF_MMA, dev)
    cs = [torch.empty((M_TOK, n), dtype=torch.float32, device=dev) for _, n in BLOCK_GEMMS]
    qx5 = nv.NVFP4Tensor(M_TOK, FFN[0], nv.SF_MMA, dev)
    qh = nv.NVFP4Tensor(M_TOK, FFN[1], nv.SF_MMA, dev)
    y5 = torch.empty((M_TOK, FFN[0]), dtype=torch.bfloat16, device=dev)
    cache = nv.KVCache(HEADS, HEAD_DIM, CHUNK, SLOTS, dev)
    ko = torch.empty((WINDOW * CHUNK, HEADS, HEAD_DIM), dtype=torch.bfloat16, device=dev)
    vo = torch.empty_like(ko)
    amax = torch.zeros(8, dtype=torch.float32, device=dev)

    # supplied tensor scale of the fused FFN's requantization: an amax history of
    # the FFN-up output (16 chunks), started by one calibration chunk and updated
    # by every step with that step's max|h|
    nv.nvfp4_quantize(x5, qx5, amax_out=amax[4:5])
    nv.nvfp4_gemm(qx5, q1, None, act=nv.ACT_GELU_TANH, q_amax_out=amax[5:6])
    hist = torch.zeros(16, dtype=torch.float32, device=dev)
    g_h = torch.zeros(1, dtype=torch.float32, device=dev)
    nv.nvfp4_amax_history_push(hist, amax[5:6], g_h)
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

    def step(events=None, inputs=None):
        X2, A3, A3B, X5, KVK, KVV = inputs if inputs is not None else (
            x2, a3, a3b, x5, kvd[slot_counter[0] % 2][0], kvd[slot_counter[0] % 2][1])
        timed("quantize_32768x3072", lambda: nv.nvfp4_quantize(X2, qx2, amax_out=amax[0:1]), 3, events)
        timed("dequantize_32768x3072", lambda: nv.nvfp4_dequantize(qx2, y2), 1, events)
        timed("quantize_8192x3072", lambda: nv.nvfp4_quantize(A3, qa3, amax_out=amax[1:2]), 3, events)
        timed("quantize_8192x14336", lambda: nv.nvfp4_quantize(A3B, qa3b, amax_out=amax[2:3]), 3, events)
        for i, (k, n) in enumerate(BLOCK_GEMMS):
            a = qa3 if k == 3072 else qa3b
            timed(f"gemm_{k}x{n}", lambda a=a, i=i: nv.nvfp4_gemm(a, wq[i], cs[i]), 1, events)
        slot = slot_counter[0] % SLOTS
        timed("kv_append_8192", lambda: nv.kv_quant_append(cache, KVK, KVV, slot), 4, events)
        win = [(slot - WINDOW + 1 + j) % SLOTS for j in range(WINDOW)]
        timed("kv_window_4x8192", lambda: nv.kv_dequant_window(cache, win, ko, vo), 1, events)
        slot_counter[0] += 1
        timed("quantize_8192x3072_ffn", lambda: nv.nvfp4_quantize(X5, qx5, amax_out=amax[3:4]), 3, events)
        timed("gemm_ffn_up_gelu_requant", lambda: nv.nvfp4_gemm(qx5, q1, None, act=nv.ACT_GELU_TANH,
                                                                q_out=qh, q_gscale_in=g_h,
                                                                q_amax_out=amax[6:7]), 2, events)
        timed("amax_history_push", lambda: nv.nvfp4_amax_history_push(hist, amax[6:7], g_h), 1, events)
        timed("gemm_ffn_down_bf16", lambda: nv.nvfp4_gemm(qh, q2, y5), 1, events)

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

    # ---- end to end through the C ABI: pinned host inputs in, the FFN output back.
    # Inputs are double-buffered on the device: a copy stream brings step i+1's
    # inputs in while step i computes (every step's copies stay inside the timed
    # region); the outputs go back on the compute stream after each step.
    hp = [pinned(h_x2), pinned(h_a3), pinned(h_a3b), pinned(h_x5), pinned(kv_chunks[0][0]),
          pinned(kv_chunks[0][1])]
    dsets = [[torch.empty(t.shape, dtype=t.dtype, device=dev) for t in hp] for _ in range(2)]
    y_host = torch.empty(y5.shape, dtype=y5.dtype).pin_memory()
    amax_host = torch.empty(amax.shape, dtype=amax.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in hp)
    d2h = y_host.numel() * y_host.element_size() + amax_host.numel() * amax_host.element_size()
    e2e_steps = max(2, min(args.steps, 10))
    copy_stream = torch.cuda.Stream(device=dev)
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    barrier()
    t2 = torch.cuda.Event(enable_timing=True)
    t3 = torch.cuda.Event(enable_timing=True)
    t2.record(stream)
    copy_stream.wait_event(t2)
    for i in range(e2e_steps):
        b = i % 2
        with torch.cuda.stream(copy_stream):
            if i >= 2:
                copy_stream.wait_event(free[b])  # step i-2 has finished reading this set
            for d, h in zip(dsets[b], hp):
                d.copy_(h, non_blocking=True)
            ready[b].record(copy_stream)
        stream.wait_event(ready[b])
        step(inputs=tuple(dsets[b]))
        free[b].record(stream)
        y_host.copy_(y5, non_blocking=True)
        amax_host.copy_(amax, non_blocking=True)
    t3.record(stream)
    barrier()
    e2e_ms = t2.elapsed_time(t3) / e2e_steps
    status = nv.get_device_status(local_rank)
    if status != nv.OK:
        raise RuntimeError("device status: " + nv.status_string(status))

    # ---- max over ranks
    ms_per_step, e2e_ms = max_over_ranks([elapsed_ms / args.steps, e2e_ms], dist, dev)
    return {"ms_per_step": ms_per_step, "e2e_ms": e2e_ms, "kernels": kernels, "clocks": clocks,
            "launches": n_launch, "h2d": h2d, "d2h": d2h}


def summarize(res, args, world):
    peaks = read_peaks()
    flops = gemm_flops()
    ab = alg_bytes()
    fp4_peak = peaks["bf16_tflops_sustained"] * 4.0  # dense FP4 = 4x dense bf16 (nominal ratio)
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
        else:
            if name in ab:
                gbs = ab[name] / (avg * 1e-3) / 1e9
                entry["gbs"] = round(gbs, 1)
                entry["frac_hbm"] = round(gbs / peaks["hbm_gbs"], 3)
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
                     "all_gemm_time_weighted": {"achieved": round(all_gemm, 1),
                                                "frac": round(all_gemm / fp4_peak, 4)},
                     "peak_source": f"{peaks['source']} bf16 sustained x4 (dense FP4/BF16 nominal ratio)"},
        "kernels": ktab,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
    }


# ----------------------------------------------------------------- CPU oracle arm
_ORACLE_WEIGHTS = {}


def oracle_weights():
    """Weights quantized once by the oracle (weight materialization, not timed)."""
    import oracle

    if not _ORACLE_WEIGHTS:
        for i, (k, n) in enumerate(BLOCK_GEMMS):
            _ORACLE_WEIGHTS[("blk", i)] = oracle.quantize(synth.weights(2, i, n, k))
        _ORACLE_WEIGHTS["w1"] = oracle.quantize(synth.weights(4, 0, FFN[1], FFN[0]))
        _ORACLE_WEIGHTS["w2"] = oracle.quantize(synth.weights(4, 1, FFN[0], FFN[1]))
    return _ORACLE_WEIGHTS


def oracle_sample_step(frac_rows: int = 128, frac_cols: int = 1):
    """The oracle on a bounded sample of one step: 1/frac_rows of every row count
    (activation rows, GEMM rows, KV tokens) and 1/frac_cols of every GEMM's output
    columns (a slice of the quantized weight rows), weights already quantized.
    Inputs are generated before the clock starts.  Returns (seconds, GEMM FLOPs)."""
    import oracle

    def part(q, nrows, ncols):  # a slice of a quantized tensor (indexing only)
        return oracle.Quantized(q.codes[:nrows, : ncols // 2], q.scales[:nrows, : ncols // 16], q.g, q.amax,
                                nrows, ncols)

    W = oracle_weights()
    if frac_cols > 1:
        W = {key: part(q, max(16, q.rows // frac_cols), q.cols) for key, q in W.items()}
    r2 = ACT_ROWS // frac_rows
    m = M_TOK // frac_rows
    t = CHUNK // frac_rows
    x2 = synth.activations(1, r2, ACT_COLS)
    a3 = synth.activations(2, m, 3072)
    a3b = synth.activations(2, m, 14336)
    x5 = synth.activations(4, m, FFN[0])
    off = synth.kv_offsets(3, HEADS, HEAD_DIM)
    kvs = [synth.kv_chunk(3, c, t, HEADS, HEAD_DIM, off) for c in range(WINDOW)]
    flops = 0.0
    t0 = time.perf_counter()
    q = oracle.quantize(x2)
    oracle.dequantize(q)
    acts = {3072: oracle.quantize(a3), 14336: oracle.quantize(a3b)}
    for i, (k, n) in enumerate(BLOCK_GEMMS):
        w, a = W[("blk", i)], acts[k]
        oracle.gemm_ref(a.codes, a.scales, a.g, w.codes, w.scales, w.g)
        flops += 2.0 * m * w.codes.shape[0] * k
    chunks = [oracle.kv_append(kk, vv) for kk, vv in kvs]
    for ch in chunks:
        oracle.kv_dequant_chunk(ch)
    qx = oracle.quantize(x5)
    c1, _ = oracle.gemm_ref(qx.codes, qx.scales, qx.g, W["w1"].codes, W["w1"].scales, W["w1"].g)
    h = oracle.gelu_tanh(c1.astype(np.float32)).astype(np.float32)
    # the (sliced) FFN-up output feeds the first columns of FFN-down's K
    w2 = part(W["w2"], W["w2"].rows, h.shape[1]) if frac_cols > 1 else W["w2"]
    qh = oracle.quantize(h)
    oracle.gemm_ref(qh.codes, qh.scales, qh.g, w2.codes, w2.scales, w2.g)
    flops += 2.0 * m * h.shape[1] * FFN[0] + 2.0 * m * w2.codes.shape[0] * h.shape[1]
    return time.perf_counter() - t0, flops


def cpu_cores_used() -> int:
    # the oracle's C code is single-threaded; numpy's float64 matmul may use BLAS threads
    try:
        import threadpoolctl

        info = threadpoolctl.threadpool_info()
        return max([1] + [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"])
    except Exception:  # noqa: BLE001
        return 1


def run_reference(args, rank, world):
    if rank != 0:
        return None
    oracle_weights()
    for _ in range(args.warmup):
        oracle_sample_step(1024, 16)
    secs, fl = [], 0.0
    for _ in range(args.steps):
        s, fl = oracle_sample_step(512, 16)
        secs.append(s)
    mean_s = statistics.mean(secs)
    value = fl / mean_s / 1e12
    sample = ("1/512 of every row count of one step (64 activation rows, 16 GEMM rows, 16 KV tokens "
              "per chunk) and 1/16 of every GEMM's output columns; weights quantized once before timing")
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": mean_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64/f32 (CPU oracle)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores_used(), "kind": "oracle",
                         "sample": sample},
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
    print(json.dumps({"kernel": args.kernel, "shape": args.shape, "iters": args.iters,
                      "ms_per_call": e0.elapsed_time(e1) / args.iters, "status": st}))
    if st != nv.OK:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", default=None,
                    help="profiling mode: gemm | gemm_fused | quantize | dequantize | kv_append | kv_window | kv_window_sink | lora_merge")
    ap.add_argument("--shape", default="8192,14336,3072", help="M,N,K for gemm; rows,cols for (de)quantize")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--kernel-warmup", type=int, default=1,
                    help="untimed calls before the timed ones in --kernel mode")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.kernel:
        run_single_kernel(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            line = summarize(res, args, world)
            if world == 1 and not args.no_cpu_baseline:
                oracle_weights()
                s, fl = oracle_sample_step(32)
                line["cpu_baseline"] = {"value": fl / s / 1e12, "unit": "TFLOP/s", "cores": cpu_cores_used(),
                                        "kind": "oracle",
                                        "sample": ("1/32 of every row count of one step (1024 activation rows, "
                                                   "256 GEMM rows, 256 KV tokens per chunk), weights "
                                                   "quantized once before timing; timed once")}
            print(json.dumps(line))
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
