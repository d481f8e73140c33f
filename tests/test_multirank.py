"""The N > 1 paths on CPU, as gloo ranks on 127.0.0.1.
  * bench.py: each rank is an independent replica (its own synthetic chunk); the job's
    time is the max over ranks; only rank 0 runs the oracle reference arm; `--gpus N`
    starts N ranks itself and refuses a WORLD_SIZE that differs from N.
  * Row-sharded quantization (one tensor's rows split across ranks): the module's
    steps with the oracle standing in for the GPU kernels; every rank's codes and
    scales equal the same rows of a one-process quantization of the whole tensor."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank timings differ; every rank must see the slowest
        mine = [10.0 + rank * 2.5, 100.0 - rank * 7.0]
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        # replicas draw different synthetic chunks
        x = synth.activations(1 + bench.rank_seed_offset(rank), 4, 32)
        digest = int(np.bitwise_xor.reduce(x.astype(np.uint64).ravel()))
        ref = bench.run_reference(type("A", (), {"warmup": 0, "steps": 0})(), rank, world) if rank != 0 else None
        out.put((rank, got, digest, ref))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_timing_and_independent_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, got, digest, ref = q.get(timeout=120)
        res[rank] = (got, digest, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == [12.5, 100.0]
    assert res[0][1] != res[1][1]
    assert res[1][2] is None  # the reference arm does no work off rank 0


def test_max_over_ranks_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1.0, 2.0], None, None) == [1.0, 2.0]


def _shard_worker(rank, world, port, out, plant_nan):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from nvfp4_w4a4_quantized_amax_b200 import sharded

    class OracleOps(sharded.LibraryOps):
        """The module's four steps with the oracle in place of the GPU kernels and the
        gloo group for the exchange (the same all_reduce_max as on GPUs)."""

        def amax(self, x, ws, stream=None):
            f = synth.bf16_bits_to_f32(x)
            ws.amax[0] = float(np.abs(f).max()) if np.isfinite(f).all() else float("nan")

        def tensor_scale(self, ws, stream=None):
            hist, g = oracle.amax_history_push(ws.history.numpy(), float(ws.amax[0]))
            ws.history.copy_(torch.from_numpy(hist))
            ws.gscale[0] = g

        def quantize(self, x, out, ws, stream=None):
            q = oracle.quantize(x, gscale=float(ws.gscale[0]))
            out.update(codes=q.codes, scales=q.scales, g=q.g)

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = synth.activations(11, 301, 96)  # every rank builds the same tensor, keeps its rows
        if plant_nan:
            x[290, 7] = 0x7FC0  # a NaN in the last rank's rows
        r0, r1 = sharded.row_range(x.shape[0], rank, world)
        ws = sharded.ShardWorkspace.create("cpu")
        res = {}
        try:
            sharded.quantize_row_shard(x[r0:r1].copy(), res, ws, ops=OracleOps())
            out.put((rank, r0, r1, res["codes"], res["scales"], res["g"], None))
        except ValueError as e:  # the oracle's amax history rejects a non-finite amax
            out.put((rank, r0, r1, None, None, None, str(e)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run_shards(world, plant_nan):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q, plant_nan)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res, key=lambda t: t[0])


@pytest.mark.parametrize("world", [2, 3])
def test_row_sharded_quantize_equals_one_process(world):
    sys.path.insert(0, ROOT)
    import oracle
    import synth

    full = oracle.quantize(synth.activations(11, 301, 96))
    res = _run_shards(world, plant_nan=False)
    assert [r[1] for r in res] == sorted(r[1] for r in res) and res[-1][2] == 301
    for rank, r0, r1, codes, scales, g, err in res:
        assert err is None
        assert g == full.g
        assert np.array_equal(codes, full.codes[r0:r1]) and np.array_equal(scales, full.scales[r0:r1])


def test_row_sharded_nan_on_one_rank_reaches_every_rank():
    res = _run_shards(2, plant_nan=True)
    assert all(err is not None for *_, err in res)


def test_bench_gpus_flag_starts_the_ranks_itself():
    """`bench.py --gpus 2` without a launcher environment starts two ranks under
    torch.distributed.run; here through the oracle arm, which runs on rank 0 only and
    prints exactly one JSON line for the job."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert "starting 2 ranks" in r.stderr


def test_bench_refuses_a_world_size_that_differs_from_gpus():
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference"],
                       capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE=3" in r.stderr
