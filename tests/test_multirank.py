"""The N > 1 path of bench.py on CPU: two gloo ranks on 127.0.0.1.  Each rank is an
independent replica (its own synthetic chunk); the job's time is the max over ranks;
only rank 0 runs the oracle reference arm."""
import os
import socket
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
