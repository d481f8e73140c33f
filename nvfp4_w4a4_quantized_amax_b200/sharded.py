"""Row-sharded quantization of one tensor across GPUs (one process per GPU).

A tensor whose rows are split across ranks still has ONE tensor scale
(techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存", §一:
one FP32 scale for the whole tensor), g = RN(amax / 2688) with amax over every row
of every rank.  Each rank therefore:
  1. takes the amax of its own rows                    (nvfp4_amax, on its GPU)
  2. combines it with the others by an all-reduce(MAX) (torch.distributed; 4 bytes)
  3. turns the global amax into g                      (nvfp4_amax_history_push with a
                                                        one-entry history, on its GPU)
  4. quantizes its rows with that g                    (nvfp4_quantize, supplied scale)
The maximum is exact and independent of the order in which ranks combine, and each
row's codes and scales depend only on the row and on g, so every rank's output is
bit-identical to the same rows of a one-GPU quantization of the whole tensor.

The all-reduce runs on the amax's binary32 bit pattern read as int32: amax >= 0, so
its bits are non-negative integers that order exactly like the values, NaN patterns
above +inf; a NaN or Inf on any rank thus reaches every rank, and step 3 then
records NVFP4_ERR_NONFINITE in each rank's device status.

This module is plumbing: the arithmetic of steps 1, 3 and 4 runs in the library's
kernels, the exchange in the process group's backend (NCCL on GPUs).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass
class ShardWorkspace:
    """Device scalars one rank needs: its amax, the one-entry history and g."""
    amax: object
    history: object
    gscale: object

    @staticmethod
    def create(device):
        import torch

        z = lambda: torch.zeros(1, dtype=torch.float32, device=device)  # noqa: E731
        return ShardWorkspace(z(), z(), z())


class LibraryOps:
    """The four steps on the GPU through the C ABI, the exchange through torch.distributed."""

    def __init__(self, group=None):
        self.group = group

    def amax(self, x, ws, stream=None):
        from . import nvfp4_amax

        nvfp4_amax(x, ws.amax, stream)

    def all_reduce_max(self, ws):
        import torch
        import torch.distributed as dist

        dist.all_reduce(ws.amax.view(torch.int32), op=dist.ReduceOp.MAX, group=self.group)

    def tensor_scale(self, ws, stream=None):
        from . import nvfp4_amax_history_push

        nvfp4_amax_history_push(ws.history, ws.amax, ws.gscale, stream)

    def quantize(self, x, out, ws, stream=None):
        from . import nvfp4_quantize

        nvfp4_quantize(x, out, gscale_in=ws.gscale, stream=stream)


def quantize_row_shard(x_local, out, ws: ShardWorkspace, ops=None, stream=None):
    """Quantize this rank's rows `x_local` [rows_r, cols] into `out` with the tensor
    scale of the whole row-sharded tensor.  Every rank of the group must call it,
    in the same order as its other collectives.  `ops` defaults to LibraryOps()."""
    ops = ops if ops is not None else LibraryOps()
    ops.amax(x_local, ws, stream)
    ops.all_reduce_max(ws)
    ops.tensor_scale(ws, stream)
    ops.quantize(x_local, out, ws, stream)


def row_range(rows: int, rank: int, world: int):
    """Rows [start, stop) of `rank` when `rows` are split over `world` ranks as evenly
    as possible (the first rows % world ranks take one more)."""
    base, extra = divmod(rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)
