"""N-split (column-parallel) quantised linear over the ranks of a process group.

Each rank holds rows [n0, n1) of the packed codes, scales and zeros of W
([N, K]; one output feature per row) and computes y[:, n0:n1] = x . W'[n0:n1]^T
with ``wq_gemm`` on its own GPU; the slices are then gathered along N so every
rank holds the whole y.  The quantisation grid is per row (or per group of a
row), so a row shard of the quantised weight is exactly the quantisation of
the row shard: no exchange is needed inside the GEMV, only the gather of y.
The OPTQ paper's reproducibility summary (row "Hardware Specification") runs
the 3-bit OPT-175B model on two A6000 GPUs; this is the layout that splits such
a layer's weights between GPUs.

Shards are 32-row aligned (the GEMV's row tile) and of equal padded length, so
the gather is one all-gather of equal chunks.  The collective is
``torch.distributed.all_gather`` (NCCL between GPUs); the local product is any
callable ``local(x, codes, scales, zeros, n_rows) -> y_shard`` (``wq_gemm`` by
default), which lets the host logic run on CPU ranks over gloo as well.
"""
from __future__ import annotations

import torch


def shard_bounds(N: int, world: int, rank: int, align: int = 32):
    """Rows [n0, n1) of rank ``rank``: equal chunks of ceil(N / world) rows
    rounded up to ``align``; trailing ranks may hold fewer rows or none."""
    if world < 1 or not 0 <= rank < world or N < 1:
        raise ValueError("need N >= 1 and 0 <= rank < world")
    per = -(-N // world)
    per = -(-per // align) * align
    n0 = min(N, rank * per)
    return n0, min(N, n0 + per), per


def shard_rows(t, n0: int, n1: int):
    """Rows [n0, n1) of a row-major [N, ...] tensor (codes, scales or zeros),
    as a contiguous tensor; None stays None (symmetric grid)."""
    return None if t is None else t[n0:n1].contiguous()


def _wq_local(bits, group, K):
    import quantized_gemm_wq_b200 as wq

    def run(x, codes, scales, zeros, n_rows, out):
        return wq.wq_gemm(x, codes, scales, zeros, bits, group, n_rows, K, y=out)
    return run


class NSplitLinear:
    """One rank's part of a column-parallel quantised linear.

    ``codes``, ``scales``, ``zeros`` are the WHOLE quantised weight (every
    rank passes the same tensors; only rows [n0, n1) are kept), or, with
    ``sharded=True``, this rank's rows already.  ``__call__(x)`` returns the
    whole y [M, N] on every rank."""

    def __init__(self, codes, scales, zeros, N: int, K: int, bits: int, group: int, *, rank=None,
                 world=None, pg=None, sharded: bool = False, local=None):
        import torch.distributed as dist
        if rank is None or world is None:
            if dist.is_available() and dist.is_initialized():
                rank, world = dist.get_rank(pg), dist.get_world_size(pg)
            else:
                rank, world = 0, 1
        self.N, self.K, self.bits, self.group = N, K, bits, group
        self.rank, self.world, self.pg = rank, world, pg
        self.n0, self.n1, self.per = shard_bounds(N, world, rank)
        if sharded:
            self.codes, self.scales, self.zeros = codes, scales, zeros
        else:
            self.codes = shard_rows(codes, self.n0, self.n1)
            self.scales = shard_rows(scales, self.n0, self.n1)
            self.zeros = shard_rows(zeros, self.n0, self.n1)
        self.local = local if local is not None else _wq_local(bits, group, K)

    @property
    def rows(self) -> int:
        return self.n1 - self.n0

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        import torch.distributed as dist
        M = x.shape[0]
        chunk = torch.zeros((M, self.per), dtype=torch.bfloat16, device=x.device)
        if self.rows:
            if self.rows == self.per:
                self.local(x, self.codes, self.scales, self.zeros, self.rows, chunk)
            else:
                part = torch.empty((M, self.rows), dtype=torch.bfloat16, device=x.device)
                self.local(x, self.codes, self.scales, self.zeros, self.rows, part)
                chunk[:, :self.rows] = part
        if self.world == 1:
            return chunk[:, :self.N].contiguous()
        parts = [torch.empty_like(chunk) for _ in range(self.world)]
        dist.all_gather(parts, chunk, group=self.pg)
        return torch.cat(parts, dim=1)[:, :self.N].contiguous()
