"""Data-parallel plumbing: one process per GPU, each owning a contiguous shard
of independent units.

TurboQuant's write and read halves are row-local (quantize, dequant) or local
to one (batch, kv head) set (the logits of a set read only that set's keys and
queries): each row is normalised, rotated, bucketed and projected on its own
(0h-n0 "ICLR 2026論文解説: TurboQuant", "Step 1: PolarQuant" and "Step 2: QJL"),
and the estimate of <q, k> reads only q and that key's packed row (Qiita
TurboQuant explainer, "Stage 2: QJL").  A multi-GPU job therefore splits the
global batch of sequences into contiguous shards, one per rank, and needs no
collective on the data path: every rank quantizes, scores and dequantizes its
own sequences.  The collectives here are only for timing (a barrier and the
max of the per-rank device times).

The functions take the world size and rank explicitly so the host logic can be
tested with gloo ranks on the CPU.
"""

from __future__ import annotations

from dataclasses import dataclass


def shard(n_units: int, world_size: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced shard [lo, hi) of n_units for this rank: the first
    n_units % world_size ranks take one unit more.  Shards are disjoint and
    cover [0, n_units) in rank order."""
    if world_size < 1 or not 0 <= rank < world_size:
        raise ValueError(f"rank {rank} outside a world of {world_size}")
    if n_units < 0:
        raise ValueError("n_units must be >= 0")
    base, extra = divmod(n_units, world_size)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


@dataclass(frozen=True)
class DecodeShard:
    """One rank's part of a decode step over a global batch of sequences.

    K and V rows are laid out [batch, kv_heads, ctx] and queries
    [batch, q_heads], so a contiguous range of sequences is a contiguous range
    of rows in each."""

    global_batch: int
    seq_lo: int
    seq_hi: int
    kv_heads: int
    q_heads: int
    ctx: int

    @property
    def batch(self) -> int:
        return self.seq_hi - self.seq_lo

    @property
    def kv_rows(self) -> tuple[int, int]:
        per = self.kv_heads * self.ctx
        return self.seq_lo * per, self.seq_hi * per

    @property
    def q_rows(self) -> tuple[int, int]:
        return self.seq_lo * self.q_heads, self.seq_hi * self.q_heads

    @property
    def n_sets(self) -> int:
        return self.batch * self.kv_heads


def decode_shard(batch_per_rank: int, world_size: int, rank: int, kv_heads: int, q_heads: int,
                 ctx: int) -> DecodeShard:
    """Weak scaling: the global batch is world_size * batch_per_rank sequences
    and rank r owns sequences [r * batch_per_rank, (r + 1) * batch_per_rank)."""
    if q_heads % kv_heads:
        raise ValueError("q_heads must be a multiple of kv_heads")
    gb = world_size * batch_per_rank
    lo, hi = shard(gb, world_size, rank)
    return DecodeShard(gb, lo, hi, kv_heads, q_heads, ctx)


def barrier(world_size: int) -> None:
    if world_size > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world_size: int, v: float, device=None) -> float:
    """The largest of the ranks' values (device times are combined this way,
    never by wall clock).  device: where the reduction tensor lives (a CUDA
    device for NCCL, None = CPU for gloo)."""
    if world_size == 1:
        return float(v)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(world_size: int, v: int, device=None) -> int:
    """Total of an integer count over ranks (units processed, launches)."""
    if world_size == 1:
        return int(v)
    import torch
    import torch.distributed as dist
    t = torch.tensor([int(v)], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())
