"""Sharding one indexer job over ranks (one process per GPU).

Queries are independent once the keys are present, so a job splits without
any exchange inside the indexer: every rank holds the keys its queries see
and runs the one-GPU library on its own queries.  The pages describe no
parallelism; the split follows the causal work of each query instead of the
query count, because a query at position p scores min(p+1, m*B) candidate
keys in the refinement stage and (p+1)/B pooled blocks in the coarse stage,
so equal query counts would leave the ranks holding late queries slowest.

* One sequence (prefill, a chunk of a long prefix, compressed keys): each rank
  takes a contiguous range of queries, the ranges cut where the running sum of
  work crosses r/world of the total.
* Several sequences (decode): each rank takes a contiguous range of whole
  sequences, cut the same way by per-sequence work, so a sequence's keys live
  on one GPU only.

Contiguous ranges keep a shard's q, w and n_visible a plain slice of the
job's tensors, so a rank calls the library on views, and the assembled index
tensor [batch, Q, top_k] is the concatenation of the shards' outputs in rank
order.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Shard:
    """Rows [seq0, seq1) x queries [t0, t1) of a [batch, Q] job."""
    seq0: int
    seq1: int
    t0: int
    t1: int

    @property
    def rows(self) -> int:
        return max(0, self.seq1 - self.seq0) * max(0, self.t1 - self.t0)


def query_work(n_visible: np.ndarray, block_size: int, top_m: int) -> np.ndarray:
    """Work of each query of the HISA indexer, in keys scored: the candidate
    keys of the refinement stage (min(n_t, top_m * B) up to the partial
    current block) plus the pooled blocks the coarse stage scores.  Queries
    that see nothing cost one unit (they still occupy a job slot)."""
    n = np.asarray(n_visible, np.int64)
    B, m = int(block_size), int(top_m)
    c = np.where(n > 0, (n - 1) // B, 0)
    cand = np.where(n > 0, np.minimum(c, m - 1) * B + (n - c * B), 0)
    return np.maximum(cand + c, 1)


def cut_points(work: np.ndarray, world: int) -> list[int]:
    """world+1 cut points 0 = x_0 <= ... <= x_world = len(work) such that the
    ranges [x_r, x_{r+1}) hold about equal work: x_r is one past the first
    index whose inclusive running sum reaches r/world of the total.  Each range's work is
    at most total/world + max(work)."""
    w = np.asarray(work, np.float64).ravel()
    if world < 1:
        raise ValueError("world must be >= 1")
    csum = np.cumsum(w)
    total = csum[-1] if len(csum) else 0.0
    cuts = [0]
    for r in range(1, world):
        cuts.append(int(np.searchsorted(csum, total * r / world, side="left")) + 1 if len(csum) else 0)
        cuts[-1] = min(max(cuts[-1], cuts[-2]), len(w))
    cuts.append(len(w))
    return cuts


def shard_job(n_visible: np.ndarray, block_size: int, top_m: int, world: int) -> list[Shard]:
    """Shards of a [batch, Q] job, one per rank, in rank order."""
    n = np.asarray(n_visible)
    batch, Q = n.shape
    work = query_work(n, block_size, top_m)
    if batch == 1:
        cuts = cut_points(work[0], world)
        return [Shard(0, 1, cuts[r], cuts[r + 1]) for r in range(world)]
    cuts = cut_points(work.sum(axis=1), world)
    return [Shard(cuts[r], cuts[r + 1], 0, Q) for r in range(world)]


def shard_work(n_visible: np.ndarray, block_size: int, top_m: int, shards: list[Shard]) -> list[int]:
    """Total work of each shard (for balance checks and reporting)."""
    work = query_work(n_visible, block_size, top_m)
    return [int(work[s.seq0:s.seq1, s.t0:s.t1].sum()) for s in shards]
