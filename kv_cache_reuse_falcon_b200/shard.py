"""Host-side sharding of independent users across ranks (no collective on the data path).

Users (segments) and rank-decode requests are independent: a row's output
depends only on its own segment ([notes] §3: candidates share one position
and never see each other, so scores do not depend on batch composition).  A
multi-GPU run therefore splits users across ranks; each rank owns its pool
replica, as each retrieval replica owns its pool ([notes] §6).
"""

from __future__ import annotations

import heapq
from typing import List

import numpy as np


def segment_cost(n_past, n_cand):
    """Mask-effective score entries of one segment: causal past n(n+1)/2 plus k(n+1)."""
    n = np.asarray(n_past, dtype=np.float64)
    k = np.asarray(n_cand, dtype=np.float64)
    return n * (n + 1) / 2 + k * (n + 1)


def shard_segments(past_lens, cand_lens, world_size: int) -> List[np.ndarray]:
    """Longest-processing-time split of segments over ranks; returns sorted index arrays per rank."""
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    cost = segment_cost(past_lens, cand_lens)
    order = np.argsort(-cost, kind="stable")
    heap = [(0.0, r) for r in range(world_size)]
    parts = [[] for _ in range(world_size)]
    for idx in order:
        load, r = heapq.heappop(heap)
        parts[r].append(int(idx))
        heapq.heappush(heap, (load + float(cost[idx]), r))
    return [np.array(sorted(p), dtype=np.int64) for p in parts]


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank` in a weak-scaling run: every rank draws its own batch of users."""
    return int(base_seed) + 7919 * int(rank)


def combine_rank_results(times, counts, group=None, device=None):
    """Whole-job numbers of a weak-scaling run from every rank's own numbers.

    times:  dict name -> this rank's duration (ms); the job takes as long as its
            slowest rank, so each becomes the maximum over ranks.
    counts: dict name -> this rank's work (candidates scored, FLOPs, bytes); each
            becomes the sum over ranks.
    group:  a torch.distributed process group (None: the default group), or
            False for a single-process run (returned unchanged).
    device: where the reduction tensors live (a CUDA device for NCCL, CPU for gloo).
    Every rank must call this with the same keys, in the same order.
    """
    if group is False:
        return dict(times), dict(counts)
    import torch
    import torch.distributed as dist
    tk, ck = list(times), list(counts)
    t = torch.tensor([float(times[k]) for k in tk], dtype=torch.float64, device=device)
    c = torch.tensor([float(counts[k]) for k in ck], dtype=torch.float64, device=device)
    if t.numel():
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    if c.numel():
        dist.all_reduce(c, op=dist.ReduceOp.SUM, group=group)
    return dict(zip(tk, t.tolist())), dict(zip(ck, c.tolist()))
