"""Multi-rank host logic on CPU (gloo, world size 2): users are split across ranks with
no exchange on the data path; gathering the per-rank results reproduces the
single-rank result exactly."""

import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from kv_cache_reuse_falcon_b200 import synth
from kv_cache_reuse_falcon_b200.shard import rank_seed, segment_cost, shard_segments


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        past = np.array([40, 7, 90, 0, 33, 64], np.int32)
        cand = np.array([5, 9, 3, 4, 20, 1], np.int32)
        batch = synth.make_prefill(77, past, cand, 2, 16)
        mine = shard_segments(past, cand, world)[rank]
        outs = {}
        for b in mine:
            lo, hi = int(batch.cu_seqlens[b]), int(batch.cu_seqlens[b + 1])
            outs[int(b)] = oracle.prefill(batch.q[lo:hi], batch.k[lo:hi], batch.v[lo:hi],
                                          [0, hi - lo], [int(past[b])])
        gathered = [None] * world
        dist.all_gather_object(gathered, outs)   # result collection only, after the compute
        if rank == 0:
            merged = {}
            for g in gathered:
                merged.update(g)
            full = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
            ok = sorted(merged) == list(range(len(past)))
            for b, o in merged.items():
                lo, hi = int(batch.cu_seqlens[b]), int(batch.cu_seqlens[b + 1])
                ok = ok and np.array_equal(o, full[lo:hi])
            q.put(ok)
    finally:
        dist.destroy_process_group()


def test_sharded_users_reassemble_to_the_unsharded_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    assert q.get(timeout=5) is True


def test_shard_plan_covers_every_user_once_and_balances():
    rng = np.random.default_rng(0)
    past = rng.integers(32, 4097, 256)
    cand = rng.integers(50, 2001, 256)
    for world in (1, 2, 4, 8):
        parts = shard_segments(past, cand, world)
        allidx = np.sort(np.concatenate(parts))
        assert np.array_equal(allidx, np.arange(256))
        loads = [segment_cost(past[p], cand[p]).sum() for p in parts]
        assert max(loads) <= 1.05 * (sum(loads) / world) + segment_cost(past, cand).max()


def test_rank_seeds_differ():
    assert len({rank_seed(5, r) for r in range(8)}) == 8


def _report_worker(rank, world, port, q):
    from kv_cache_reuse_falcon_b200.shard import combine_rank_results
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = {"step_ms": 10.0 + rank, "prefill_ms": 5.0 - rank, "e2e_ms": 20.0 * (rank + 1)}
        counts = {"candidates": 1000.0 * (rank + 1), "flops": 1e12}
        t, c = combine_rank_results(times, counts, device="cpu")
        q.put((rank, t, c))
    finally:
        dist.destroy_process_group()


def test_cross_rank_report_takes_max_times_and_summed_work():
    """The multi-GPU benchmark's reduction: the job's time is its slowest rank's, its work the sum."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_report_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, c in res:
        assert t == {"step_ms": 11.0, "prefill_ms": 5.0, "e2e_ms": 40.0}
        assert c == {"candidates": 3000.0, "flops": 2e12}


def test_single_process_report_is_unchanged():
    from kv_cache_reuse_falcon_b200.shard import combine_rank_results
    t, c = combine_rank_results({"a": 1.5}, {"n": 3}, group=False)
    assert t == {"a": 1.5} and c == {"n": 3}
