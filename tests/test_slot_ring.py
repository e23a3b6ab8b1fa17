"""CPU checks of the pool's slot ring (round-robin slot assignment, host side) and of the
host-side argument checks of the pool-sharing calls ([notes] §6: slots are reused in
rotation; the retrieval stage hands the ranking node each request's slot id)."""

import ctypes
import threading

import pytest

from kv_cache_reuse_falcon_b200 import binding as ub


def test_slots_rotate_through_the_pool():
    r = ub.SlotRing(6)
    assert r.acquire(2) == [0, 1]
    assert r.acquire(3) == [2, 3, 4]
    r.release([0, 1])
    # the scan continues after the last slot handed out, then wraps
    assert r.acquire(2) == [5, 0]
    assert r.free_count() == 1
    r.release([2, 3, 4])
    assert r.acquire(4) == [1, 2, 3, 4]
    assert r.free_count() == 0


def test_acquire_takes_all_or_nothing():
    r = ub.SlotRing(4)
    r.acquire(3)
    with pytest.raises(ub.UnipinError) as e:
        r.acquire(2)
    assert e.value.code == -4            # UNIPIN_ERR_OUT_OF_RANGE
    assert r.free_count() == 1           # nothing was taken
    assert r.acquire(1) == [3]
    assert r.acquire(0) == []


def test_release_checks_every_id_first():
    r = ub.SlotRing(5)
    ids = r.acquire(3)                   # 0, 1, 2
    for bad in ([0, 3], [0, 0], [7], [-1], [1, 2, 4]):
        with pytest.raises(ub.UnipinError) as e:
            r.release(bad)
        assert e.value.code == -1        # UNIPIN_ERR_INVALID_ARG
        assert r.free_count() == 2       # nothing was freed
    r.release(ids)
    assert r.free_count() == 5
    with pytest.raises(ub.UnipinError):
        r.release([1])                   # already free


def test_ring_rejects_bad_sizes():
    with pytest.raises(ub.UnipinError):
        ub.SlotRing(0)
    r = ub.SlotRing(3)
    with pytest.raises(ub.UnipinError):
        r.acquire(-1)
    with pytest.raises(ub.UnipinError):
        r.acquire(4)


def test_concurrent_acquire_release_never_hands_out_a_slot_twice():
    S, threads, rounds = 64, 8, 400
    r = ub.SlotRing(S)
    held = set()
    lock = threading.Lock()
    errors = []

    def worker(seed):
        import random
        rnd = random.Random(seed)
        for _ in range(rounds):
            n = rnd.randint(1, 4)
            try:
                ids = r.acquire(n)
            except ub.UnipinError:
                continue                 # ring momentarily short of free slots
            with lock:
                if held & set(ids) or len(set(ids)) != n:
                    errors.append(ids)
                held.update(ids)
            with lock:
                held.difference_update(ids)
            r.release(ids)

    ts = [threading.Thread(target=worker, args=(i,)) for i in range(threads)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors
    assert r.free_count() == S


def test_share_calls_check_their_arguments_without_a_device():
    lib = ub.LIB
    desc = ub.KVPoolShare()
    pool = ub.KVPool()
    assert lib.unipin_kvpool_share_export(None, ctypes.byref(desc)) == -1
    assert lib.unipin_kvpool_share_export(ctypes.byref(pool), ctypes.byref(desc)) == -1    # null tensors
    assert lib.unipin_kvpool_share_open(ctypes.byref(desc), None) == -1
    assert lib.unipin_kvpool_share_open(ctypes.byref(desc), ctypes.byref(pool)) == -1      # zero shape
    assert lib.unipin_kvpool_share_close(ctypes.byref(desc), ctypes.byref(pool)) == -1     # nothing open
    assert ctypes.sizeof(ub.KVPoolShare) == 176    # handles, offsets, shape, dtype and the two scales
    with pytest.raises(ValueError):
        ub.SharedPool(b"short")
