"""A pool shared across processes ([notes] §6: the retrieval process exports
CUDA IPC handles of its pool, the ranking process maps the same device memory
and reads the request's slot there).  The parent writes the pool through
unipin_kvpool_write into slots from a SlotRing and exports it; a child
process (spawned, its own CUDA context) opens it, reads the rows back and runs
the rank decode over it.  Both must see the same bytes and get the same output
bits; the output must also match the oracle."""

import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

from kv_cache_reuse_falcon_b200 import synth

pytestmark = pytest.mark.gpu

L, S, H, N_CAP, D, LAYER = 2, 6, 2, 300, 64, 1
PAST, CAND, SEED = [300, 17, 129], [40, 1, 77], 8100


def _inputs():
    rng = np.random.Generator(np.random.PCG64(SEED))
    d = synth.make_decode(SEED, PAST, CAND, H, D, n_slots=S, rng=rng)
    ks, vs = synth.pool_rows(rng, PAST, H, D)
    return d, ks, vs


def _child(desc_path: str, slots, out_path: str):
    import numpy as np
    import torch
    from kv_cache_reuse_falcon_b200 import binding as ub
    from tests.gpu_helpers import DevDecode
    torch.cuda.init()
    with open(desc_path, "rb") as f:
        shared = ub.SharedPool(f.read())
    d, _, _ = _inputs()
    d.slot_ids[:] = slots
    dd = DevDecode(d)
    out = ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, shared.k, shared.v, LAYER, dd.max_k,
                              out_fp32=True, workspace=None)
    torch.cuda.synchronize()
    rows_k = [shared.k[LAYER, s, :, :n].view(torch.int16).cpu().numpy() for s, n in zip(slots, PAST)]
    rows_v = [shared.v[LAYER, s, :, :n].view(torch.int16).cpu().numpy() for s, n in zip(slots, PAST)]
    np.savez(out_path, out=out.cpu().numpy(), **{"k%d" % i: a for i, a in enumerate(rows_k)},
             **{"v%d" % i: a for i, a in enumerate(rows_v)})
    shared.close()


def test_pool_shared_with_another_process(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from kv_cache_reuse_falcon_b200 import binding as ub
    from tests.gpu_helpers import DevDecode, host_pool_layer, nan_pool, parity, to_dev_bf16, to_dev_i32

    d, ks, vs = _inputs()
    ring = ub.SlotRing(S)
    ring.acquire(2)                                  # earlier requests hold slots 0, 1
    slots = ring.acquire(len(PAST))                  # this batch: 2, 3, 4
    d.slot_ids[:] = slots
    pk, pv = nan_pool(L, S, H, N_CAP, D)
    # the retrieval side: past K/V packed [T, H, D] per request, written into the slots
    k_tok = np.concatenate([kb.transpose(1, 0, 2) for kb in ks])
    v_tok = np.concatenate([vb.transpose(1, 0, 2) for vb in vs])
    cu = np.concatenate([[0], np.cumsum(PAST)]).astype(np.int32)
    ub.kvpool_write(pk, pv, LAYER, to_dev_bf16(k_tok), to_dev_bf16(v_tok), to_dev_i32(cu),
                    to_dev_i32(PAST), to_dev_i32(slots), max(PAST))
    dd = DevDecode(d)
    local = ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, LAYER, dd.max_k,
                                out_fp32=True, workspace=None)
    torch.cuda.synchronize()

    desc_path = str(tmp_path / "pool.ipc")
    with open(desc_path, "wb") as f:
        f.write(ub.kvpool_share_export(pk, pv))      # the file the ranking process opens
    out_path = str(tmp_path / "child.npz")
    ctx = mp.get_context("spawn")
    p = ctx.Process(target=_child, args=(desc_path, list(slots), out_path))
    p.start()
    p.join(180)
    if p.is_alive():
        p.terminate()
        p.join(10)
        pytest.fail("child process did not finish")
    assert p.exitcode == 0 and os.path.exists(out_path)
    got = np.load(out_path)
    for i, (s, n) in enumerate(zip(slots, PAST)):
        assert np.array_equal(got["k%d" % i].view(np.uint16), ks[i])
        assert np.array_equal(got["v%d" % i].view(np.uint16), vs[i])
    assert np.array_equal(got["out"], local.cpu().numpy())
    hk, hv = host_pool_layer(L, S, H, N_CAP, D, LAYER, slots, PAST, ks, vs)
    ref = oracle.decode(d.q, d.k, d.v, d.cu_seqlens, d.slot_ids, d.past_lens, hk, hv, 0)
    parity(got["out"], ref, "decode over the shared pool")
    ring.release(slots)
