"""GPU parity with grouped-query heads ([notes] §6: the pool holds "KV heads").

Queries have H heads, keys/values H_kv = H / G; query head h reads key/value
head h // G.  The prefill (with its fused pool write), both rank-decode paths
(the small-candidate kernel, where the G query heads of a key/value head share
one sweep of the history, and the many-candidate engine) and the gradients are
compared with the fp64 oracle on the same seeded inputs, over NaN-poisoned pools.
"""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth
from tests.gpu_helpers import bf16_tensor_bits, nan_pool, parity, to_dev_bf16, to_dev_i32
from tests.test_gpu_backward import grad_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ub():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_reuse_falcon_b200 import binding
    return binding


def gqa_prefill(seed, past, cand, H, Hkv, D):
    rng = np.random.Generator(np.random.PCG64(seed))
    cu = synth.cu_from_lens(np.array(past) + np.array(cand))
    T = int(cu[-1])
    q = synth.normal_bf16(rng, (T, H, D))
    k = synth.normal_bf16(rng, (T, Hkv, D))
    v = synth.normal_bf16(rng, (T, Hkv, D))
    return cu, np.array(past, np.int32), q, k, v, rng


@pytest.mark.parametrize("H,Hkv,D", [(8, 2, 64), (4, 1, 128), (6, 3, 32)])
def test_gqa_prefill_with_pool_write(ub, H, Hkv, D):
    past, cand = [200, 0, 70, 513], [40, 9, 1, 130]
    S, n_cap, L = 6, 700, 2
    cu, pl, q, k, v, _ = gqa_prefill(7000 + H + D, past, cand, H, Hkv, D)
    slots = np.array([5, 0, 3, 1], np.int32)
    pk, pv = nan_pool(L, S, Hkv, n_cap, D)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ub.masked_prefill_attn(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), to_dev_i32(cu), to_dev_i32(pl),
                                 int(np.diff(cu).max()), out_fp32=True, pool_k=pk, pool_v=pv,
                                 slot_ids=to_dev_i32(slots), layer=1, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    parity(out.cpu().numpy(), oracle.prefill(q, k, v, cu, pl), "gqa prefill H=%d Hkv=%d D=%d" % (H, Hkv, D))
    hk = np.full((L, S, Hkv, n_cap, D), synth.BF16_NAN, dtype=np.uint16)
    hv = hk.copy()
    oracle.pool_write(hk, hv, 1, k, v, cu, pl, slots)
    assert bf16_tensor_bits(pk).tobytes() == hk.tobytes()
    assert bf16_tensor_bits(pv).tobytes() == hv.tobytes()


DECODE = [
    # (cand lens, H, Hkv, D): small-k kernel while max_k * G <= 64, the engine beyond
    ([16, 3, 12, 1], 8, 2, 64),       # 16 * 4 = 64 columns
    ([1, 1, 1, 1], 8, 1, 64),
    ([16, 9, 5, 16], 4, 1, 128),
    ([7, 2, 5, 3], 16, 2, 128),       # 7 * 8 = 56 columns, G = 8
    ([30, 12, 5, 32], 4, 1, 128),     # 32 * 4 > 64: many-candidate engine
    ([100, 40, 3, 77], 4, 2, 64),
]


@pytest.mark.parametrize("case", range(len(DECODE)))
@pytest.mark.parametrize("mode", ["none", "split"])
def test_gqa_rank_decode(ub, case, mode):
    cand, H, Hkv, D = DECODE[case]
    past = [2048, 0, 129, 1000]
    S, n_cap, layer = 8, 2048, 1
    rng = np.random.Generator(np.random.PCG64(7100 + case))
    cu = synth.cu_from_lens(np.array(cand))
    Tc = int(cu[-1])
    qc = synth.normal_bf16(rng, (Tc, H, D))
    kc = synth.normal_bf16(rng, (Tc, Hkv, D))
    vc = synth.normal_bf16(rng, (Tc, Hkv, D))
    slots = rng.permutation(S)[:4].astype(np.int32)
    pk, pv = nan_pool(layer + 1, S, Hkv, n_cap, D)
    hk = np.full((1, S, Hkv, n_cap, D), synth.BF16_NAN, dtype=np.uint16)
    hv = hk.copy()
    for s, n in zip(slots, past):
        kr, vr = synth.normal_bf16(rng, (Hkv, n, D)), synth.normal_bf16(rng, (Hkv, n, D))
        if n:
            pk[layer, s, :, :n] = to_dev_bf16(kr)
            pv[layer, s, :, :n] = to_dev_bf16(vr)
            hk[0, s, :, :n], hv[0, s, :, :n] = kr, vr
    ws = None
    if mode == "split":
        nbytes = ub.rank_decode_workspace_size(4, H, D, max(cand), Tc, n_cap, H_kv=Hkv)
        ws = torch.empty(nbytes // 4 + 4, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ub.rank_decode_attn(to_dev_bf16(qc), to_dev_bf16(kc), to_dev_bf16(vc), to_dev_i32(cu), to_dev_i32(slots),
                              to_dev_i32(past), pk, pv, layer, max(cand), out_fp32=True, workspace=ws,
                              dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    ref = oracle.decode(qc, kc, vc, cu, slots, np.array(past, np.int32), hk, hv, 0)
    parity(out.cpu().numpy(), ref, "gqa decode case %d %s" % (case, mode))


@pytest.mark.parametrize("H,Hkv,D", [(4, 2, 64), (8, 1, 32), (4, 2, 128)])
def test_gqa_backward(ub, H, Hkv, D):
    past, cand = [200, 37, 300], [77, 5, 130]
    cu, pl, q, k, v, rng = gqa_prefill(7200 + H, past, cand, H, Hkv, D)
    g = synth.normal_bf16(rng, q.shape)
    dq_, dk_, dv_, cu_d, pl_d = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), to_dev_i32(cu), to_dev_i32(pl)
    T = q.shape[0]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    ms = int(np.diff(cu).max())
    out = ub.masked_prefill_attn(dq_, dk_, dv_, cu_d, pl_d, ms, out_fp32=False, lse=lse, dev_status=status)
    gq, gk, gv = ub.masked_prefill_bwd(dq_, dk_, dv_, out, to_dev_bf16(g), lse, cu_d, pl_d, ms, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    assert tuple(gk.shape) == (T, Hkv, D)
    rq, rk, rv = oracle.prefill_bwd(q, k, v, g, cu, pl)
    grad_parity(gq.cpu().numpy(), rq, "gqa dq")
    grad_parity(gk.cpu().numpy(), rk, "gqa dk")
    grad_parity(gv.cpu().numpy(), rv, "gqa dv")
