"""GPU parity of the small-candidate-count rank decode (k <= 128 per request).

Requests with at most 128 candidates (head dim 64 or 128) take the kernel that
puts the pool keys on the MMA's M dimension and splits each request's key
range over several thread blocks.  Every case compares the fp32 output with
the fp64 oracle on the same seeded inputs over a NaN-poisoned pool (a stray
read of a row at or beyond a request's history length shows up as NaN):
max-abs <= 1e-2, relative L2 <= 2e-3.
"""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth
from tests.gpu_helpers import (DevDecode, DevPrefill, bf16_tensor_bits, fill_pool_rows, host_pool_layer,
                               nan_pool, parity, to_dev_i32)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ub():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_reuse_falcon_b200 import binding
    return binding


def setup_decode(seed, past, cand, H, D, S, n_cap, L=2, layer=1):
    rng = np.random.Generator(np.random.PCG64(seed))
    d = synth.make_decode(seed, past, cand, H, D, n_slots=S, rng=rng)
    ks, vs = synth.pool_rows(rng, past, H, D)
    pk, pv = nan_pool(L, S, H, n_cap, D)
    fill_pool_rows(pk, pv, layer, d.slot_ids, past, ks, vs)
    hk, hv = host_pool_layer(L, S, H, n_cap, D, layer, d.slot_ids, past, ks, vs)
    return d, DevDecode(d), pk, pv, hk, hv


def workspace_for(ub, mode, d, H, D, n_cap):
    if mode == "none":
        return None
    if mode == "counter":
        return torch.empty(64, dtype=torch.float32, device="cuda")        # 256 bytes: no split
    nbytes = ub.rank_decode_workspace_size(d.R, H, D, int(d.cand_lens.max()), int(d.cu_seqlens[-1]), n_cap)
    return torch.empty(nbytes // 4 + 4, dtype=torch.float32, device="cuda")


def decode(ub, dd, pk, pv, layer, ws, out_fp32=True):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, layer, dd.max_k,
                              out_fp32=out_fp32, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    return out


# ragged histories: none, one key, around the 128-key tile edge, several tiles, full capacity
PAST = [2048, 0, 1, 127, 128, 129, 1000, 777]

SMALL_K_CASES = [
    # (candidates per request, H, D, n_cap)
    ([1] * 8, 2, 64, 2048),                              # the S=1 retrieval step over the pool
    ([16] * 8, 2, 64, 2048),
    ([64] * 8, 2, 64, 2048),
    ([128] * 8, 2, 64, 2048),
    ([3, 16, 1, 9, 14, 2, 16, 7], 2, 64, 2048),         # ragged k within one padding class
    ([17, 33, 1, 64, 50, 0, 20, 64], 3, 64, 2048),       # padded to 64, a request with no candidate
    ([100, 65, 128, 1, 90, 127, 70, 66], 2, 64, 2048),   # padded to 128
    ([1] * 8, 2, 128, 2048),
    ([16] * 8, 2, 128, 2048),
    ([40, 64, 3, 17, 64, 33, 1, 60], 2, 128, 2048),
    ([128, 100, 65, 1, 128, 7, 90, 128], 2, 128, 2048),
]


@pytest.mark.parametrize("case", range(len(SMALL_K_CASES)))
@pytest.mark.parametrize("mode", ["none", "counter", "split"])
def test_small_k_decode_matches_oracle(ub, case, mode):
    cand, H, D, n_cap = SMALL_K_CASES[case]
    S = 12
    d, dd, pk, pv, hk, hv = setup_decode(5000 + case, PAST, cand, H, D, S, n_cap)
    ws = workspace_for(ub, mode, d, H, D, n_cap)
    out = decode(ub, dd, pk, pv, 1, ws).cpu().numpy()
    ref = oracle.decode(d.q, d.k, d.v, d.cu_seqlens, d.slot_ids, d.past_lens, hk, hv, 0)
    parity(out, ref, "small-k decode case %d mode %s" % (case, mode))


def test_small_k_split_is_used_and_repeats_bit_exactly(ub):
    """With a full workspace the pool sweep is split (the split is re-zeroed every call): two
    calls give identical bits, and the unsplit result agrees within tolerance."""
    cand, H, D, n_cap = [16] * 8, 2, 64, 2048
    d, dd, pk, pv, hk, hv = setup_decode(5100, PAST, cand, H, D, 12, n_cap)
    nbytes = ub.rank_decode_workspace_size(8, H, D, 16, int(d.cu_seqlens[-1]), n_cap)
    assert nbytes > 512
    ws = workspace_for(ub, "split", d, H, D, n_cap)
    o1 = decode(ub, dd, pk, pv, 1, ws)
    o2 = decode(ub, dd, pk, pv, 1, ws)
    assert torch.equal(o1, o2)
    o_static = decode(ub, dd, pk, pv, 1, None)
    o_counter = decode(ub, dd, pk, pv, 1, workspace_for(ub, "counter", d, H, D, n_cap))
    assert torch.equal(o_static, o_counter), "static striding and the work counter differ"
    parity(o1.cpu().numpy(), o_static.cpu().numpy().astype(np.float64), "split vs unsplit")


def test_small_k_bf16_output_is_rounded_fp32_output(ub):
    cand, H, D, n_cap = [5, 16, 64, 1, 33, 40, 2, 9], 2, 128, 2048
    d, dd, pk, pv, _, _ = setup_decode(5200, PAST, cand, H, D, 12, n_cap)
    for mode in ("none", "split"):
        ws = workspace_for(ub, mode, d, H, D, n_cap)
        o32 = decode(ub, dd, pk, pv, 1, ws, out_fp32=True)
        o16 = decode(ub, dd, pk, pv, 1, ws, out_fp32=False)
        assert np.array_equal(bf16_tensor_bits(o16), synth.f32_to_bf16_bits(o32.cpu().numpy()))


def test_small_k_decode_equals_prefill_candidate_rows(ub):
    """Candidates decoded over the pool the prefill wrote score what the prefill gave them."""
    past, cand = [300, 0, 129, 1000, 2048, 64], [16, 4, 1, 9, 16, 12]
    H, D, L, S, n_cap = 2, 64, 2, 8, 2048
    batch = synth.make_prefill(5300, past, cand, H, D, n_slots=S)
    dp = DevPrefill(batch)
    pk, pv = nan_pool(L, S, H, n_cap, D)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pre = ub.masked_prefill_attn(dp.q, dp.k, dp.v, dp.cu, dp.past, dp.max_seqlen, out_fp32=True, pool_k=pk,
                                 pool_v=pv, slot_ids=dp.slots, layer=1, dev_status=status)
    cidx = np.concatenate([np.arange(batch.cu_seqlens[b] + past[b], batch.cu_seqlens[b + 1])
                           for b in range(len(past))])
    d = synth.DecodeBatch(H, D, batch.past_lens, batch.cand_lens, synth.cu_from_lens(np.array(cand)),
                          batch.slot_ids, batch.q[cidx], batch.k[cidx], batch.v[cidx])
    for mode in ("none", "split"):
        dec = decode(ub, DevDecode(d), pk, pv, 1, workspace_for(ub, mode, d, H, D, n_cap))
        assert torch.isfinite(dec).all()
        pre_c = pre[torch.from_numpy(cidx).cuda()]
        parity(dec.cpu().numpy(), pre_c.cpu().numpy().astype(np.float64), "prefill vs small-k decode " + mode)
    ref = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, tokens=cidx)
    parity(dec.cpu().numpy(), ref, "small-k decode vs oracle prefill rows")


def test_small_k_request_out_of_range_gives_zeros_and_status(ub):
    """A request whose slot id is out of range: status OUT_OF_RANGE, its rows are zeros, the other
    requests are still scored."""
    cand, H, D, n_cap = [16, 8, 16], 2, 64, 1024
    past = [1000, 300, 129]
    for mode in ("none", "split"):
        d, dd, pk, pv, hk, hv = setup_decode(5400, past, cand, H, D, 4, n_cap)
        bad = d.slot_ids.copy()
        bad[1] = 9
        dd.slots = to_dev_i32(bad)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = torch.full((int(d.cu_seqlens[-1]), H, D), float("nan"), device="cuda")
        ws = workspace_for(ub, mode, d, H, D, n_cap)
        ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, 1, dd.max_k, out=out,
                            out_fp32=True, workspace=ws, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == -4
        o = out.cpu().numpy()
        lo, hi = int(d.cu_seqlens[1]), int(d.cu_seqlens[2])
        assert np.count_nonzero(o[lo:hi]) == 0
        keep = np.r_[0:lo, hi:o.shape[0]]
        ref = oracle.decode(d.q, d.k, d.v, d.cu_seqlens, d.slot_ids, d.past_lens, hk, hv, 0, tokens=keep)
        parity(o[keep], ref, "valid requests next to a bad one (%s)" % mode)
