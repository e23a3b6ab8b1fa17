"""GPU vs oracle parity for the masked prefill, the pool write and the rank decode.

Every case feeds the same seeded bf16 inputs to the CUDA path (through the C
ABI) and to the fp64 CPU oracle, and compares the fp32 outputs element by
element: max-abs <= 1e-2 and relative L2 <= 2e-3.  Index and byte work (the
pool write, slot addressing) must be bit-exact.  Sizes span several 128-row
tiles with ragged tails; full-size workloads compare sampled rows.
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


def run_prefill(ub, dp: DevPrefill, out_fp32=True, pool=None, slots=None, layer=0):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kw = {}
    if pool is not None:
        kw = dict(pool_k=pool[0], pool_v=pool[1], slot_ids=slots, layer=layer)
    out = ub.masked_prefill_attn(dp.q, dp.k, dp.v, dp.cu, dp.past, dp.max_seqlen, out_fp32=out_fp32,
                                 dev_status=status, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    return out


PREFILL_CASES = [
    # (past lens, cand lens, H, D)
    ([64, 64], [16, 16], 2, 32),                 # tiny workload shape
    ([200, 37, 300], [77, 5, 260], 2, 64),       # ragged tails, several tiles
    ([128, 256], [128, 1], 2, 64),               # tile-aligned past
    ([1, 0, 129, 5], [0, 7, 3, 300], 1, 64),     # n=1, n=0, k=0
    ([300, 17], [100, 140], 2, 128),             # D = 128
    ([90, 513], [40, 33], 3, 32),                # D = 32, several tiles
]


@pytest.mark.parametrize("case", range(len(PREFILL_CASES)))
def test_prefill_matches_oracle(ub, case):
    past, cand, H, D = PREFILL_CASES[case]
    batch = synth.make_prefill(1000 + case, past, cand, H, D)
    dp = DevPrefill(batch)
    out = run_prefill(ub, dp).cpu().numpy()
    ref = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    parity(out, ref, "prefill case %d" % case)


def test_prefill_bf16_output_is_rounded_fp32_output(ub):
    batch = synth.make_prefill(1100, [200, 37], [77, 90], 2, 64)
    dp = DevPrefill(batch)
    o32 = run_prefill(ub, dp, out_fp32=True)
    o16 = run_prefill(ub, dp, out_fp32=False)
    assert torch.equal(o16.view(torch.int16), o32.to(torch.bfloat16).view(torch.int16))


def test_prefill_empty_segments_and_edges(ub):
    # empty segment, a segment of one past token, one of one candidate
    batch = synth.make_prefill(1200, [0, 1, 0, 130], [0, 0, 1, 0], 2, 64)
    dp = DevPrefill(batch)
    out = run_prefill(ub, dp).cpu().numpy()
    ref = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    parity(out, ref, "edges")
    v = synth.bf16_bits_to_f64(batch.v)
    # closed forms: a lone past token and a lone candidate return their own value
    np.testing.assert_allclose(out[0], v[0], atol=1e-6, rtol=0)
    np.testing.assert_allclose(out[1], v[1], atol=1e-6, rtol=0)


# -------------------------------------------------------------------- pool write

def test_kvpool_write_bit_exact_on_nan_poisoned_pool(ub):
    past, cand = [5, 0, 130, 64, 200], [3, 4, 1, 0, 9]
    H, D, L, S, n_cap = 2, 64, 3, 9, 256
    batch = synth.make_prefill(1300, past, cand, H, D, n_slots=S)
    dp = DevPrefill(batch)
    pk, pv = nan_pool(L, S, H, n_cap, D)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ub.kvpool_write(pk, pv, 2, dp.k, dp.v, dp.cu, dp.past, dp.slots, dp.max_past, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    hk = np.full((L, S, H, n_cap, D), synth.BF16_NAN, dtype=np.uint16)
    hv = hk.copy()
    oracle.pool_write(hk, hv, 2, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, batch.slot_ids)
    assert bf16_tensor_bits(pk).tobytes() == hk.tobytes()
    assert bf16_tensor_bits(pv).tobytes() == hv.tobytes()


@pytest.mark.parametrize("D", [128, 64, 32])
def test_fused_prefill_pool_write_bit_exact(ub, D):
    """The prefill stores each segment's past K/V tiles into its slot as it loads them: whole
    64-key tiles, the right-aligned last tile, and histories shorter than one tile (copied
    row by row); nothing else in the pool changes."""
    past, cand = [100, 7, 260, 0, 1, 63, 64, 65], [20, 3, 40, 5, 2, 1, 0, 9]
    H, L, S, n_cap = 2, 2, 9, 300
    batch = synth.make_prefill(1400, past, cand, H, D, n_slots=S)
    dp = DevPrefill(batch)
    pk, pv = nan_pool(L, S, H, n_cap, D)
    out = run_prefill(ub, dp, pool=(pk, pv), slots=dp.slots, layer=1).cpu().numpy()
    hk = np.full((L, S, H, n_cap, D), synth.BF16_NAN, dtype=np.uint16)
    hv = hk.copy()
    oracle.pool_write(hk, hv, 1, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, batch.slot_ids)
    assert bf16_tensor_bits(pk).tobytes() == hk.tobytes()
    assert bf16_tensor_bits(pv).tobytes() == hv.tobytes()
    ref = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    parity(out, ref, "fused prefill")


# ------------------------------------------------------------------ rank decode

DECODE_CASES = [
    # (past lens, cand lens, H, D, S, n_cap)
    ([200, 0, 37], [77, 5, 300], 2, 64, 6, 256),
    ([1000, 129, 256], [1, 130, 64], 2, 128, 4, 1024),
    ([64, 513], [16, 40], 2, 32, 3, 600),
    ([2048] * 4, [16] * 4, 2, 64, 8, 2048),      # small k, long history: split-n with a workspace
]


def run_decode(ub, dd: DevDecode, pk, pv, layer, workspace=None, out_fp32=True):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, layer, dd.max_k,
                              out_fp32=out_fp32, workspace=workspace, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    return out


@pytest.mark.parametrize("case", range(len(DECODE_CASES)))
@pytest.mark.parametrize("split", ["none", "counter", "full"])
def test_decode_matches_oracle(ub, case, split):
    past, cand, H, D, S, n_cap = DECODE_CASES[case]
    L, layer = 2, 1
    rng = np.random.Generator(np.random.PCG64(2000 + case))
    d = synth.make_decode(2000 + case, past, cand, H, D, n_slots=S, rng=rng)
    ks, vs = synth.pool_rows(rng, past, H, D)
    dd = DevDecode(d)
    pk, pv = nan_pool(L, S, H, n_cap, D)
    fill_pool_rows(pk, pv, layer, d.slot_ids, past, ks, vs)
    ws = None
    if split == "counter":
        ws = torch.empty(64, dtype=torch.float32, device="cuda")      # 256 bytes: work counter only
    elif split == "full":
        nbytes = ub.rank_decode_workspace_size(len(past), H, D, dd.max_k, int(d.cu_seqlens[-1]), n_cap)
        if nbytes <= 256:
            pytest.skip("no split for this shape")
        ws = torch.empty(nbytes // 4 + 4, dtype=torch.float32, device="cuda")
    out = run_decode(ub, dd, pk, pv, layer, workspace=ws).cpu().numpy()
    hk, hv = host_pool_layer(L, S, H, n_cap, D, layer, d.slot_ids, past, ks, vs)
    ref = oracle.decode(d.q, d.k, d.v, d.cu_seqlens, d.slot_ids, d.past_lens, hk, hv, 0)
    parity(out, ref, "decode case %d split=%s" % (case, split))


def test_split_decode_is_used_for_small_k(ub):
    assert ub.rank_decode_workspace_size(32, 8, 64, 16, 32 * 16, 2048) > 256
    assert ub.rank_decode_workspace_size(32, 8, 64, 1000, 32 * 1000, 2048) == 256


def test_work_distribution_does_not_change_results(ub):
    """Static striding (no workspace) and the shared work counter give identical bits."""
    batch = synth.make_prefill(1500, [300, 0, 129, 1000, 40], [50, 4, 130, 9, 300], 2, 64)
    dp = DevPrefill(batch)
    o_dyn = ub.masked_prefill_attn(dp.q, dp.k, dp.v, dp.cu, dp.past, dp.max_seqlen, workspace="auto")
    o_sta = ub.masked_prefill_attn(dp.q, dp.k, dp.v, dp.cu, dp.past, dp.max_seqlen, workspace=None)
    torch.cuda.synchronize()
    assert torch.equal(o_dyn, o_sta)


# ------------------------------------------------------------------- invariants

def test_candidate_permutation_permutes_outputs_bit_exactly(ub):
    n, k, H, D = 300, 200, 2, 64
    batch = synth.make_prefill(3000, [n], [k], H, D)
    perm = np.random.default_rng(3).permutation(k)
    idx = np.concatenate([np.arange(n), n + perm])
    b2 = synth.PrefillBatch(H, D, batch.past_lens, batch.cand_lens, batch.cu_seqlens,
                            batch.q[idx], batch.k[idx], batch.v[idx])
    o1 = run_prefill(ub, DevPrefill(batch)).cpu().numpy()
    o2 = run_prefill(ub, DevPrefill(b2)).cpu().numpy()
    assert np.array_equal(o2[:n], o1[:n])
    assert np.array_equal(o2[n:], o1[n + perm])


def test_k1_candidate_is_independent_of_its_batch(ub):
    n, H, D = 257, 2, 64
    batch = synth.make_prefill(3100, [n], [150], H, D)
    full = run_prefill(ub, DevPrefill(batch)).cpu().numpy()
    for c in (0, 77, 149):
        idx = np.concatenate([np.arange(n), [n + c]])
        alone = synth.PrefillBatch(H, D, np.array([n], np.int32), np.array([1], np.int32),
                                   np.array([0, n + 1], np.int32), batch.q[idx], batch.k[idx], batch.v[idx])
        o = run_prefill(ub, DevPrefill(alone)).cpu().numpy()
        assert np.array_equal(o[n], full[n + c])


@pytest.mark.parametrize("D", [128, 64])
def test_prefill_candidate_rows_equal_decode_over_written_pool(ub, D):
    """Decode over the pool the prefill wrote gives the prefill's candidate rows: bit for bit at
    D = 128 (both calls sweep 64-key tiles), within tolerance at D = 64 (the prefill sweeps 64-key
    tiles, the many-candidate decode 128-key tiles)."""
    past, cand = [300, 0, 129, 1000], [50, 4, 130, 9]
    H, L, S, n_cap = 2, 2, 6, 1024
    batch = synth.make_prefill(3200, past, cand, H, D, n_slots=S)
    dp = DevPrefill(batch)
    pk, pv = nan_pool(L, S, H, n_cap, D)
    pre = run_prefill(ub, dp, pool=(pk, pv), slots=dp.slots, layer=1)
    cidx = np.concatenate([np.arange(batch.cu_seqlens[b] + past[b], batch.cu_seqlens[b + 1]) for b in range(4)])
    d = synth.DecodeBatch(H, D, batch.past_lens, batch.cand_lens, synth.cu_from_lens(np.array(cand)),
                          batch.slot_ids, batch.q[cidx], batch.k[cidx], batch.v[cidx])
    dec = run_decode(ub, DevDecode(d), pk, pv, 1)
    pre_c = pre[torch.from_numpy(cidx).cuda()]
    assert torch.isfinite(dec).all()
    parity(dec.cpu().numpy(), pre_c.cpu().numpy().astype(np.float64), "prefill vs decode")
    if D == 128:
        assert torch.equal(dec, pre_c), "decode rows differ from prefill candidate rows in some bits"


# ------------------------------------------------------------- error reporting

def test_host_side_argument_errors(ub):
    batch = synth.make_prefill(4000, [10], [5], 1, 64)
    dp = DevPrefill(batch)
    with pytest.raises(ub.UnipinError) as e:     # unsupported head dim
        q48 = torch.zeros((15, 1, 48), dtype=torch.bfloat16, device="cuda")
        ub.masked_prefill_attn(q48, q48, q48, dp.cu, dp.past, 15)
    assert e.value.code == -2
    pk, pv = nan_pool(2, 2, 1, 16, 64)
    with pytest.raises(ub.UnipinError) as e:     # layer out of range
        ub.kvpool_write(pk, pv, 5, dp.k, dp.v, dp.cu, dp.past, to_dev_i32([0]), 10)
    assert e.value.code == -4
    with pytest.raises(ub.UnipinError) as e:     # misaligned tensor
        base = torch.zeros(15 * 64 + 1, dtype=torch.bfloat16, device="cuda")
        qm = base[1:].view(15, 1, 64)
        ub.masked_prefill_attn(qm, dp.k, dp.v, dp.cu, dp.past, 15)
    assert e.value.code == -3


def test_device_side_range_errors_are_reported(ub):
    batch = synth.make_prefill(4100, [10, 20], [5, 5], 1, 64, n_slots=4)
    dp = DevPrefill(batch)
    pk, pv = nan_pool(1, 4, 1, 16, 64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # past length 20 > n_cap 16: the block reports and writes nothing
    ub.kvpool_write(pk, pv, 0, dp.k, dp.v, dp.cu, dp.past, dp.slots, 16, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -4
    # slot id 7 of 4 in the decode
    d = synth.make_decode(4200, [3], [2], 1, 64, n_slots=4)
    dd = DevDecode(d)
    dd.slots = to_dev_i32([7])
    status.zero_()
    out = torch.zeros((2, 1, 64), dtype=torch.float32, device="cuda")
    ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, 0, 2, out=out, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -4
    assert torch.count_nonzero(out) == 0
    # a segment longer than the stated max_seqlen
    status.zero_()
    ub.masked_prefill_attn(dp.q, dp.k, dp.v, dp.cu, dp.past, 8, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -4


def test_bounded_wait_times_out_with_status_not_hang(ub):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ub.selftest_bounded_wait(status, 20000)   # 20 ms limit on a barrier nothing completes
    torch.cuda.synchronize()
    assert int(status.item()) == -6
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float(x.sum().item()) == 4.0


def test_fma_pipe_exp2_against_cuda_exp2f(ub):
    """The polynomial exp2 the softmax uses for one score pair in four, against CUDA's exp2f."""
    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 20, device="cuda"),
                   torch.tensor([0.0, 1.0, -1.0, 8.0, -0.5, 0.5, 3.0, -126.0], device="cuda")])
    y = ub.selftest_exp2(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 1.2e-4, rel
    # integers are exact (p(0) = 1), arguments at or below -127 and -inf give 0
    ints = torch.arange(-120, 9, device="cuda", dtype=torch.float32)
    assert torch.equal(ub.selftest_exp2(ints), torch.exp2(ints))
    low = torch.tensor([-127.0, -200.0, -1e30, float("-inf")], device="cuda")
    assert torch.count_nonzero(ub.selftest_exp2(low)) == 0
