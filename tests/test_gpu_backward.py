"""GPU parity of the masked-prefill gradients (dQ, dK, dV) and the forward's row statistic.

The same seeded bf16 inputs and upstream gradient feed the CUDA path (forward
with its row log-sum-exp, then the backward call) and the fp64 oracle's
chain-rule gradients.  P and dS enter the tensor cores as bf16, so each
gradient tensor is compared by relative L2 error (<= 1e-2, an order of
magnitude above the ~1e-3 that bf16 rounding of P and dS gives) and by
max-abs error relative to the tensor's largest reference value (<= 2e-2).
"""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth
from tests.gpu_helpers import DevPrefill, to_dev_bf16

pytestmark = pytest.mark.gpu

LOG2E = 1.4426950408889634
GRAD_REL_L2 = 1e-2
GRAD_MAX_ABS_REL = 2e-2


@pytest.fixture(scope="module")
def ub():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_reuse_falcon_b200 import binding
    return binding


def grad_parity(gpu, ref, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    assert np.isfinite(gpu).all(), what + ": non-finite gradient"
    err = gpu - ref
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.abs(err).max() / max(np.abs(ref).max(), 1e-300))
    assert rel <= GRAD_REL_L2 and mx <= GRAD_MAX_ABS_REL, "%s: rel_l2=%.3e max_abs/max=%.3e" % (what, rel, mx)
    return rel, mx


def run_fwd_bwd(ub, batch, g_bits):
    dp = DevPrefill(batch)
    T, H, D = batch.q.shape
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    out = ub.masked_prefill_attn(dp.q, dp.k, dp.v, dp.cu, dp.past, dp.max_seqlen, out_fp32=False, lse=lse,
                                 dev_status=status)
    dout = to_dev_bf16(g_bits)
    dq, dk, dv = ub.masked_prefill_bwd(dp.q, dp.k, dp.v, out, dout, lse, dp.cu, dp.past, dp.max_seqlen,
                                       dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    return lse, dq, dk, dv


BWD_CASES = [
    # (past lens, cand lens, H, D)
    ([64, 64], [16, 16], 2, 32),                 # the tiny workload's shape
    ([200, 37, 300], [77, 5, 260], 2, 64),       # ragged tails, several tiles
    ([1, 0, 129, 5], [0, 7, 3, 300], 1, 64),     # n=1, n=0, k=0
    ([128, 256], [128, 1], 2, 64),               # tile-aligned history
    ([90, 513], [40, 33], 3, 32),                # D = 32, several tiles
    ([200, 37, 300], [77, 5, 260], 2, 128),      # D = 128: dQ in two halves over the score columns
    ([1, 0, 129, 256], [0, 7, 3, 300], 1, 128),  # n=1, n=0, k=0, tile-aligned, D = 128
]


@pytest.mark.parametrize("case", range(len(BWD_CASES)))
def test_backward_matches_oracle(ub, case):
    past, cand, H, D = BWD_CASES[case]
    batch = synth.make_prefill(6000 + case, past, cand, H, D)
    g = synth.normal_bf16(np.random.Generator(np.random.PCG64(6100 + case)), batch.q.shape)
    lse, dq, dk, dv = run_fwd_bwd(ub, batch, g)
    rq, rk, rv = oracle.prefill_bwd(batch.q, batch.k, batch.v, g, batch.cu_seqlens, batch.past_lens)
    grad_parity(dq.cpu().numpy(), rq, "dq case %d" % case)
    grad_parity(dk.cpu().numpy(), rk, "dk case %d" % case)
    grad_parity(dv.cpu().numpy(), rv, "dv case %d" % case)


def test_forward_row_statistic_matches_oracle(ub):
    past, cand, H, D = [200, 0, 513], [77, 9, 40], 2, 64
    batch = synth.make_prefill(6200, past, cand, H, D)
    dp = DevPrefill(batch)
    T = batch.T
    lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    ub.masked_prefill_attn(dp.q, dp.k, dp.v, dp.cu, dp.past, dp.max_seqlen, out_fp32=True, lse=lse)
    torch.cuda.synchronize()
    _, ref = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, return_lse=True)
    assert np.abs(lse.cpu().numpy() - ref * LOG2E).max() < 2e-3


def test_backward_prefill_workload(ub):
    """B=64, n=256, k=128, H=8, D=64 (the prefill workload), every gradient element."""
    w = synth.workload("prefill_B64")
    rng = np.random.Generator(np.random.PCG64(w.seed))
    past, cand = w.lengths(rng)
    batch = synth.make_prefill(w.seed, past, cand, w.H, w.D, rng=rng)
    g = synth.normal_bf16(rng, batch.q.shape)
    _, dq, dk, dv = run_fwd_bwd(ub, batch, g)
    rq, rk, rv = oracle.prefill_bwd(batch.q, batch.k, batch.v, g, batch.cu_seqlens, batch.past_lens)
    for name, a, b in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        grad_parity(a.cpu().numpy(), b, name + " prefill workload")


def test_backward_candidate_permutation_permutes_gradients(ub):
    """Permuting a segment's candidates permutes their gradients; the past tokens' gradients
    change only by the order of the dQ additions."""
    n, k, H, D = 300, 200, 2, 64
    batch = synth.make_prefill(6300, [n], [k], H, D)
    g = synth.normal_bf16(np.random.Generator(np.random.PCG64(6301)), batch.q.shape)
    perm = np.random.default_rng(3).permutation(k)
    idx = np.concatenate([np.arange(n), n + perm])
    b2 = synth.PrefillBatch(H, D, batch.past_lens, batch.cand_lens, batch.cu_seqlens,
                            batch.q[idx], batch.k[idx], batch.v[idx])
    _, q1, k1, v1 = run_fwd_bwd(ub, batch, g)
    _, q2, k2, v2 = run_fwd_bwd(ub, b2, g[idx])
    pidx = torch.from_numpy(n + perm).cuda()
    for a, b in ((q1, q2), (k1, k2), (v1, v2)):
        assert torch.equal(b[n:], a[pidx]) or torch.allclose(b[n:], a[pidx], rtol=1e-5, atol=1e-6)
        assert torch.allclose(b[:n], a[:n], rtol=1e-4, atol=1e-5)
