"""Pins for the oracle's backward pass (gradients of the masked attention).

The gradients are checked against things other than the oracle itself:
* central finite differences of a dense fp64 forward written here (full score
  matrix, -inf fill), on tiny ragged batches with fp64 inputs;
* torch's fp64 autograd of the same dense masked attention, on bf16 inputs;
* closed forms: a row with one key passes its whole dO to that key's value and
  no gradient to its query or key; candidates of a user with no history get
  dV = dO and dQ = dK = 0; identical keys give dQ = 0; the key gradients of a
  segment and head sum to zero (adding one vector to every key moves each
  row's scores by a per-row constant, which the softmax ignores);
* invariants: permuting candidates permutes their gradients and leaves the
  past tokens' gradients unchanged;
* planted mistakes (K and V swapped, scale 1, dropped self term, a candidate
  counted as past) each fail the autograd pin.
"""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth


def mask_of(T, n_past, cand_self=True):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return ((i < n_past) & (j <= i)) | ((i >= n_past) & (j < n_past)) | ((i >= n_past) & (j == i) & cand_self)


def dense_forward(q, k, v, cu, past, scale):
    """fp64 forward of packed segments, one dense masked softmax per (segment, head)."""
    out = np.zeros_like(q)
    for b in range(len(past)):
        lo, hi = int(cu[b]), int(cu[b + 1])
        m = mask_of(hi - lo, int(past[b]))
        for h in range(q.shape[1]):
            s = np.where(m, q[lo:hi, h] @ k[lo:hi, h].T * scale, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            w = np.exp(s)
            out[lo:hi, h] = (w / w.sum(axis=1, keepdims=True)) @ v[lo:hi, h]
    return out


def torch_grads(qb, kb, vb, gb, cu, past, scale, cand_self=True):
    """fp64 autograd of the dense masked attention on bf16 inputs."""
    q, k, v, g = (torch.from_numpy(synth.bf16_bits_to_f64(x)).requires_grad_(True) for x in (qb, kb, vb, gb))
    g = g.detach()
    outs = []
    for b in range(len(past)):
        lo, hi = int(cu[b]), int(cu[b + 1])
        m = torch.from_numpy(mask_of(hi - lo, int(past[b]), cand_self))
        qs, ks, vs = q[lo:hi].transpose(0, 1), k[lo:hi].transpose(0, 1), v[lo:hi].transpose(0, 1)
        s = (qs @ ks.transpose(1, 2)) * scale
        s = s.masked_fill(~m, float("-inf"))
        o = torch.softmax(s, dim=-1) @ vs
        outs.append(o.transpose(0, 1))
    loss = (torch.cat(outs) * g).sum()
    loss.backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


CASES = [([5, 0], [3, 2]), ([1, 4, 7], [2, 0, 3]), ([6], [4])]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_backward_equals_central_differences(case):
    past, cand = CASES[case]
    H, D = 2, 4
    cu = synth.cu_from_lens(np.array(past) + np.array(cand))
    T = int(cu[-1])
    rng = np.random.default_rng(100 + case)
    q, k, v, g = (rng.standard_normal((T, H, D)) for _ in range(4))
    scale = 0.7
    dq, dk, dv = oracle.prefill_bwd_f64(q, k, v, g, cu, past, scale=scale)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            lp = (dense_forward(q, k, v, cu, past, scale) * g).sum()
            x[idx] = keep - eps
            lm = (dense_forward(q, k, v, cu, past, scale) * g).sum()
            x[idx] = keep
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_equals_torch_autograd_on_bf16_inputs():
    past, cand, H, D = [9, 0, 17, 1], [4, 3, 6, 5], 2, 16
    batch = synth.make_prefill(31, past, cand, H, D)
    rng = np.random.Generator(np.random.PCG64(32))
    g = synth.normal_bf16(rng, batch.q.shape)
    scale = 1 / np.sqrt(D)
    dq, dk, dv = oracle.prefill_bwd(batch.q, batch.k, batch.v, g, batch.cu_seqlens, batch.past_lens)
    tq, tk, tv = torch_grads(batch.q, batch.k, batch.v, g, batch.cu_seqlens, batch.past_lens, scale)
    for a, b in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


def test_backward_closed_forms():
    H, D = 2, 8
    rng = np.random.default_rng(7)
    # no history: each candidate attends only to itself
    q, k, v, g = (rng.standard_normal((4, H, D)) for _ in range(4))
    dq, dk, dv = oracle.prefill_bwd_f64(q, k, v, g, [0, 4], [0])
    assert np.array_equal(dv, g) and not dq.any() and not dk.any()
    # row 0 of a segment has one key: its dO goes to v_0 alone, no query/key gradient from it
    q, k, v, g = (rng.standard_normal((3, H, D)) for _ in range(4))
    g[1:] = 0.0
    dq, dk, dv = oracle.prefill_bwd_f64(q, k, v, g, [0, 3], [3])
    assert np.array_equal(dv[0], g[0]) and not dv[1:].any() and not dq.any() and not dk.any()
    # identical keys: every row's scores are equal, so no query gradient
    q, v, g = (rng.standard_normal((7, H, D)) for _ in range(3))
    k = np.broadcast_to(rng.standard_normal((1, H, D)), (7, H, D)).copy()
    dq, _, _ = oracle.prefill_bwd_f64(q, k, v, g, [0, 7], [4])
    assert np.abs(dq).max() < 1e-14
    # key gradients of a segment and head sum to zero
    q, k, v, g = (rng.standard_normal((11, H, D)) for _ in range(4))
    _, dk, _ = oracle.prefill_bwd_f64(q, k, v, g, [0, 5, 11], [3, 2])
    assert np.abs(dk[:5].sum(axis=0)).max() < 1e-12 and np.abs(dk[5:].sum(axis=0)).max() < 1e-12


def test_permuting_candidates_permutes_their_gradients_only():
    n, kc, H, D = 7, 5, 2, 8
    rng = np.random.default_rng(9)
    q, k, v, g = (rng.standard_normal((n + kc, H, D)) for _ in range(4))
    perm = rng.permutation(kc)
    idx = np.concatenate([np.arange(n), n + perm])
    a = oracle.prefill_bwd_f64(q, k, v, g, [0, n + kc], [n])
    b = oracle.prefill_bwd_f64(q[idx], k[idx], v[idx], g[idx], [0, n + kc], [n])
    for x, y in zip(a, b):
        np.testing.assert_allclose(y[:n], x[:n], rtol=1e-12, atol=1e-14)
        assert np.array_equal(y[n:], x[n + perm])


def test_planted_backward_mistakes_fail_the_autograd_pin():
    past, cand, H, D = [6, 3], [3, 4], 1, 8
    batch = synth.make_prefill(41, past, cand, H, D)
    g = synth.normal_bf16(np.random.Generator(np.random.PCG64(42)), batch.q.shape)
    scale = 1 / np.sqrt(D)
    ref = torch_grads(batch.q, batch.k, batch.v, g, batch.cu_seqlens, batch.past_lens, scale)

    def pinned(grads):
        return all(np.allclose(a, b, rtol=1e-10, atol=1e-12) for a, b in zip(grads, ref))

    cu, pl = batch.cu_seqlens, batch.past_lens
    assert pinned(oracle.prefill_bwd(batch.q, batch.k, batch.v, g, cu, pl))
    assert not pinned(oracle.prefill_bwd(batch.q, batch.v, batch.k, g, cu, pl))             # K, V swapped
    assert not pinned(oracle.prefill_bwd(batch.q, batch.k, batch.v, g, cu, pl, scale=1.0))  # wrong scale
    assert not pinned(oracle.prefill_bwd(batch.q, batch.k, batch.v, g, cu, pl, cand_self=False))
    assert not pinned(oracle.prefill_bwd(batch.q, batch.k, batch.v, g, cu, [7, 3]))          # a candidate as past
