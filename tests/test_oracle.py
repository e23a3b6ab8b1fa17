"""Pins for the CPU oracle: it is checked against things other than itself.

* a hand-transcribed mask fixture (tests/golden/mfalcon_masks.txt), read back
  out of the oracle with a probe whose output *is* the attention weights;
* a dense brute-force fp64 implementation (full (n+k)^2 score matrix, -inf
  fill) written independently here;
* library reductions: past rows equal torch's causal SDPA run on the past
  tokens alone; a candidate row equals an unmasked single-query SDPA over
  [K_past; k_i];
* closed forms (row 0 = v_0, n=0 gives v_i, constant V, identical keys give the
  mean of the allowed values);
* invariants the pages state: permuting candidates only permutes their
  outputs, a k=1 candidate's output is independent of the batch it sits in,
  and candidate rows of the prefill equal rank decode over the written pool;
* plausible mistakes (a dropped self term, a wrong scale, a transposed
  operand) each fail at least one of the pins above.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mfalcon_masks.txt")


def read_golden_masks():
    cases = []
    with open(GOLDEN) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    i = 0
    while i < len(lines):
        _, n, k = lines[i].split()
        n, k = int(n), int(k)
        rows = lines[i + 1:i + 1 + n + k]
        m = np.array([[int(c) for c in r] for r in rows], dtype=np.int64)
        assert m.shape == (n + k, n + k)
        cases.append((n, k, m))
        i += 1 + n + k
    return cases


def f64(bits):
    return synth.bf16_bits_to_f64(bits)


def bits(x):
    return synth.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def dense_reference(q, k, v, n_past, scale, cand_self=True):
    """Independent brute force for ONE segment: full score matrix, -inf fill, softmax by rows."""
    qd, kd, vd = f64(q), f64(k), f64(v)          # [T, H, D]
    T, H, D = qd.shape
    out = np.zeros((T, H, D))
    ii = np.arange(T)[:, None]
    jj = np.arange(T)[None, :]
    causal_past = (ii < n_past) & (jj <= ii)
    cand_sees_past = (ii >= n_past) & (jj < n_past)
    cand_self_m = (ii >= n_past) & (jj == ii) & cand_self
    mask = causal_past | cand_sees_past | cand_self_m
    for h in range(H):
        s = (qd[:, h, :] @ kd[:, h, :].T) * scale
        s = np.where(mask, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        w = np.exp(s - m)
        den = w.sum(axis=1, keepdims=True)
        o = w @ vd[:, h, :]
        out[:, h, :] = np.where(den > 0, o / np.where(den > 0, den, 1.0), 0.0)
    return out


# ---------------------------------------------------------------- golden mask

@pytest.mark.parametrize("case", range(4))
def test_mask_matches_hand_transcribed_golden(case):
    n, k, golden = read_golden_masks()[case]
    T = n + k
    H = 1
    D = T  # V = identity: output row i is the attention-weight row itself
    q = bits(np.random.default_rng(case).standard_normal((T, H, D)))
    kk = bits(np.zeros((T, H, D)))        # equal scores -> uniform weights over the allowed set
    v = bits(np.eye(T).reshape(T, H, D))
    out = oracle.prefill(q, kk, v, [0, T], [n])[:, 0, :]
    counts = golden.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(out, golden / counts, rtol=0, atol=1e-15)


def test_golden_file_is_the_stated_rule_not_a_copy_of_the_oracle():
    # Sanity on the fixture itself: every row has a key, no candidate sees another candidate.
    for n, k, m in read_golden_masks():
        assert (m.sum(axis=1) >= 1).all()
        c = m[n:, n:]
        assert (c == np.eye(k, dtype=np.int64)).all()
        p = m[:n, :n]
        assert (p == np.tril(np.ones((n, n), dtype=np.int64))).all()
        assert (m[:n, n:] == 0).all()


# --------------------------------------------------------------- brute force

@pytest.mark.parametrize("seed", range(6))
def test_oracle_equals_dense_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 4))
    past = rng.integers(0, 9, size=B)
    cand = rng.integers(0, 9, size=B)
    H, D = int(rng.integers(1, 3)), int(rng.choice([2, 4, 8]))
    batch = synth.make_prefill(seed, past, cand, H, D)
    out = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    scale = 1.0 / np.sqrt(D)
    for b in range(B):
        lo, hi = batch.cu_seqlens[b], batch.cu_seqlens[b + 1]
        if hi == lo:
            continue
        ref = dense_reference(batch.q[lo:hi], batch.k[lo:hi], batch.v[lo:hi], int(past[b]), scale)
        np.testing.assert_allclose(out[lo:hi], ref, rtol=0, atol=1e-12)


def test_oracle_lse_equals_logsumexp_of_dense_scores():
    batch = synth.make_prefill(7, [6], [4], 2, 8)
    out, lse = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, return_lse=True)
    qd, kd = f64(batch.q), f64(batch.k)
    for h in range(2):
        s = qd[:, h] @ kd[:, h].T / np.sqrt(8)
        for i in range(10):
            allowed = [j for j in range(10) if (j <= i if i < 6 else (j < 6 or j == i))]
            ref = np.log(np.sum(np.exp(s[i, allowed])))
            assert abs(lse[i, h] - ref) < 1e-12


def test_cand_self_false_reading_drops_only_the_diagonal():
    batch = synth.make_prefill(3, [5, 0], [3, 2], 1, 4)
    out = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, cand_self=False)
    ref = dense_reference(batch.q[:8], batch.k[:8], batch.v[:8], 5, 0.5, cand_self=False)
    np.testing.assert_allclose(out[:8], ref, atol=1e-12, rtol=0)
    # n=0 and no self: empty key set, defined as 0
    assert np.all(out[8:] == 0.0)


# ---------------------------------------------------------- library reductions

def sdpa64(q, k, v, causal):
    """torch SDPA in fp64 on CPU; q/k/v as [L, H, D] float64 numpy."""
    tq = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))[None]
    tk = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None]
    tv = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    return o[0].numpy().transpose(1, 0, 2)


@pytest.mark.parametrize("n,k", [(1, 1), (17, 5), (64, 16), (130, 7)])
def test_past_rows_equal_causal_sdpa_without_candidates(n, k):
    batch = synth.make_prefill(11, [n], [k], 2, 16)
    out = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    ref = sdpa64(f64(batch.q[:n]), f64(batch.k[:n]), f64(batch.v[:n]), causal=True)
    np.testing.assert_allclose(out[:n], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n,k", [(0, 3), (9, 4), (64, 16)])
def test_candidate_row_equals_single_query_sdpa_over_past_and_self(n, k):
    batch = synth.make_prefill(12, [n], [k], 2, 16)
    out = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    q, kk, v = f64(batch.q), f64(batch.k), f64(batch.v)
    for c in range(k):
        i = n + c
        keys = np.concatenate([kk[:n], kk[i:i + 1]], axis=0)
        vals = np.concatenate([v[:n], v[i:i + 1]], axis=0)
        ref = sdpa64(q[i:i + 1], keys, vals, causal=False)
        np.testing.assert_allclose(out[i:i + 1], ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- closed forms

def test_closed_forms():
    batch = synth.make_prefill(13, [6, 0], [3, 4], 2, 8)
    out = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    v = f64(batch.v)
    # row 0 of a segment with n>0 sees only itself
    np.testing.assert_array_equal(out[0], v[0])
    # a segment with n=0: every candidate sees only itself
    np.testing.assert_array_equal(out[9:13], v[9:13])

    # constant V rows -> that constant
    T, H, D = 12, 2, 8
    b2 = synth.make_prefill(14, [8], [4], H, D)
    const = bits(np.full((T, H, D), 0.375))
    out2 = oracle.prefill(b2.q, b2.k, const, b2.cu_seqlens, b2.past_lens)
    np.testing.assert_allclose(out2, 0.375, rtol=0, atol=1e-14)

    # identical keys -> mean of the allowed values
    same_k = np.broadcast_to(b2.k[:1], b2.k.shape).copy()
    out3 = oracle.prefill(b2.q, same_k, b2.v, b2.cu_seqlens, b2.past_lens)
    vv = f64(b2.v)
    for i in range(T):
        allowed = list(range(i + 1)) if i < 8 else list(range(8)) + [i]
        np.testing.assert_allclose(out3[i], vv[allowed].mean(axis=0), rtol=0, atol=1e-13)


def test_two_key_softmax_by_hand():
    # D=1, scale 1: row 1 sees keys 0,1 with scores q1*k0, q1*k1 -> weights 1:e^1
    q = bits(np.array([[[1.0]], [[1.0]]]))
    k = bits(np.array([[[0.0]], [[1.0]]]))
    v = bits(np.array([[[2.0]], [[-4.0]]]))
    out = oracle.prefill(q, k, v, [0, 2], [2], scale=1.0)
    e = np.e
    assert abs(out[1, 0, 0] - (2.0 * 1 + (-4.0) * e) / (1 + e)) < 1e-15
    assert out[0, 0, 0] == 2.0


# ----------------------------------------------------------------- invariants

def test_permuting_candidates_permutes_outputs_only():
    n, k, H, D = 20, 9, 2, 16
    batch = synth.make_prefill(15, [n], [k], H, D)
    perm = np.random.default_rng(1).permutation(k)
    idx = np.concatenate([np.arange(n), n + perm])
    out = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    outp = oracle.prefill(batch.q[idx], batch.k[idx], batch.v[idx], batch.cu_seqlens, batch.past_lens)
    np.testing.assert_array_equal(outp[:n], out[:n])
    np.testing.assert_array_equal(outp[n:], out[n + perm])


def test_k1_candidate_independent_of_its_batch():
    n, H, D = 30, 2, 8
    batch = synth.make_prefill(16, [n], [12], H, D)
    full = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    for c in (0, 5, 11):
        idx = np.concatenate([np.arange(n), [n + c]])
        alone = oracle.prefill(batch.q[idx], batch.k[idx], batch.v[idx], [0, n + 1], [n])
        np.testing.assert_array_equal(alone[n], full[n + c])


def test_prefill_candidate_rows_equal_decode_over_written_pool():
    past, cand = [13, 0, 40], [5, 3, 7]
    H, D, L, S, n_cap = 2, 8, 3, 6, 48
    batch = synth.make_prefill(17, past, cand, H, D, n_slots=S)
    pk = np.full((L, S, H, n_cap, D), synth.BF16_NAN, dtype=np.uint16)
    pv = pk.copy()
    layer = 1
    oracle.pool_write(pk, pv, layer, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, batch.slot_ids)
    out = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    cand_idx = np.concatenate([np.arange(batch.cu_seqlens[b] + past[b], batch.cu_seqlens[b + 1])
                               for b in range(3)])
    cu_c = synth.cu_from_lens(np.array(cand))
    dec = oracle.decode(batch.q[cand_idx], batch.k[cand_idx], batch.v[cand_idx], cu_c, batch.slot_ids,
                        batch.past_lens, pk, pv, layer)
    np.testing.assert_allclose(dec, out[cand_idx], rtol=0, atol=1e-13)
    assert np.isfinite(dec).all()


def test_decode_with_empty_history_returns_own_value():
    H, D = 2, 8
    d = synth.make_decode(18, [0, 0], [2, 3], H, D, n_slots=4)
    pk = np.full((1, 4, H, 8, D), synth.BF16_NAN, dtype=np.uint16)
    out = oracle.decode(d.q, d.k, d.v, d.cu_seqlens, d.slot_ids, d.past_lens, pk, pk.copy(), 0)
    np.testing.assert_array_equal(out, f64(d.v))


def test_sampled_tokens_equal_full_evaluation():
    batch = synth.make_prefill(19, [30, 5], [10, 20], 2, 8)
    full = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    toks = np.array([0, 7, 29, 30, 39, 40, 44, 64])
    part = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, tokens=toks)
    np.testing.assert_array_equal(part, full[toks])


# -------------------------------------------------------------------- pool write

def test_pool_write_mirror_against_numpy_indexing():
    past, cand = [5, 0, 11, 3], [2, 4, 1, 6]
    H, D, L, S, n_cap = 3, 8, 2, 7, 12
    batch = synth.make_prefill(20, past, cand, H, D, n_slots=S)
    pk = np.full((L, S, H, n_cap, D), synth.BF16_NAN, dtype=np.uint16)
    pv = pk.copy()
    oracle.pool_write(pk, pv, 1, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, batch.slot_ids)
    ek = np.full_like(pk, synth.BF16_NAN)
    ev = ek.copy()
    for b in range(4):
        s, lo, n = batch.slot_ids[b], batch.cu_seqlens[b], past[b]
        ek[1, s, :, :n, :] = batch.k[lo:lo + n].transpose(1, 0, 2)
        ev[1, s, :, :n, :] = batch.v[lo:lo + n].transpose(1, 0, 2)
    assert pk.tobytes() == ek.tobytes()
    assert pv.tobytes() == ev.tobytes()


def test_pool_write_rejects_out_of_range():
    batch = synth.make_prefill(21, [5], [1], 1, 8, n_slots=2)
    pk = np.zeros((1, 2, 1, 4, 8), dtype=np.uint16)
    with pytest.raises(ValueError):   # n_b = 5 > n_cap = 4
        oracle.pool_write(pk, pk.copy(), 0, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, batch.slot_ids)
    with pytest.raises(ValueError):   # slot 2 of 2
        oracle.pool_write(np.zeros((1, 2, 1, 8, 8), np.uint16), np.zeros((1, 2, 1, 8, 8), np.uint16), 0,
                          batch.k, batch.v, batch.cu_seqlens, batch.past_lens, np.array([2], np.int32))


# -------------------------------------------------- planted mistakes are caught

def test_planted_mistakes_fail_the_pins():
    """Each plausible oracle mistake, planted on the CPU, fails a pin above."""
    n, k, H, D = 9, 4, 2, 16
    batch = synth.make_prefill(22, [n], [k], H, D)
    q, kk, v = f64(batch.q), f64(batch.k), f64(batch.v)

    def cand_pin(out):
        i = n + 1
        ref = sdpa64(q[i:i + 1], np.concatenate([kk[:n], kk[i:i + 1]]),
                     np.concatenate([v[:n], v[i:i + 1]]), causal=False)
        return np.abs(out[i:i + 1] - ref).max() < 1e-12

    def past_pin(out):
        ref = sdpa64(q[:n], kk[:n], v[:n], causal=True)
        return np.abs(out[:n] - ref).max() < 1e-12

    good = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    assert cand_pin(good) and past_pin(good)
    # dropped self term
    assert not cand_pin(oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens,
                                       cand_self=False))
    # wrong scale (1 instead of 1/sqrt(D))
    assert not past_pin(oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens, scale=1.0))
    # K and V swapped
    assert not past_pin(oracle.prefill(batch.q, batch.v, batch.k, batch.cu_seqlens, batch.past_lens))
    # wrong past length (one candidate treated as past)
    assert not cand_pin(oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, [n + 1]))


# ------------------------------------------------------------------ generator

def test_generator_is_deterministic_and_rounds_like_torch():
    a = synth.make_prefill(5, [4, 3], [2, 2], 2, 8, n_slots=9)
    b = synth.make_prefill(5, [4, 3], [2, 2], 2, 8, n_slots=9)
    assert a.q.tobytes() == b.q.tobytes() and (a.slot_ids == b.slot_ids).all()
    assert len(set(a.slot_ids.tolist())) == 2
    x = np.random.default_rng(0).standard_normal(4096).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(synth.f32_to_bf16_bits(x), ref)
    back = synth.bf16_bits_to_f64(ref)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())
