"""Pins for grouped-query attention in the oracle ([notes] §6 calls the pool's H "KV heads").

Query head h reads key/value head h // G (G = H / Hkv).  Checked against:
* the same computation with K/V repeated G times along the head axis (plain
  multi-head attention) - prefill, rank decode and gradients (a kv head's
  gradient is the sum of its query heads');
* torch's causal SDPA with enable_gqa on past rows;
* the plausible mistake of mapping query head h to kv head h % Hkv, which
  must not agree.
"""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth


def gqa_batch(seed, past, cand, H, Hkv, D):
    rng = np.random.Generator(np.random.PCG64(seed))
    cu = synth.cu_from_lens(np.array(past) + np.array(cand))
    T = int(cu[-1])
    q = synth.normal_bf16(rng, (T, H, D))
    k = synth.normal_bf16(rng, (T, Hkv, D))
    v = synth.normal_bf16(rng, (T, Hkv, D))
    return cu, np.array(past, np.int32), q, k, v, rng


@pytest.mark.parametrize("H,Hkv", [(4, 2), (8, 1), (6, 3)])
def test_gqa_prefill_equals_mha_on_repeated_kv(H, Hkv):
    G = H // Hkv
    cu, past, q, k, v, _ = gqa_batch(10 + H, [9, 0, 17], [4, 3, 5], H, Hkv, 8)
    out = oracle.prefill(q, k, v, cu, past)
    ref = oracle.prefill(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), cu, past)
    assert np.array_equal(out, ref)
    if Hkv > 1:
        wrong = oracle.prefill(q, np.tile(k, (1, G, 1)), np.tile(v, (1, G, 1)), cu, past)
        assert not np.allclose(out, wrong)


def test_gqa_past_rows_equal_torch_sdpa_with_groups():
    H, Hkv, D, n = 8, 2, 16, 23
    cu, past, q, k, v, _ = gqa_batch(30, [n], [0], H, Hkv, D)
    out = oracle.prefill(q, k, v, cu, past)
    f = lambda a: torch.from_numpy(synth.bf16_bits_to_f64(a)).transpose(0, 1)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(f(q), f(k), f(v), is_causal=True, enable_gqa=True)
    np.testing.assert_allclose(out, ref[0].transpose(0, 1).numpy(), rtol=1e-12, atol=1e-12)


def test_gqa_decode_equals_mha_on_repeated_pool():
    H, Hkv, D, S, n_cap = 4, 2, 8, 5, 40
    G = H // Hkv
    past, cand = [30, 0, 12], [3, 2, 4]
    rng = np.random.Generator(np.random.PCG64(40))
    cu = synth.cu_from_lens(np.array(cand))
    Tc = int(cu[-1])
    qc = synth.normal_bf16(rng, (Tc, H, D))
    kc = synth.normal_bf16(rng, (Tc, Hkv, D))
    vc = synth.normal_bf16(rng, (Tc, Hkv, D))
    slots = np.array([4, 0, 2], np.int32)
    pk = synth.normal_bf16(rng, (1, S, Hkv, n_cap, D))
    pv = synth.normal_bf16(rng, (1, S, Hkv, n_cap, D))
    out = oracle.decode(qc, kc, vc, cu, slots, past, pk, pv, 0)
    ref = oracle.decode(qc, np.repeat(kc, G, 1), np.repeat(vc, G, 1), cu, slots, past,
                        np.repeat(pk, G, 2), np.repeat(pv, G, 2), 0)
    assert np.array_equal(out, ref)


def test_gqa_gradients_sum_over_the_group():
    H, Hkv, D = 6, 2, 8
    G = H // Hkv
    cu, past, q, k, v, rng = gqa_batch(50, [7, 3], [3, 4], H, Hkv, D)
    g = synth.normal_bf16(rng, q.shape)
    dq, dk, dv = oracle.prefill_bwd(q, k, v, g, cu, past)
    rq, rk, rv = oracle.prefill_bwd(q, np.repeat(k, G, 1), np.repeat(v, G, 1), g, cu, past)
    T = q.shape[0]
    np.testing.assert_allclose(dq, rq, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dk, rk.reshape(T, Hkv, G, D).sum(2), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, rv.reshape(T, Hkv, G, D).sum(2), rtol=1e-12, atol=1e-13)
