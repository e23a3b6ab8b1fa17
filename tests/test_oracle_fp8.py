"""Pins for the E4M3 pool variant of the oracle (an extrapolation of the pages' FP8
E4M3 recipe for linear layers to the KV pool; the encoding is the E4M3 format's own
definition: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinity, NaN at
exponent 15 / mantissa 7, largest finite 448).

Checked against torch's float8_e4m3fn conversions (a library routine of its own), the
format's closed forms and worked values, and planted mistakes."""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth


def torch_codes(x32):
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.isnan(ours).sum() == 2            # 0x7F and 0xFF only


def test_worked_values():
    # exponent field e, mantissa m: (1 + m/8) * 2^(e-7); subnormals m/8 * 2^-6
    cases = {1.0: 0x38, -1.0: 0xB8, 448.0: 0x7E, -448.0: 0xFE, 2.0 ** -9: 0x01, 2.0 ** -6: 0x08,
             0.875 * 2.0 ** -6: 0x07, 1.0625: 0x38, 1.1875: 0x3A, 1.125: 0x39, 240.0: 0x77,
             0.0: 0x00, 2.0 ** -10: 0x00, 3 * 2.0 ** -10: 0x02}
    x = np.array(list(cases), np.float32)
    assert oracle.e4m3_encode(x).tolist() == list(cases.values())
    assert oracle.e4m3_encode(np.array([-0.0], np.float32))[0] == 0x80


def test_saturates_to_448_and_nan():
    x = np.array([448.0, 463.9, 464.0, 500.0, 1e6, 3e38, -1e30], np.float32)
    assert oracle.e4m3_encode(x).tolist() == [0x7E] * 6 + [0xFE]
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_encode_matches_torch_in_range():
    rng = np.random.Generator(np.random.PCG64(11))
    grid = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    grid = grid[np.isfinite(grid)]
    mids = (np.sort(grid)[1:] + np.sort(grid)[:-1]) / 2
    x = np.concatenate([grid, mids, rng.normal(0, 3, 20000), rng.normal(0, 100, 5000),
                        rng.uniform(-2 ** -5, 2 ** -5, 5000)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    assert np.array_equal(oracle.e4m3_encode(x), torch_codes(x))


def test_encode_is_nearest_value():
    rng = np.random.Generator(np.random.PCG64(12))
    x = rng.normal(0, 20, 3000).astype(np.float32)
    x = x[np.abs(x) <= 448]
    vals = oracle.e4m3_decode(oracle.e4m3_encode(x))
    grid = np.unique(oracle.e4m3_decode(np.arange(256, dtype=np.uint8)))
    grid = grid[np.isfinite(grid)]
    best = np.min(np.abs(x.astype(np.float64)[:, None] - grid[None, :]), axis=1)
    assert np.array_equal(np.abs(vals - x.astype(np.float64)), best)


def pool_case(seed, H=2, D=16):
    rng = np.random.Generator(np.random.PCG64(seed))
    past, cand = [9, 0, 21], [3, 2, 4]
    cu = synth.cu_from_lens(np.array(past) + np.array(cand))
    T = int(cu[-1])
    k = synth.normal_bf16(rng, (T, H, D))
    v = synth.normal_bf16(rng, (T, H, D))
    return cu, np.array(past, np.int32), k, v


@pytest.mark.parametrize("ks,vs", [(1.0, 1.0), (0.25, 2.0), (0.037, 1.3)])
def test_pool_write_matches_torch_quantization(ks, vs):
    cu, past, k, v = pool_case(20)
    L, S, n_cap = 2, 4, 24
    slots = np.array([3, 0, 1], np.int32)
    pk = np.full((L, S, 2, n_cap, 16), 0xAB, np.uint8)
    pv = pk.copy()
    oracle.pool_write_e4m3(pk, pv, 1, k, v, cu, past, slots, ks, vs)
    kf = synth.bf16_bits_to_f64(k).astype(np.float32) * (np.float32(1) / np.float32(ks))
    vf = synth.bf16_bits_to_f64(v).astype(np.float32) * (np.float32(1) / np.float32(vs))
    assert np.all(np.abs(kf) <= 448) and np.all(np.abs(vf) <= 448)
    ek, ev = torch_codes(kf), torch_codes(vf)
    for b, (s, n) in enumerate(zip(slots, past)):
        for j in range(n):
            assert np.array_equal(pk[1, s, :, j], ek[cu[b] + j])
            assert np.array_equal(pv[1, s, :, j], ev[cu[b] + j])
    untouched = np.ones(pk.shape, bool)
    for s, n in zip(slots, past):
        untouched[1, s, :, :n] = False
    assert np.all(pk[untouched] == 0xAB) and np.all(pv[untouched] == 0xAB)
    if ks != 1.0:
        # planted mistake: multiplying by the scale instead of dividing by it
        wrong = torch_codes(synth.bf16_bits_to_f64(k).astype(np.float32) * np.float32(ks))
        assert not np.array_equal(pk[1, 3, :, :9], wrong[cu[0]:cu[0] + 9].transpose(1, 0, 2))


def test_dequant_power_of_two_scale_is_exact():
    codes = np.arange(256, dtype=np.uint8)
    codes = codes[np.isfinite(oracle.e4m3_decode(codes))]
    for sc in (1.0, 0.125, 8.0):
        bits = oracle.e4m3_dequant_bf16(codes, sc)
        assert np.array_equal(synth.bf16_bits_to_f64(bits), oracle.e4m3_decode(codes) * sc)


def test_dequant_matches_torch_rounding():
    codes = np.arange(256, dtype=np.uint8)
    codes = codes[np.isfinite(oracle.e4m3_decode(codes))]
    sc = np.float32(0.0371)
    bits = oracle.e4m3_dequant_bf16(codes, float(sc))
    f = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32) * torch.tensor(sc)
    ref = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


def test_decode_e4m3_equals_decode_over_dequantized_pool():
    rng = np.random.Generator(np.random.PCG64(30))
    H, D, S, n_cap = 2, 16, 3, 20
    cand, past = [2, 3], [11, 0]
    cu = synth.cu_from_lens(np.array(cand))
    Tc = int(cu[-1])
    qc, kc, vc = (synth.normal_bf16(rng, (Tc, H, D)) for _ in range(3))
    pk8 = rng.integers(0, 256, (1, S, H, n_cap, D), dtype=np.uint8)
    pv8 = rng.integers(0, 256, (1, S, H, n_cap, D), dtype=np.uint8)
    pk8[(pk8 & 0x7F) == 0x7F] = 0x30     # no NaN codes
    pv8[(pv8 & 0x7F) == 0x7F] = 0x30
    slots = np.array([2, 0], np.int32)
    out = oracle.decode_e4m3(qc, kc, vc, cu, slots, np.array(past, np.int32), pk8, pv8, 0, 0.5, 0.25)
    pk = oracle.e4m3_dequant_bf16(pk8, 0.5)
    pv = oracle.e4m3_dequant_bf16(pv8, 0.25)
    ref = oracle.decode(qc, kc, vc, cu, slots, np.array(past, np.int32), pk, pv, 0)
    assert np.array_equal(out, ref)
    # the scales matter: a swapped pair gives a different result
    swapped = oracle.decode_e4m3(qc, kc, vc, cu, slots, np.array(past, np.int32), pk8, pv8, 0, 0.25, 0.5)
    assert not np.allclose(out[:2], swapped[:2])
