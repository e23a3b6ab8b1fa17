"""GPU parity for the E4M3 pool variant.

The pool stores E4M3 codes of k / k_scale and v / v_scale (float32 product,
nearest even, saturating at 448); attention reads code c as
bfloat16(value(c) * scale).  Checked against the oracle: the pool bytes
bit for bit (the pool write and the prefill's write into an E4M3 pool), and
the rank decode over an E4M3 pool element by element at the decode tolerance
(both the small-candidate kernel, which expands the codes in shared memory,
and the many-candidate engine, which decodes a dequantized copy, each with and
without split-n).  With power-of-two scales the dequantized rows are exact, so
a decode over the E4M3 pool must equal, bit for bit, the decode over a bfloat16
pool that holds those rows.
"""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth
from tests.gpu_helpers import bf16_tensor_bits, parity, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ub():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_reuse_falcon_b200 import binding
    return binding


def codes_pool(shape, fill=0xAB):
    k = torch.full(shape, fill, dtype=torch.uint8, device="cuda")
    return k, k.clone()


def segs(seed, past, cand, H, D):
    rng = np.random.Generator(np.random.PCG64(seed))
    cu = synth.cu_from_lens(np.array(past) + np.array(cand))
    T = int(cu[-1])
    k = synth.normal_bf16(rng, (T, H, D))
    v = synth.normal_bf16(rng, (T, H, D))
    return rng, cu, np.array(past, np.int32), k, v


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("scales", [(1.0, 1.0), (0.25, 2.0), (0.037, 1.3), (0.002, 0.004)])
def test_pool_write_e4m3_bit_exact(ub, D, scales):
    H, L, S, n_cap = 2, 2, 5, 300
    past, cand = [130, 0, 257, 1], [3, 4, 0, 2]
    _, cu, pl, k, v = segs(100 + D, past, cand, H, D)
    slots = np.array([4, 0, 2, 1], np.int32)
    pk, pv = codes_pool((L, S, H, n_cap, D))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ub.kvpool_write(pk, pv, 1, to_dev_bf16(k), to_dev_bf16(v), to_dev_i32(cu), to_dev_i32(pl), to_dev_i32(slots),
                    max(past), dev_status=status, pool_scales=scales)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    hk = np.full((L, S, H, n_cap, D), 0xAB, np.uint8)
    hv = hk.copy()
    oracle.pool_write_e4m3(hk, hv, 1, k, v, cu, pl, slots, *scales)
    assert pk.cpu().numpy().tobytes() == hk.tobytes()
    assert pv.cpu().numpy().tobytes() == hv.tobytes()


@pytest.mark.parametrize("H,Hkv,D", [(4, 4, 128), (8, 2, 64)])
def test_prefill_into_e4m3_pool(ub, H, Hkv, D):
    past, cand = [200, 0, 70, 513], [40, 9, 1, 130]
    rng = np.random.Generator(np.random.PCG64(7300 + D))
    cu = synth.cu_from_lens(np.array(past) + np.array(cand))
    T = int(cu[-1])
    q = synth.normal_bf16(rng, (T, H, D))
    k = synth.normal_bf16(rng, (T, Hkv, D))
    v = synth.normal_bf16(rng, (T, Hkv, D))
    pl = np.array(past, np.int32)
    slots = np.array([5, 0, 3, 1], np.int32)
    L, S, n_cap = 2, 6, 700
    pk, pv = codes_pool((L, S, Hkv, n_cap, D))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ub.masked_prefill_attn(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), to_dev_i32(cu), to_dev_i32(pl),
                                 int(np.diff(cu).max()), out_fp32=True, pool_k=pk, pool_v=pv,
                                 slot_ids=to_dev_i32(slots), layer=1, dev_status=status, pool_scales=(0.5, 0.125))
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    parity(out.cpu().numpy(), oracle.prefill(q, k, v, cu, pl), "prefill with an E4M3 pool")
    hk = np.full((L, S, Hkv, n_cap, D), 0xAB, np.uint8)
    hv = hk.copy()
    oracle.pool_write_e4m3(hk, hv, 1, k, v, cu, pl, slots, 0.5, 0.125)
    assert pk.cpu().numpy().tobytes() == hk.tobytes()
    assert pv.cpu().numpy().tobytes() == hv.tobytes()


DECODE = [
    # (cand lens, H, Hkv, D): small-k kernel (k * G <= 64) and the many-candidate engine
    ([16, 3, 12, 1], 8, 8, 64),
    ([1, 1, 1, 1], 8, 2, 64),
    ([30, 12, 5, 32], 4, 4, 128),
    ([16, 9, 2, 13], 8, 2, 64),      # 64 candidate columns at D=64: decoded from a dequantized copy
    ([64, 20, 1, 50], 2, 2, 128),
    ([100, 40, 3, 77], 4, 2, 64),
    ([200, 1, 150, 7], 2, 2, 128),
]


def decode_case(seed, cand, H, Hkv, D, scales):
    past = [2048, 0, 129, 1000]
    S, n_cap, layer = 8, 2048, 1
    rng = np.random.Generator(np.random.PCG64(seed))
    cu = synth.cu_from_lens(np.array(cand))
    Tc = int(cu[-1])
    qc = synth.normal_bf16(rng, (Tc, H, D))
    kc = synth.normal_bf16(rng, (Tc, Hkv, D))
    vc = synth.normal_bf16(rng, (Tc, Hkv, D))
    slots = rng.permutation(S)[:4].astype(np.int32)
    hk = np.full((layer + 1, S, Hkv, n_cap, D), 0x7F, np.uint8)     # NaN codes outside the written rows
    hv = hk.copy()
    for s, n in zip(slots, past):
        if n:
            # codes of N(0, 1) keys/values under the given scales
            kr = oracle.e4m3_encode((rng.normal(0, 1, (Hkv, n, D)) / scales[0]).astype(np.float32))
            vr = oracle.e4m3_encode((rng.normal(0, 1, (Hkv, n, D)) / scales[1]).astype(np.float32))
            hk[layer, s, :, :n], hv[layer, s, :, :n] = kr, vr
    return qc, kc, vc, cu, slots, np.array(past, np.int32), hk, hv, layer, Tc


# scales that are bfloat16 values: the small-k kernel expands the codes in shared
# memory; 0.03 is not one, so those decodes take the dequantized copy
SCALES = [(0.046875, 0.0302734375), (0.0625, 0.03)]


@pytest.mark.parametrize("case", range(len(DECODE)))
@pytest.mark.parametrize("mode", ["none", "split"])
@pytest.mark.parametrize("scales", SCALES)
def test_rank_decode_over_e4m3_pool(ub, case, mode, scales):
    cand, H, Hkv, D = DECODE[case]
    qc, kc, vc, cu, slots, pl, hk, hv, layer, Tc = decode_case(7400 + case, cand, H, Hkv, D, scales)
    pk = torch.from_numpy(hk).cuda().view(torch.float8_e4m3fn)
    pv = torch.from_numpy(hv).cuda().view(torch.float8_e4m3fn)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = "auto"
    if mode == "none":
        # no room for split-n partials (the engine still gets its dequantized rows)
        nbytes = ub.rank_decode_pool_workspace_size(pk, pv, 4, H, max(cand), Tc, pool_scales=scales)
        base = ub.rank_decode_workspace_size(4, H, D, max(cand), Tc, 2048, H_kv=Hkv)
        ws = torch.empty((nbytes - base + 256) // 4, dtype=torch.float32, device="cuda")
    out = ub.rank_decode_attn(to_dev_bf16(qc), to_dev_bf16(kc), to_dev_bf16(vc), to_dev_i32(cu), to_dev_i32(slots),
                              to_dev_i32(pl), pk, pv, layer, max(cand), out_fp32=True, workspace=ws,
                              dev_status=status, pool_scales=scales)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    ref = oracle.decode_e4m3(qc, kc, vc, cu, slots, pl, hk[layer:layer + 1], hv[layer:layer + 1], 0, *scales)
    parity(out.cpu().numpy(), ref, "E4M3 decode case %d %s" % (case, mode))


@pytest.mark.parametrize("case", [0, 1, 2, 5])
@pytest.mark.parametrize("scales", [(0.125, 0.0625), (0.0546875, 3.0), (2.0 ** -110, 2.0 ** 100), (300.0, 1.0)])
def test_e4m3_decode_equals_bf16_decode_of_dequantized_rows(ub, case, scales):
    """Every finite code, subnormals and both zeros included, under bfloat16-valued scales (one
    product and two products, small and large): the small-k kernel's in-place expansion gives the
    bfloat16 rows the oracle dequantizes, so its decode equals, bit for bit, the decode of a
    bfloat16 pool holding those rows (both run the same kernel with the same split)."""
    cand, H, Hkv, D = DECODE[case]
    qc, kc, vc, cu, slots, pl, hk, hv, layer, Tc = decode_case(7500 + case, cand, H, Hkv, D, scales)
    rng = np.random.Generator(np.random.PCG64(7550 + case))
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    for s_, n in zip(slots, pl):
        hk[layer, s_, :, :n] = rng.choice(finite, size=(Hkv, n, D))
        hv[layer, s_, :, :n] = rng.choice(finite, size=(Hkv, n, D))
    args = (to_dev_bf16(qc), to_dev_bf16(kc), to_dev_bf16(vc), to_dev_i32(cu), to_dev_i32(slots), to_dev_i32(pl))
    out8 = ub.rank_decode_attn(*args, torch.from_numpy(hk).cuda(), torch.from_numpy(hv).cuda(), layer, max(cand),
                               out_fp32=True, pool_scales=scales)
    bk = to_dev_bf16(oracle.e4m3_dequant_bf16(hk, scales[0]))
    bv = to_dev_bf16(oracle.e4m3_dequant_bf16(hv, scales[1]))
    out16 = ub.rank_decode_attn(*args, bk, bv, layer, max(cand), out_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(out8, out16)


@pytest.mark.parametrize("scales", SCALES)
def test_e4m3_decode_rejects_bad_slot_with_zero_rows(ub, scales):
    cand, H, Hkv, D = DECODE[0]
    qc, kc, vc, cu, slots, pl, hk, hv, layer, Tc = decode_case(7600, cand, H, Hkv, D, scales)
    slots = slots.copy()
    slots[2] = 99
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ub.rank_decode_attn(to_dev_bf16(qc), to_dev_bf16(kc), to_dev_bf16(vc), to_dev_i32(cu), to_dev_i32(slots),
                              to_dev_i32(pl), torch.from_numpy(hk).cuda(), torch.from_numpy(hv).cuda(), layer,
                              max(cand), out_fp32=True, dev_status=status, pool_scales=scales)
    torch.cuda.synchronize()
    assert int(status.item()) == -4
    o = out.cpu().numpy()
    assert np.all(o[cu[2]:cu[3]] == 0)
    good = [r for r in range(4) if r != 2]
    ref = oracle.decode_e4m3(qc, kc, vc, cu, np.where(slots == 99, 0, slots).astype(np.int32), pl,
                             hk[layer:layer + 1], hv[layer:layer + 1], 0, *scales)
    for r in good:
        parity(o[cu[r]:cu[r + 1]], ref[cu[r]:cu[r + 1]], "E4M3 decode, request %d beside a rejected one" % r)


def test_e4m3_pool_needs_a_workspace_in_the_engine(ub):
    cand, H, Hkv, D = DECODE[5]
    qc, kc, vc, cu, slots, pl, hk, hv, layer, Tc = decode_case(7700, cand, H, Hkv, D, (1.0, 1.0))
    with pytest.raises(ub.UnipinError):
        ub.rank_decode_attn(to_dev_bf16(qc), to_dev_bf16(kc), to_dev_bf16(vc), to_dev_i32(cu), to_dev_i32(slots),
                            to_dev_i32(pl), torch.from_numpy(hk).cuda(), torch.from_numpy(hv).cuda(), layer,
                            max(cand), workspace=None)


def test_e4m3_small_k_decode_needs_no_workspace(ub):
    """The small-candidate kernel reads the codes itself (scales that are bfloat16 values):
    without a workspace it runs unsplit."""
    cand, H, Hkv, D = DECODE[4]
    scales = SCALES[0]
    qc, kc, vc, cu, slots, pl, hk, hv, layer, Tc = decode_case(7800, cand, H, Hkv, D, scales)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ub.rank_decode_attn(to_dev_bf16(qc), to_dev_bf16(kc), to_dev_bf16(vc), to_dev_i32(cu), to_dev_i32(slots),
                              to_dev_i32(pl), torch.from_numpy(hk).cuda(), torch.from_numpy(hv).cuda(), layer,
                              max(cand), out_fp32=True, workspace=None, dev_status=status, pool_scales=scales)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    ref = oracle.decode_e4m3(qc, kc, vc, cu, slots, pl, hk[layer:layer + 1], hv[layer:layer + 1], 0, *scales)
    parity(out.cpu().numpy(), ref, "E4M3 small-k decode without a workspace")


@pytest.mark.parametrize("case", [0, 4, 3])
@pytest.mark.parametrize("scales", SCALES)
def test_e4m3_nan_codes_poison_their_head_only(ub, case, scales):
    """A NaN code (0x7F / 0xFF) in a history row that is read poisons that request's outputs of that
    key/value head - the whole rows for a key, the one element for a value - as in the oracle's
    decode; every other output matches the oracle."""
    cand, H, Hkv, D = DECODE[case]
    qc, kc, vc, cu, slots, pl, hk, hv, layer, Tc = decode_case(7900 + case, cand, H, Hkv, D, scales)
    G = H // Hkv
    hv[layer, slots[0], 1, 1500, 7] = 0x7F      # request 0, kv head 1: a V row
    hk[layer, slots[3], 0, 3, 60] = 0xFF        # request 3, kv head 0: a K row
    hk[layer, slots[2], 1, 200, 0] = 0x7F       # request 2: beyond its 129 rows, never read
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ub.rank_decode_attn(to_dev_bf16(qc), to_dev_bf16(kc), to_dev_bf16(vc), to_dev_i32(cu), to_dev_i32(slots),
                              to_dev_i32(pl), torch.from_numpy(hk).cuda(), torch.from_numpy(hv).cuda(), layer,
                              max(cand), out_fp32=True, dev_status=status, pool_scales=scales)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o = out.cpu().numpy()
    ref = oracle.decode_e4m3(qc, kc, vc, cu, slots, pl, hk[layer:layer + 1], hv[layer:layer + 1], 0, *scales)
    poisoned = np.zeros(o.shape, bool)
    poisoned[cu[0]:cu[1], G:2 * G, 7] = True     # a NaN value: its element of every output row
    poisoned[cu[3]:cu[4], 0:G, :] = True         # a NaN key: its score, so the whole row
    assert np.isnan(ref[poisoned]).all()
    assert np.isnan(o[poisoned]).all()
    parity(o[~poisoned], ref[~poisoned], "E4M3 decode beside NaN codes")
