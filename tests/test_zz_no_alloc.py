"""The allocation-free rank decode entry point, checked against the regular one.

unipin_rank_decode_attn_noalloc serves callers that cannot allocate device
memory while they run (their memory belongs to another framework's pool, or
their serving loop must not allocate after start-up): its scratch is a fixed
array inside the library.  This file is collected last on purpose, so a
failure here leaves every other test already run; it also passes alone.
"""

import ctypes

import numpy as np
import pytest
import torch

from kv_cache_reuse_falcon_b200 import synth
from tests.gpu_helpers import DevDecode, fill_pool_rows, nan_pool, parity, to_dev_bf16, to_dev_i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ub():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_reuse_falcon_b200 import binding
    return binding


def _setup(seed, past, cand, H, D, S, n_cap, layer):
    rng = np.random.Generator(np.random.PCG64(seed))
    d = synth.make_decode(seed, past, cand, H, D, n_slots=S, rng=rng)
    ks, vs = synth.pool_rows(rng, past, H, D)
    pk, pv = nan_pool(layer + 1, S, H, n_cap, D)
    fill_pool_rows(pk, pv, layer, d.slot_ids, past, ks, vs)
    return d, DevDecode(d), pk, pv


@pytest.mark.parametrize("shape", [
    # small k: the split-n partial results live in the library's array
    ([2048] * 8, [16] * 8, 4, 64, 12, 2048),
    # ragged lengths, one request without history, D=128
    ([700, 0, 1500, 129], [300, 40, 260, 128], 4, 128, 6, 1536),
])
def test_noalloc_decode_matches_regular_decode_twice_in_a_row(ub, shape):
    past, cand, H, D, S, n_cap = shape
    layer = 1
    d, dd, pk, pv = _setup(7000, past, cand, H, D, S, n_cap, layer)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, layer, dd.max_k,
                              out_fp32=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for _ in range(2):   # the shared array keeps the previous call's contents
        out = torch.full_like(ref, float("nan"))
        ub.rank_decode_attn_noalloc(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, layer, dd.max_k,
                                    out, out_fp32=True, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        parity(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "no-alloc decode")


def test_noalloc_decode_runs_unsplit_beyond_its_array(ub):
    """A shape whose split-n scratch exceeds the fixed array runs without the split: the regular
    decode's result (which splits, with its own workspace) within fp32 rounding."""
    limit = ub.rank_decode_noalloc_scratch_bytes()
    H, D, n_cap = 4, 128, 4096
    R, k = 37, 256          # 148 (request, head) units: under two waves of blocks, so the sweep splits
    assert ub.rank_decode_workspace_size(R, H, D, k, R * k, n_cap) > limit
    past, cand = [1000 + 61 * r for r in range(R)], [k] * R
    layer, S = 0, 40
    d, dd, pk, pv = _setup(7100, past, cand, H, D, S, n_cap, layer)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, layer, dd.max_k,
                              out_fp32=True, dev_status=status)
    out = torch.full_like(ref, float("nan"))
    ub.rank_decode_attn_noalloc(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, layer, dd.max_k,
                                out, out_fp32=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    parity(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "no-alloc decode, unsplit")


def test_noalloc_decode_refuses_an_e4m3_pool_beyond_small_k(ub):
    """With more than 64 candidate columns the engine would need the pool's dequantized rows,
    which do not fit a fixed array: UNSUPPORTED before any launch."""
    P = ctypes.c_void_p
    pool = ub.KVPool(16, 16, 1, 1, 4, 512, 64, ub.POOL_E4M3, 1.0, 1.0)   # never dereferenced
    rc = ub.LIB.unipin_rank_decode_attn_noalloc(P(16), P(16), P(16), P(16), 1, P(16), P(16), P(16), 3, 4, 64,
                                                100, 300, 0.1, ctypes.byref(pool), 0, None, None)
    assert rc == -2


def test_noalloc_decode_over_an_e4m3_pool_with_small_k(ub):
    """The small-candidate kernel reads E4M3 codes itself, so the no-alloc call takes such a pool;
    checked against the oracle's decode over the dequantized rows."""
    import oracle
    H, Hkv, D, S, n_cap, layer = 8, 2, 64, 6, 2048, 0
    past, cand = [2048, 517, 0, 1300], [8, 3, 5, 1]     # 8 x 4 query heads per kv head = 32 columns
    scales = (0.046875, 0.0205078125)     # bfloat16 values: the kernel expands the codes itself
    rng = np.random.Generator(np.random.PCG64(7200))
    cu = synth.cu_from_lens(np.array(cand))
    Tc = int(cu[-1])
    qc = synth.normal_bf16(rng, (Tc, H, D))
    kc = synth.normal_bf16(rng, (Tc, Hkv, D))
    vc = synth.normal_bf16(rng, (Tc, Hkv, D))
    slots = np.array([5, 0, 3, 2], np.int32)
    hk = np.full((1, S, Hkv, n_cap, D), 0x7F, np.uint8)
    hv = hk.copy()
    for s_, n in zip(slots, past):
        hk[0, s_, :, :n] = oracle.e4m3_encode((rng.normal(0, 1, (Hkv, n, D)) / scales[0]).astype(np.float32))
        hv[0, s_, :, :n] = oracle.e4m3_encode((rng.normal(0, 1, (Hkv, n, D)) / scales[1]).astype(np.float32))
    pl = np.array(past, np.int32)
    out = torch.full((Tc, H, D), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ub.rank_decode_attn_noalloc(to_dev_bf16(qc), to_dev_bf16(kc), to_dev_bf16(vc), to_dev_i32(cu), to_dev_i32(slots),
                                to_dev_i32(pl), torch.from_numpy(hk).cuda(), torch.from_numpy(hv).cuda(), layer,
                                max(cand), out, out_fp32=True, dev_status=status, pool_scales=scales)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    ref = oracle.decode_e4m3(qc, kc, vc, cu, slots, pl, hk, hv, 0, *scales)
    parity(out.cpu().numpy(), ref, "no-alloc E4M3 decode")
