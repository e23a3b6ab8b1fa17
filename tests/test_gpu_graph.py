"""The hot path inside a CUDA graph: every call is asynchronous, allocates
nothing and syncs nothing, so a serving loop can capture a whole step (the
prefill with its pool write, then the rank decode of every layer) once and
replay it.  Replays must give the same bits as eager calls, and as the oracle
within the parity tolerance."""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_reuse_falcon_b200 import synth
from tests.gpu_helpers import DevDecode, DevPrefill, fill_pool_rows, host_pool_layer, nan_pool, parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ub():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_reuse_falcon_b200 import binding
    return binding


def test_prefill_and_pool_write_replay_from_a_graph(ub):
    past, cand, H, D, S, L = [300, 17, 129], [100, 140, 3], 2, 128, 5, 2
    batch = synth.make_prefill(7100, past, cand, H, D, n_slots=S)
    dp = DevPrefill(batch)
    pk, pv = nan_pool(L, S, H, max(past), D)
    out = torch.empty(dp.q.shape, dtype=torch.float32, device="cuda")
    ws = torch.empty(64, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call():
        ub.masked_prefill_attn(dp.q, dp.k, dp.v, dp.cu, dp.past, dp.max_seqlen, out=out, out_fp32=True,
                               pool_k=pk, pool_v=pv, slot_ids=dp.slots, layer=1, workspace=ws,
                               dev_status=status, stream=torch.cuda.current_stream())

    call()                                   # first call: one-time set-up, outside the capture
    torch.cuda.synchronize()
    eager = out.clone()
    pool_eager = pk.clone(), pv.clone()
    out.zero_()
    pk.fill_(0), pv.fill_(0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    assert torch.equal(out, eager)
    # the replay rewrote exactly the written rows; the zeroed rest stays zero
    for b, (s, n) in enumerate(zip(batch.slot_ids, past)):
        assert torch.equal(pk[1, int(s), :, :n].view(torch.int16), pool_eager[0][1, int(s), :, :n].view(torch.int16))
        assert torch.equal(pv[1, int(s), :, :n].view(torch.int16), pool_eager[1][1, int(s), :, :n].view(torch.int16))
    ref = oracle.prefill(batch.q, batch.k, batch.v, batch.cu_seqlens, batch.past_lens)
    parity(out.cpu().numpy(), ref, "prefill from a graph")


@pytest.mark.parametrize("split", [False, True])
def test_layered_rank_decode_replays_from_a_graph(ub, split):
    """Every layer's decode in one graph; with a full workspace the small launch
    splits the pool sweep and runs the merge kernel too."""
    R, H, D, S, L, n_cap = 4, 2, 64, 8, 3, 1024
    past = [1000, 257, 1024, 3]
    cand = [16, 3, 9, 1] if split else [130, 64, 300, 1]
    rng = np.random.Generator(np.random.PCG64(7200 + split))
    pk, pv = nan_pool(L, S, H, n_cap, D)
    ds, hosts = [], []
    d0 = synth.make_decode(7200, past, cand, H, D, n_slots=S, rng=rng)
    for layer in range(L):
        ks, vs = synth.pool_rows(rng, past, H, D)
        fill_pool_rows(pk, pv, layer, d0.slot_ids, past, ks, vs)
        hosts.append(host_pool_layer(L, S, H, n_cap, D, layer, d0.slot_ids, past, ks, vs))
        q = synth.normal_bf16(rng, (int(d0.cu_seqlens[-1]), H, D))
        k = synth.normal_bf16(rng, (int(d0.cu_seqlens[-1]), H, D))
        v = synth.normal_bf16(rng, (int(d0.cu_seqlens[-1]), H, D))
        ds.append(synth.DecodeBatch(H, D, d0.past_lens, d0.cand_lens, d0.cu_seqlens, d0.slot_ids, q, k, v))
    dds = [DevDecode(d) for d in ds]
    max_k = max(cand)
    nbytes = ub.rank_decode_workspace_size(R, H, D, max_k, int(d0.cu_seqlens[-1]), n_cap)
    if split:
        assert nbytes > 256
    else:
        nbytes = 256                       # the work counter only: no split
    ws = torch.empty(nbytes // 4 + 4, dtype=torch.float32, device="cuda")
    outs = [torch.empty(dd.q.shape, dtype=torch.float32, device="cuda") for dd in dds]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        s = torch.cuda.current_stream()
        for layer, dd in enumerate(dds):
            ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, layer, max_k,
                                out=outs[layer], out_fp32=True, workspace=ws, dev_status=status, stream=s)

    step()
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    for layer in range(L):
        assert torch.equal(outs[layer], eager[layer]), layer
        hk, hv = hosts[layer]
        d = ds[layer]
        ref = oracle.decode(d.q, d.k, d.v, d.cu_seqlens, d.slot_ids, d.past_lens, hk, hv, 0)
        parity(outs[layer].cpu().numpy(), ref, "decode layer %d from a graph" % layer)


@pytest.mark.parametrize("scales", [(0.03125, 0.0546875), (0.0625, 0.03)])
def test_e4m3_rank_decode_replays_from_a_graph(ub, scales):
    """Two layers of an E4M3 pool: with bfloat16-valued scales the small-k kernel reads the codes in
    place; with 0.03 the call dequantizes into its workspace first (a second kernel in the graph)."""
    R, H, D, S, L, n_cap = 4, 2, 64, 8, 2, 1024
    past, cand = [1000, 257, 1024, 0], [16, 3, 9, 1]
    rng = np.random.Generator(np.random.PCG64(7300))
    d0 = synth.make_decode(7300, past, cand, H, D, n_slots=S, rng=rng)
    hk = np.full((L, S, H, n_cap, D), 0x7F, np.uint8)
    hv = hk.copy()
    for layer in range(L):
        for s_, n in zip(d0.slot_ids, past):
            hk[layer, s_, :, :n] = oracle.e4m3_encode((rng.normal(0, 1, (H, n, D)) / scales[0]).astype(np.float32))
            hv[layer, s_, :, :n] = oracle.e4m3_encode((rng.normal(0, 1, (H, n, D)) / scales[1]).astype(np.float32))
    pk = torch.from_numpy(hk).cuda().view(torch.float8_e4m3fn)
    pv = torch.from_numpy(hv).cuda().view(torch.float8_e4m3fn)
    dd = DevDecode(d0)
    max_k, Tc = max(cand), int(d0.cu_seqlens[-1])
    nbytes = ub.rank_decode_pool_workspace_size(pk, pv, R, H, max_k, Tc, pool_scales=scales)
    ws = torch.empty(nbytes // 4 + 4, dtype=torch.float32, device="cuda")
    outs = [torch.empty(dd.q.shape, dtype=torch.float32, device="cuda") for _ in range(L)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        for layer in range(L):
            ub.rank_decode_attn(dd.q, dd.k, dd.v, dd.cu, dd.slots, dd.past, pk, pv, layer, max_k, out=outs[layer],
                                out_fp32=True, workspace=ws, dev_status=status, stream=torch.cuda.current_stream(),
                                pool_scales=scales)

    step()
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, ub.status_string(int(status.item()))
    for layer in range(L):
        assert torch.equal(outs[layer], eager[layer]), layer
        ref = oracle.decode_e4m3(d0.q, d0.k, d0.v, d0.cu_seqlens, d0.slot_ids, d0.past_lens,
                                 hk[layer:layer + 1], hv[layer:layer + 1], 0, *scales)
        parity(outs[layer].cpu().numpy(), ref, "E4M3 decode layer %d from a graph" % layer)
