"""Shared helpers for the GPU tests: device copies of seeded inputs and the parity metric."""

import numpy as np
import torch

from kv_cache_reuse_falcon_b200 import synth

MAX_ABS = 1e-2      # tolerance on the fp32 output, element-wise
REL_L2 = 2e-3       # ||O_gpu - O_ref||_2 / ||O_ref||_2 over the compared tensor


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def to_dev_i32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def bf16_tensor_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def nan_pool(L, S, H, n_cap, D, device="cuda"):
    """Two pool tensors filled with the bf16 NaN pattern 0x7FC0."""
    k = torch.full((L, S, H, n_cap, D), 0x7FC0, dtype=torch.int16, device=device).view(torch.bfloat16)
    v = torch.full((L, S, H, n_cap, D), 0x7FC0, dtype=torch.int16, device=device).view(torch.bfloat16)
    return k, v


def parity(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), "%s: non-finite output" % what
    err = gpu - ref
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)) if err.size else 0.0
    assert max_abs <= MAX_ABS and rel <= REL_L2, "%s: max_abs=%.3e rel_l2=%.3e" % (what, max_abs, rel)
    return max_abs, rel


class DevPrefill:
    """A PrefillBatch copied to the device."""

    def __init__(self, batch: synth.PrefillBatch, device="cuda"):
        self.batch = batch
        self.q = to_dev_bf16(batch.q, device)
        self.k = to_dev_bf16(batch.k, device)
        self.v = to_dev_bf16(batch.v, device)
        self.cu = to_dev_i32(batch.cu_seqlens, device)
        self.past = to_dev_i32(batch.past_lens, device)
        self.slots = to_dev_i32(batch.slot_ids, device) if batch.slot_ids is not None else None
        lens = np.diff(batch.cu_seqlens)
        self.max_seqlen = int(lens.max()) if lens.size else 0
        self.max_past = int(batch.past_lens.max()) if batch.past_lens.size else 0


class DevDecode:
    def __init__(self, d: synth.DecodeBatch, device="cuda"):
        self.d = d
        self.q = to_dev_bf16(d.q, device)
        self.k = to_dev_bf16(d.k, device)
        self.v = to_dev_bf16(d.v, device)
        self.cu = to_dev_i32(d.cu_seqlens, device)
        self.past = to_dev_i32(d.past_lens, device)
        self.slots = to_dev_i32(d.slot_ids, device)
        self.max_k = int(d.cand_lens.max()) if d.cand_lens.size else 0


def fill_pool_rows(pool_k: torch.Tensor, pool_v: torch.Tensor, layer: int, slots, past_lens, ks, vs):
    """Write per-request cached rows ([H, n, D] bf16 bits) into the device pool slots."""
    for s, n, kb, vb in zip(slots, past_lens, ks, vs):
        n = int(n)
        if n == 0:
            continue
        pool_k[layer, int(s), :, :n, :] = to_dev_bf16(kb, pool_k.device)
        pool_v[layer, int(s), :, :n, :] = to_dev_bf16(vb, pool_v.device)


def host_pool_layer(L, S, H, n_cap, D, layer, slots, past_lens, ks, vs):
    """Host mirror of one layer of the pool ([1, S, H, n_cap, D] NaN-filled + the cached rows)."""
    pk = np.full((1, S, H, n_cap, D), synth.BF16_NAN, dtype=np.uint16)
    pv = pk.copy()
    for s, n, kb, vb in zip(slots, past_lens, ks, vs):
        n = int(n)
        pk[0, int(s), :, :n, :] = kb
        pv[0, int(s), :, :n, :] = vb
    return pk, pv
