"""Seeded synthetic inputs for the masked prefill / pool write / rank decode path.

This module only draws numbers.  It holds none of the attention arithmetic and
imports neither the CUDA binding nor the CPU oracle, so both sides can take
their inputs from here without sharing any of the method's code.

Recipe (the pages fix no input distribution; these choices are ours):

* Generator: ``numpy.random.Generator(PCG64(seed))``.
* Values: ``standard_normal(dtype=float32)``, rounded to bfloat16 (round to
  nearest even), drawn in chunks of at most 2**26 values in C order.  Arrays
  hold the raw bfloat16 bit patterns as ``uint16``.
* Draw order inside one workload: the per-segment lengths (past ``n_b`` then
  candidate ``k_b``), the slot permutation, then Q, K, V, then pool rows.
* Seeds: ``20261202 + i`` for the i-th named workload in ``WORKLOADS``.

Pool rows that no request reads are never drawn: callers fill them with a NaN
pattern (``BF16_NAN``) so that a stray read shows up as NaN in the output.
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

BF16_NAN = np.uint16(0x7FC0)
BASE_SEED = 20261202


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 bit patterns (uint16), via float32, both steps round-to-nearest-even."""
    f = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round-to-nearest-even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64, exact."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


_CHUNK = 1 << 26


def normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) samples as bfloat16 bit patterns of the given shape."""
    shape = tuple(int(x) for x in np.atleast_1d(shape)) if not isinstance(shape, tuple) else shape
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        u = rng.standard_normal(hi - lo, dtype=np.float32).view(np.uint32)
        out[lo:hi] = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    return out.reshape(shape)


@dataclasses.dataclass
class PrefillBatch:
    """One packed prefill batch: B segments ``[n_b past || k_b candidates]``."""

    H: int
    D: int
    past_lens: np.ndarray      # int32 [B]
    cand_lens: np.ndarray      # int32 [B]
    cu_seqlens: np.ndarray     # int32 [B+1]
    q: np.ndarray              # uint16 (bf16 bits) [T, H, D]
    k: np.ndarray
    v: np.ndarray
    slot_ids: Optional[np.ndarray] = None  # int32 [B], distinct

    @property
    def B(self) -> int:
        return int(self.past_lens.shape[0])

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])


@dataclasses.dataclass
class DecodeBatch:
    """R rank-decode requests: request r scores ``k_r`` candidates over slot ``slot_ids[r]``."""

    H: int
    D: int
    past_lens: np.ndarray      # int32 [R]  (n_r cached rows in the slot)
    cand_lens: np.ndarray      # int32 [R]
    cu_seqlens: np.ndarray     # int32 [R+1] over candidates
    slot_ids: np.ndarray       # int32 [R]
    q: np.ndarray              # uint16 [T_c, H, D]
    k: np.ndarray
    v: np.ndarray

    @property
    def R(self) -> int:
        return int(self.past_lens.shape[0])


def cu_from_lens(lens: np.ndarray) -> np.ndarray:
    cu = np.zeros(len(lens) + 1, dtype=np.int64)
    np.cumsum(np.asarray(lens, dtype=np.int64), out=cu[1:])
    if cu[-1] >= 2**31:
        raise ValueError("total tokens exceed int32")
    return cu.astype(np.int32)


def make_prefill(seed: int, past_lens, cand_lens, H: int, D: int,
                 n_slots: Optional[int] = None, rng: Optional[np.random.Generator] = None) -> PrefillBatch:
    """Packed bf16 Q/K/V ~ N(0,1) for the given per-segment lengths.

    If ``n_slots`` is given, also draws distinct slot ids (the first B entries of
    a random permutation of ``range(n_slots)``) before Q, K, V.
    """
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    past = np.asarray(past_lens, dtype=np.int32)
    cand = np.asarray(cand_lens, dtype=np.int32)
    if past.shape != cand.shape:
        raise ValueError("past_lens and cand_lens differ in length")
    slots = None
    if n_slots is not None:
        if n_slots < len(past):
            raise ValueError("fewer slots than segments")
        slots = rng.permutation(n_slots)[: len(past)].astype(np.int32)
    cu = cu_from_lens(past + cand)
    T = int(cu[-1])
    q = normal_bf16(rng, (T, H, D))
    k = normal_bf16(rng, (T, H, D))
    v = normal_bf16(rng, (T, H, D))
    return PrefillBatch(H=H, D=D, past_lens=past, cand_lens=cand, cu_seqlens=cu,
                        q=q, k=k, v=v, slot_ids=slots)


def make_decode(seed: int, past_lens, cand_lens, H: int, D: int, n_slots: int,
                rng: Optional[np.random.Generator] = None) -> DecodeBatch:
    """Candidate Q/K/V plus distinct slot ids for R decode requests."""
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    past = np.asarray(past_lens, dtype=np.int32)
    cand = np.asarray(cand_lens, dtype=np.int32)
    if n_slots < len(past):
        raise ValueError("fewer slots than requests")
    slots = rng.permutation(n_slots)[: len(past)].astype(np.int32)
    cu = cu_from_lens(cand)
    T = int(cu[-1])
    q = normal_bf16(rng, (T, H, D))
    k = normal_bf16(rng, (T, H, D))
    v = normal_bf16(rng, (T, H, D))
    return DecodeBatch(H=H, D=D, past_lens=past, cand_lens=cand, cu_seqlens=cu,
                       slot_ids=slots, q=q, k=k, v=v)


def pool_rows(rng: np.random.Generator, past_lens, H: int, D: int):
    """Per-request cached rows ``[H, n_r, D]`` (bf16 bits), drawn in request order, K then V."""
    ks, vs = [], []
    for n in np.asarray(past_lens):
        ks.append(normal_bf16(rng, (H, int(n), D)))
        vs.append(normal_bf16(rng, (H, int(n), D)))
    return ks, vs


def ragged_lengths(rng: np.random.Generator, B: int, n_lo: int, n_hi: int, k_lo: int, k_hi: int):
    """Integer lengths n ~ U{n_lo..n_hi}, then k ~ U{k_lo..k_hi} (inclusive)."""
    n = rng.integers(n_lo, n_hi + 1, size=B).astype(np.int32)
    k = rng.integers(k_lo, k_hi + 1, size=B).astype(np.int32)
    return n, k


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str          # "prefill", "prefill+pool", "decode", "ragged", "backward"
    B: int
    H: int
    D: int
    n: int = 0         # fixed past length (0 for ragged)
    k: int = 0         # fixed candidate count (0 for ragged)
    L: int = 0         # pool layers
    S: int = 0         # pool slots
    n_cap: int = 0     # pool rows per slot
    ragged: Optional[tuple] = None   # (n_lo, n_hi, k_lo, k_hi)
    layers_per_step: int = 1

    @property
    def seed(self) -> int:
        return BASE_SEED + [w.name for w in WORKLOADS].index(self.name)

    def lengths(self, rng: np.random.Generator):
        if self.ragged is not None:
            return ragged_lengths(rng, self.B, *self.ragged)
        return (np.full(self.B, self.n, dtype=np.int32), np.full(self.B, self.k, dtype=np.int32))


# The five workloads, in the order the pages' serving shapes were turned into
# synthetic cases, plus the L40S latency-table shape (B=8, n=992, k=656).
WORKLOADS: List[Workload] = [
    Workload("tiny_prefill_B2_H2_D32_n64_k16", "prefill", B=2, H=2, D=32, n=64, k=16),
    Workload("prefill_B64_H8_D64_n256_k128", "prefill", B=64, H=8, D=64, n=256, k=128),
    Workload("prefill_pool_B128_H8_D64_n1024_k512", "prefill+pool", B=128, H=8, D=64, n=1024, k=512,
             L=12, S=256, n_cap=1024),
    Workload("decode_R32_H8_D64_n2048_k1000_L12", "decode", B=32, H=8, D=64, n=2048, k=1000,
             L=12, S=256, n_cap=2048, layers_per_step=12),
    Workload("ragged_B256_H8_D128_n32-4096_k50-2000", "ragged", B=256, H=8, D=128,
             L=1, S=256, n_cap=4096, ragged=(32, 4096, 50, 2000)),
    Workload("table2_B8_H8_D64_n992_k656", "prefill", B=8, H=8, D=64, n=992, k=656),
    # gradients of the masked prefill (joint training) at the prefill shape
    Workload("backward_B64_H8_D64_n256_k128", "backward", B=64, H=8, D=64, n=256, k=128),
]


def workload(name: str) -> Workload:
    for w in WORKLOADS:
        if w.name == name or w.name.startswith(name):
            return w
    raise KeyError(name)
