"""Python binding of the C ABI in ``include/unipin.h``.

Argument marshalling only: torch tensors supply device pointers and the
current CUDA stream; every step of the computation runs in the CUDA kernels of
``libunipin.so``.  If the library is missing or fails to load, importing this
module raises: there is no fallback.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libunipin.so")

UNIPIN_OK = 0
STATUS_NAMES = {
    0: "UNIPIN_OK",
    -1: "UNIPIN_ERR_INVALID_ARG",
    -2: "UNIPIN_ERR_UNSUPPORTED",
    -3: "UNIPIN_ERR_MISALIGNED",
    -4: "UNIPIN_ERR_OUT_OF_RANGE",
    -5: "UNIPIN_ERR_CUDA",
    -6: "UNIPIN_ERR_DEVICE_TIMEOUT",
}

EXPORTS = (
    "unipin_masked_prefill_attn",
    "unipin_masked_prefill_bwd",
    "unipin_masked_prefill_bwd_workspace_size",
    "unipin_kvpool_write",
    "unipin_rank_decode_attn",
    "unipin_rank_decode_workspace_size",
    "unipin_rank_decode_pool_workspace_size",
    "unipin_masked_prefill_workspace_size",
    "unipin_status_string",
    "unipin_selftest_bounded_wait",
    "unipin_selftest_exp2",
    "unipin_rank_decode_attn_noalloc",
    "unipin_rank_decode_noalloc_scratch_bytes",
    "unipin_kvpool_share_export",
    "unipin_kvpool_share_open",
    "unipin_kvpool_share_close",
    "unipin_slot_ring_create",
    "unipin_slot_ring_acquire",
    "unipin_slot_ring_release",
    "unipin_slot_ring_free_count",
    "unipin_slot_ring_destroy",
)


class UnipinError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (where, STATUS_NAMES.get(code, "?"), code))


POOL_BF16, POOL_E4M3 = 0, 1    # unipin_pool_dtype


class KVPool(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("L", ctypes.c_int), ("S", ctypes.c_int),
                ("H", ctypes.c_int), ("n_cap", ctypes.c_int), ("D", ctypes.c_int), ("dtype", ctypes.c_int),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


class KVPoolShare(ctypes.Structure):
    """unipin_kvpool_share: IPC handles, offsets and shape of a pool (plain bytes)."""
    _fields_ = [("k_handle", ctypes.c_ubyte * 64), ("v_handle", ctypes.c_ubyte * 64),
                ("k_offset", ctypes.c_ulonglong), ("v_offset", ctypes.c_ulonglong),
                ("L", ctypes.c_int), ("S", ctypes.c_int), ("H", ctypes.c_int), ("n_cap", ctypes.c_int),
                ("D", ctypes.c_int), ("dtype", ctypes.c_int), ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


def _load(path: str = _LIB_PATH):
    if not os.path.exists(path):
        raise ImportError("libunipin.so not built (run __graft_entry__.build() or "
                          "python kv_cache_reuse_falcon_b200/build.py): %s" % path)
    lib = ctypes.CDLL(path)
    P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.unipin_masked_prefill_attn.argtypes = [P, P, P, P, I, P, P, P, I, I, I, I, I, I, F, P, P, I, P, SZ, P, P]
    lib.unipin_masked_prefill_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, SZ, P, P]
    lib.unipin_masked_prefill_bwd.restype = I
    lib.unipin_masked_prefill_bwd_workspace_size.argtypes = [I, I]
    lib.unipin_masked_prefill_bwd_workspace_size.restype = SZ
    lib.unipin_masked_prefill_workspace_size.argtypes = []
    lib.unipin_masked_prefill_workspace_size.restype = SZ
    lib.unipin_masked_prefill_attn.restype = I
    lib.unipin_kvpool_write.argtypes = [P, I, P, P, P, P, P, I, I, I, P, P]
    lib.unipin_kvpool_write.restype = I
    lib.unipin_rank_decode_attn.argtypes = [P, P, P, P, I, P, P, P, I, I, I, I, I, F, P, I, P, SZ, P, P]
    lib.unipin_rank_decode_attn.restype = I
    lib.unipin_rank_decode_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.unipin_rank_decode_workspace_size.restype = SZ
    lib.unipin_rank_decode_pool_workspace_size.argtypes = [P, I, I, I, I]
    lib.unipin_rank_decode_pool_workspace_size.restype = SZ
    lib.unipin_status_string.argtypes = [I]
    lib.unipin_status_string.restype = ctypes.c_char_p
    lib.unipin_selftest_bounded_wait.argtypes = [P, ctypes.c_uint, P]
    lib.unipin_selftest_bounded_wait.restype = I
    lib.unipin_selftest_exp2.argtypes = [P, P, I, P]
    lib.unipin_selftest_exp2.restype = I
    lib.unipin_rank_decode_attn_noalloc.argtypes = [P, P, P, P, I, P, P, P, I, I, I, I, I, F, P, I, P, P]
    lib.unipin_rank_decode_attn_noalloc.restype = I
    lib.unipin_rank_decode_noalloc_scratch_bytes.argtypes = []
    lib.unipin_rank_decode_noalloc_scratch_bytes.restype = SZ
    lib.unipin_kvpool_share_export.argtypes = [P, P]
    lib.unipin_kvpool_share_export.restype = I
    lib.unipin_kvpool_share_open.argtypes = [P, P]
    lib.unipin_kvpool_share_open.restype = I
    lib.unipin_kvpool_share_close.argtypes = [P, P]
    lib.unipin_kvpool_share_close.restype = I
    lib.unipin_slot_ring_create.argtypes = [I, ctypes.POINTER(P)]
    lib.unipin_slot_ring_create.restype = I
    lib.unipin_slot_ring_acquire.argtypes = [P, I, ctypes.POINTER(I)]
    lib.unipin_slot_ring_acquire.restype = I
    lib.unipin_slot_ring_release.argtypes = [P, I, ctypes.POINTER(I)]
    lib.unipin_slot_ring_release.restype = I
    lib.unipin_slot_ring_free_count.argtypes = [P]
    lib.unipin_slot_ring_free_count.restype = I
    lib.unipin_slot_ring_destroy.argtypes = [P]
    lib.unipin_slot_ring_destroy.restype = None
    return lib


LIB = _load()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != UNIPIN_OK:
        raise UnipinError(rc, where)


def _tokens(t: torch.Tensor, name: str, D: Optional[int] = None):
    if t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous() or not t.is_cuda:
        raise ValueError("%s must be a contiguous CUDA bfloat16 tensor [T, H, D]" % name)
    if D is not None and t.shape[2] != D:
        raise ValueError("%s has head dim %d, expected %d" % (name, t.shape[2], D))


def _kv_heads(q, k, v) -> int:
    """Key/value heads of grouped-query inputs (k and v [T, H_kv, D], H a multiple of H_kv)."""
    if k.shape != v.shape or k.shape[0] != q.shape[0]:
        raise ValueError("k and v must be [T, H_kv, D] with the tokens of q")
    if q.shape[1] % k.shape[1] != 0:
        raise ValueError("query heads (%d) must be a multiple of key/value heads (%d)" % (q.shape[1], k.shape[1]))
    return int(k.shape[1])


def _index(t: torch.Tensor, name: str, n: int):
    if t.dtype != torch.int32 or t.dim() != 1 or t.shape[0] != n or not t.is_contiguous() or not t.is_cuda:
        raise ValueError("%s must be a contiguous CUDA int32 tensor of length %d" % (name, n))


_E4M3_TYPES = (torch.float8_e4m3fn, torch.uint8)


def _pool(pool_k: torch.Tensor, pool_v: torch.Tensor, pool_scales=None) -> KVPool:
    """A pool descriptor: bfloat16 tensors, or E4M3 codes (float8_e4m3fn or uint8) with
    pool_scales = (k_scale, v_scale) (default (1, 1))."""
    for name, t in (("pool_k", pool_k), ("pool_v", pool_v)):
        if (t.dtype != torch.bfloat16 and t.dtype not in _E4M3_TYPES) or t.dim() != 5 or not t.is_contiguous() \
                or not t.is_cuda:
            raise ValueError("%s must be a contiguous CUDA tensor [L, S, H, n_cap, D] of bfloat16 or E4M3 codes "
                             "(float8_e4m3fn or uint8)" % name)
    if pool_k.shape != pool_v.shape or (pool_k.dtype == torch.bfloat16) != (pool_v.dtype == torch.bfloat16):
        raise ValueError("pool_k and pool_v differ in shape or element type")
    L, S, H, n_cap, D = pool_k.shape
    if pool_k.dtype == torch.bfloat16:
        return KVPool(pool_k.data_ptr(), pool_v.data_ptr(), L, S, H, n_cap, D, POOL_BF16, 1.0, 1.0)
    ks, vs = (1.0, 1.0) if pool_scales is None else (float(pool_scales[0]), float(pool_scales[1]))
    return KVPool(pool_k.data_ptr(), pool_v.data_ptr(), L, S, H, n_cap, D, POOL_E4M3, ks, vs)


def _workspace(workspace, nbytes: int, device):
    """'auto': a fresh device buffer of nbytes; None: no workspace; else the given tensor."""
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a CUDA tensor")
        if nbytes <= 0:
            return None, 0
        workspace = torch.empty((nbytes + 15) // 16 * 4, dtype=torch.float32, device=device)
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace, workspace.numel() * workspace.element_size()


def masked_prefill_workspace_size() -> int:
    return int(LIB.unipin_masked_prefill_workspace_size())


def masked_prefill_attn(q, k, v, cu_seqlens, past_lens, max_seqlen: int, out=None, out_fp32: bool = True,
                        scale: Optional[float] = None, pool_k=None, pool_v=None, slot_ids=None, layer: int = 0,
                        workspace="auto", dev_status=None, stream=None, lse=None, pool_scales=None):
    """M-FALCON masked prefill; optionally also writes the past K/V into pool slots (an E4M3 pool
    takes pool_scales = (k_scale, v_scale)) and the per-row log-sum-exp (base 2, fp32 [T, H]) into `lse`."""
    _tokens(q, "q")
    T, H, D = q.shape
    _tokens(k, "k", D)
    _tokens(v, "v", D)
    H_kv = _kv_heads(q, k, v)
    B = past_lens.shape[0]
    _index(cu_seqlens, "cu_seqlens", B + 1)
    _index(past_lens, "past_lens", B)
    if out is None:
        out = torch.empty((T, H, D), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
    elif out.dtype != (torch.float32 if out_fp32 else torch.bfloat16) or out.shape != q.shape or not out.is_contiguous():
        raise ValueError("out has the wrong dtype or shape")
    pool = None
    if pool_k is not None:
        pool = _pool(pool_k, pool_v, pool_scales)
        _index(slot_ids, "slot_ids", B)
    if lse is not None and (lse.dtype != torch.float32 or lse.shape != (T, H) or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 tensor [T, H]")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws, ws_bytes = _workspace(workspace, masked_prefill_workspace_size(), q.device)
    rc = LIB.unipin_masked_prefill_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), int(bool(out_fp32)), _ptr(lse),
                                        _ptr(cu_seqlens), _ptr(past_lens), B, H, H_kv, D, int(max_seqlen), T, scale,
                                        ctypes.byref(pool) if pool is not None else None,
                                        _ptr(slot_ids) if pool is not None else None, int(layer),
                                        _ptr(ws), ws_bytes, _ptr(dev_status), _stream(stream))
    _check(rc, "unipin_masked_prefill_attn")
    return out


def masked_prefill_bwd_workspace_size(total_tokens: int, H: int) -> int:
    return int(LIB.unipin_masked_prefill_bwd_workspace_size(int(total_tokens), int(H)))


def masked_prefill_bwd(q, k, v, out, dout, lse, cu_seqlens, past_lens, max_seqlen: int, scale: Optional[float] = None,
                       dq=None, dk=None, dv=None, workspace="auto", dev_status=None, stream=None):
    """Gradients (dq, dk, dv), fp32 [T, H, D], of the masked prefill for the upstream gradient dout.

    `out` is the forward's bf16 output and `lse` the row statistic the forward wrote."""
    _tokens(q, "q")
    T, H, D = q.shape
    for name, t in (("k", k), ("v", v), ("out", out), ("dout", dout)):
        _tokens(t, name, D)
    H_kv = _kv_heads(q, k, v)
    if lse.dtype != torch.float32 or lse.shape != (T, H) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor [T, H]")
    B = past_lens.shape[0]
    _index(cu_seqlens, "cu_seqlens", B + 1)
    _index(past_lens, "past_lens", B)
    grads = []
    for g, heads in ((dq, H), (dk, H_kv), (dv, H_kv)):
        if g is None:
            g = torch.empty((T, heads, D), dtype=torch.float32, device=q.device)
        elif g.dtype != torch.float32 or tuple(g.shape) != (T, heads, D) or not g.is_contiguous():
            raise ValueError("gradient outputs must be contiguous float32: dq [T, H, D], dk and dv [T, H_kv, D]")
        grads.append(g)
    ws, ws_bytes = _workspace(workspace, masked_prefill_bwd_workspace_size(T, H), q.device)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    rc = LIB.unipin_masked_prefill_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                                       _ptr(grads[0]), _ptr(grads[1]), _ptr(grads[2]), _ptr(cu_seqlens),
                                       _ptr(past_lens), B, H, H_kv, D, int(max_seqlen), T, scale, _ptr(ws), ws_bytes,
                                       _ptr(dev_status), _stream(stream))
    _check(rc, "unipin_masked_prefill_bwd")
    return tuple(grads)


def kvpool_write(pool_k, pool_v, layer: int, k, v, cu_seqlens, past_lens, slot_ids, max_past: int,
                 dev_status=None, stream=None, pool_scales=None):
    """Each segment's past K/V rows into its pool slot at `layer`: a byte copy into a bfloat16 pool,
    E4M3 codes of k / k_scale and v / v_scale into an E4M3 pool."""
    pool = _pool(pool_k, pool_v, pool_scales)
    _tokens(k, "k", pool.D)
    _tokens(v, "v", pool.D)
    B = past_lens.shape[0]
    _index(cu_seqlens, "cu_seqlens", B + 1)
    _index(past_lens, "past_lens", B)
    _index(slot_ids, "slot_ids", B)
    rc = LIB.unipin_kvpool_write(ctypes.byref(pool), int(layer), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                 _ptr(past_lens), _ptr(slot_ids), B, int(max_past), int(k.shape[0]),
                                 _ptr(dev_status), _stream(stream))
    _check(rc, "unipin_kvpool_write")


def rank_decode_workspace_size(R: int, H: int, D: int, max_k: int, total_cand: int, n_cap: int,
                               H_kv: Optional[int] = None) -> int:
    """Workspace bytes of rank_decode_attn; H are query heads, H_kv the pool's key/value heads (default H)."""
    return int(LIB.unipin_rank_decode_workspace_size(R, H, H if H_kv is None else int(H_kv), D, max_k, total_cand,
                                                      n_cap))


def rank_decode_pool_workspace_size(pool_k, pool_v, R: int, H: int, max_k: int, total_cand: int,
                                    pool_scales=None) -> int:
    """Workspace bytes of rank_decode_attn over this pool (an E4M3 pool also needs room for its
    dequantized rows)."""
    pool = _pool(pool_k, pool_v, pool_scales)
    return int(LIB.unipin_rank_decode_pool_workspace_size(ctypes.byref(pool), int(R), int(H), int(max_k),
                                                          int(total_cand)))


def rank_decode_attn(q_c, k_c, v_c, cu_seqlens_c, slot_ids, past_lens, pool_k, pool_v, layer: int, max_k: int,
                     out=None, out_fp32: bool = True, scale: Optional[float] = None, workspace="auto",
                     dev_status=None, stream=None, pool_scales=None):
    """Candidates attend to their slot's cached past rows plus themselves (a bfloat16 pool, or an
    E4M3 pool with pool_scales = (k_scale, v_scale))."""
    _tokens(q_c, "q_c")
    T, H, D = q_c.shape
    _tokens(k_c, "k_c", D)
    _tokens(v_c, "v_c", D)
    pool = _pool(pool_k, pool_v, pool_scales)
    if _kv_heads(q_c, k_c, v_c) != pool.H:
        raise ValueError("k_c and v_c must have the pool's %d key/value heads" % pool.H)
    R = past_lens.shape[0]
    _index(cu_seqlens_c, "cu_seqlens_c", R + 1)
    _index(slot_ids, "slot_ids", R)
    _index(past_lens, "past_lens", R)
    if out is None:
        out = torch.empty((T, H, D), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q_c.device)
    elif out.dtype != (torch.float32 if out_fp32 else torch.bfloat16) or out.shape != q_c.shape or not out.is_contiguous():
        raise ValueError("out has the wrong dtype or shape")
    ws, ws_bytes = _workspace(workspace, int(LIB.unipin_rank_decode_pool_workspace_size(
        ctypes.byref(pool), R, H, int(max_k), T)) if isinstance(workspace, str) else 0, q_c.device)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    rc = LIB.unipin_rank_decode_attn(_ptr(q_c), _ptr(k_c), _ptr(v_c), _ptr(out), int(bool(out_fp32)),
                                     _ptr(cu_seqlens_c), _ptr(slot_ids), _ptr(past_lens), R, H, D, int(max_k), T,
                                     scale, ctypes.byref(pool), int(layer), _ptr(ws), ws_bytes,
                                     _ptr(dev_status), _stream(stream))
    _check(rc, "unipin_rank_decode_attn")
    return out


def rank_decode_attn_noalloc(q_c, k_c, v_c, cu_seqlens_c, slot_ids, past_lens, pool_k, pool_v, layer: int,
                             max_k: int, out, out_fp32: bool = True, scale: Optional[float] = None,
                             dev_status=None, stream=None, pool_scales=None):
    """Rank decode through the entry point that allocates nothing (the caller passes `out`).

    For callers that cannot allocate device memory while serving: the scratch
    lives in a fixed device array inside the library, shared by every call, so
    calls must not overlap on the GPU.
    """
    _tokens(q_c, "q_c")
    T, H, D = q_c.shape
    _tokens(k_c, "k_c", D)
    _tokens(v_c, "v_c", D)
    pool = _pool(pool_k, pool_v, pool_scales)
    if _kv_heads(q_c, k_c, v_c) != pool.H:
        raise ValueError("k_c and v_c must have the pool's %d key/value heads" % pool.H)
    R = past_lens.shape[0]
    _index(cu_seqlens_c, "cu_seqlens_c", R + 1)
    _index(slot_ids, "slot_ids", R)
    _index(past_lens, "past_lens", R)
    if out.dtype != (torch.float32 if out_fp32 else torch.bfloat16) or out.shape != q_c.shape or not out.is_contiguous():
        raise ValueError("out has the wrong dtype or shape")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    rc = LIB.unipin_rank_decode_attn_noalloc(_ptr(q_c), _ptr(k_c), _ptr(v_c), _ptr(out), int(bool(out_fp32)),
                                             _ptr(cu_seqlens_c), _ptr(slot_ids), _ptr(past_lens), R, H, D,
                                             int(max_k), T, scale, ctypes.byref(pool), int(layer),
                                             _ptr(dev_status), _stream(stream))
    _check(rc, "unipin_rank_decode_attn_noalloc")
    return out


def rank_decode_noalloc_scratch_bytes() -> int:
    return int(LIB.unipin_rank_decode_noalloc_scratch_bytes())


def selftest_bounded_wait(dev_status, limit_us: int, stream=None):
    rc = LIB.unipin_selftest_bounded_wait(_ptr(dev_status), int(limit_us), _stream(stream))
    _check(rc, "unipin_selftest_bounded_wait")


def selftest_exp2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The softmax's FMA-pipe exp2 on a CUDA float32 tensor."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA float32 tensor")
    y = torch.empty_like(x)
    _check(LIB.unipin_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "unipin_selftest_exp2")
    return y


def status_string(code: int) -> str:
    return LIB.unipin_status_string(int(code)).decode()


# ------------------------------------------------- pool sharing and slot ring

def kvpool_share_export(pool_k: torch.Tensor, pool_v: torch.Tensor, pool_scales=None) -> bytes:
    """IPC description of a pool (bytes to hand to another process, e.g. through a file)."""
    pool = _pool(pool_k, pool_v, pool_scales)
    desc = KVPoolShare()
    _check(LIB.unipin_kvpool_share_export(ctypes.byref(pool), ctypes.byref(desc)), "unipin_kvpool_share_export")
    return bytes(desc)


class _DeviceArray:
    """A zero-copy view of device memory owned elsewhere, for torch.as_tensor."""

    def __init__(self, ptr: int, shape, typestr: str = "<i2"):
        self.__cuda_array_interface__ = {"shape": tuple(int(x) for x in shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


class SharedPool:
    """A pool exported by another process, mapped into this one.

    ``k`` and ``v`` are tensors [L, S, H, n_cap, D] over the exporter's memory
    (bfloat16, or float8_e4m3fn codes with ``scales`` = (k_scale, v_scale)),
    usable with every call of this module; ``close()`` unmaps them.
    """

    def __init__(self, desc: bytes, device=None):
        if len(desc) != ctypes.sizeof(KVPoolShare):
            raise ValueError("a pool description is %d bytes" % ctypes.sizeof(KVPoolShare))
        self._desc = KVPoolShare.from_buffer_copy(desc)
        self._pool = KVPool()
        _check(LIB.unipin_kvpool_share_open(ctypes.byref(self._desc), ctypes.byref(self._pool)),
               "unipin_kvpool_share_open")
        d = self._desc
        shape = (d.L, d.S, d.H, d.n_cap, d.D)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        if d.dtype == POOL_E4M3:
            self.k = torch.as_tensor(_DeviceArray(self._pool.k, shape, "|u1"), device=dev).view(torch.float8_e4m3fn)
            self.v = torch.as_tensor(_DeviceArray(self._pool.v, shape, "|u1"), device=dev).view(torch.float8_e4m3fn)
        else:
            self.k = torch.as_tensor(_DeviceArray(self._pool.k, shape), device=dev).view(torch.bfloat16)
            self.v = torch.as_tensor(_DeviceArray(self._pool.v, shape), device=dev).view(torch.bfloat16)
        self.scales = (d.k_scale, d.v_scale)

    def close(self):
        if self._pool.k:
            self.k = self.v = None
            _check(LIB.unipin_kvpool_share_close(ctypes.byref(self._desc), ctypes.byref(self._pool)),
                   "unipin_kvpool_share_close")


class SlotRing:
    """Round-robin assignment of pool slots to requests (host side, thread-safe)."""

    def __init__(self, S: int):
        h = ctypes.c_void_p()
        _check(LIB.unipin_slot_ring_create(int(S), ctypes.byref(h)), "unipin_slot_ring_create")
        self._h = h
        self._destroy = LIB.unipin_slot_ring_destroy
        self.S = int(S)

    def acquire(self, n: int):
        ids = (ctypes.c_int * max(int(n), 1))()
        _check(LIB.unipin_slot_ring_acquire(self._h, int(n), ids), "unipin_slot_ring_acquire")
        return [ids[i] for i in range(int(n))]

    def release(self, slot_ids):
        slot_ids = [int(s) for s in slot_ids]
        ids = (ctypes.c_int * max(len(slot_ids), 1))(*slot_ids)
        _check(LIB.unipin_slot_ring_release(self._h, len(slot_ids), ids), "unipin_slot_ring_release")

    def free_count(self) -> int:
        n = LIB.unipin_slot_ring_free_count(self._h)
        if n < 0:
            raise UnipinError(n, "unipin_slot_ring_free_count")
        return n

    def close(self):
        if getattr(self, "_h", None):
            self._destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()
