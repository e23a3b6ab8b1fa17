"""CPU oracle (fp64) for the masked prefill, its gradients, the pool write and the rank decode.

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
CPU-baseline leg may call this package; the library under
``kv_cache_reuse_falcon_b200`` never imports it, and it imports nothing from
there.  The arithmetic lives in ``oracle.c`` (plain C, OpenMP over independent
rows); this file only builds it with gcc and marshals numpy arrays.

Sources followed (see ``oracle.c`` for the mask and the formulas):
UniPinRec reproduction notes (slinene.github.io), sub-module details §3
"attention mask" and §6 "serving: cross-process KV sharing"; UniPinRec paper
review (liuzhao09.github.io), §2.2 and §2.4.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        lib.oracle_prefill_rows.argtypes = [P, P, P, P, P, I, I, I, I, ctypes.c_double, I, P, I64, P, P]
        lib.oracle_prefill_rows.restype = I
        lib.oracle_decode_rows.argtypes = [P, P, P, P, P, P, I, I, I, I, ctypes.c_double, I,
                                           P, P, I, I, I, I, P, I64, P, P]
        lib.oracle_decode_rows.restype = I
        lib.oracle_prefill_bwd.argtypes = [P, P, P, P, P, P, I, I, I, I, ctypes.c_double, I, P, P, P]
        lib.oracle_prefill_bwd.restype = I
        lib.oracle_prefill_bwd_f64.argtypes = [P, P, P, P, P, P, I, I, I, I, ctypes.c_double, I, P, P, P]
        lib.oracle_prefill_bwd_f64.restype = I
        lib.oracle_pool_write.argtypes = [P, P, I, I, I, I, I, I, P, P, P, P, P, I]
        lib.oracle_pool_write_e4m3.argtypes = [P, P, I, I, I, I, I, I, P, P, P, P, P, I, ctypes.c_float,
                                               ctypes.c_float]
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_dequant_bf16.argtypes = [P, I64, ctypes.c_float, P]
        lib.oracle_pool_write.restype = I
        lib.oracle_num_threads.restype = I
        lib.oracle_set_num_threads.argtypes = [I]
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("expected bfloat16 bit patterns as uint16, got %s" % a.dtype)
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _kv_heads(q, k, v) -> int:
    """Key/value heads of grouped-query inputs: k and v share a shape whose head count divides q's."""
    if k.shape != v.shape or k.shape[0] != q.shape[0] or k.shape[2] != q.shape[2]:
        raise ValueError("k and v must be [T, Hkv, D] with q's T and D")
    if q.shape[1] % k.shape[1] != 0:
        raise ValueError("query heads must be a multiple of key/value heads")
    return int(k.shape[1])


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def prefill(q, k, v, cu_seqlens, past_lens, scale: Optional[float] = None, cand_self: bool = True,
            tokens=None, return_lse: bool = False):
    """M-FALCON masked attention of packed segments; returns float64 [ntok, H, D] (and lse [ntok, H]).

    k and v may have fewer heads than q (grouped-query attention: query head h reads kv head
    h // (H // Hkv))."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    T, H, D = q.shape
    Hkv = _kv_heads(q, k, v)
    cu = _i32(cu_seqlens)
    past = _i32(past_lens)
    B = past.shape[0]
    if cu.shape[0] != B + 1 or int(cu[-1]) != T:
        raise ValueError("cu_seqlens does not match q")
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    ntok = T if tok is None else tok.shape[0]
    out = np.zeros((ntok, H, D), dtype=np.float64)
    lse = np.zeros((ntok, H), dtype=np.float64) if return_lse else None
    rc = _load().oracle_prefill_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(cu), _ptr(past), B, H, Hkv, D, scale,
                                     int(bool(cand_self)), _ptr(tok), ntok, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_prefill_rows rejected its arguments")
    return (out, lse) if return_lse else out


def decode(qc, kc, vc, cu_c, slot_ids, past_lens, pool_k, pool_v, layer: int,
           scale: Optional[float] = None, cand_self: bool = True, tokens=None, return_lse: bool = False):
    """Rank decode: candidates over pool rows of their slot plus themselves; float64 [ntok, H, D]."""
    qc, kc, vc = _u16(qc), _u16(kc), _u16(vc)
    pool_k, pool_v = _u16(pool_k), _u16(pool_v)
    Tc, H, D = qc.shape
    Hkv = _kv_heads(qc, kc, vc)
    L, S, Hp, n_cap, Dp = pool_k.shape
    if (Hp, Dp) != (Hkv, D) or pool_v.shape != pool_k.shape:
        raise ValueError("pool shape does not match candidates")
    cu = _i32(cu_c)
    slots = _i32(slot_ids)
    past = _i32(past_lens)
    R = past.shape[0]
    if cu.shape[0] != R + 1 or int(cu[-1]) != Tc:
        raise ValueError("cu_c does not match qc")
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    ntok = Tc if tok is None else tok.shape[0]
    out = np.zeros((ntok, H, D), dtype=np.float64)
    lse = np.zeros((ntok, H), dtype=np.float64) if return_lse else None
    rc = _load().oracle_decode_rows(_ptr(qc), _ptr(kc), _ptr(vc), _ptr(cu), _ptr(slots), _ptr(past),
                                    R, H, Hkv, D, scale, int(bool(cand_self)), _ptr(pool_k), _ptr(pool_v),
                                    L, S, n_cap, int(layer), _ptr(tok), ntok, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode_rows rejected its arguments")
    return (out, lse) if return_lse else out


def pool_write(pool_k, pool_v, layer: int, k, v, cu_seqlens, past_lens, slot_ids) -> None:
    """In-place CPU mirror of the pool write (byte copy of the past K/V rows into their slots)."""
    if pool_k.dtype != np.uint16 or not pool_k.flags.c_contiguous:
        raise TypeError("pool_k must be a C-contiguous uint16 array")
    if pool_v.dtype != np.uint16 or not pool_v.flags.c_contiguous:
        raise TypeError("pool_v must be a C-contiguous uint16 array")
    L, S, H, n_cap, D = pool_k.shape
    k, v = _u16(k), _u16(v)
    cu, past, slots = _i32(cu_seqlens), _i32(past_lens), _i32(slot_ids)
    rc = _load().oracle_pool_write(_ptr(pool_k), _ptr(pool_v), L, S, H, n_cap, D, int(layer),
                                   _ptr(k), _ptr(v), _ptr(cu), _ptr(past), _ptr(slots), past.shape[0])
    if rc != 0:
        raise ValueError("oracle_pool_write rejected its arguments")


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes (uint8) of float32 values: nearest value, ties to even, saturating at +-448."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    lib = _load()
    out = np.empty(x.shape, np.uint8)
    flat, of = x.reshape(-1), out.reshape(-1)
    for i in range(flat.shape[0]):
        of[i] = lib.oracle_e4m3_encode(float(flat[i]))
    return out


def e4m3_decode(codes) -> np.ndarray:
    """The real value (float64) of each E4M3 code."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    lib = _load()
    return np.array([lib.oracle_e4m3_decode(int(b)) for b in c.reshape(-1)], np.float64).reshape(c.shape)


def e4m3_dequant_bf16(codes, scale: float) -> np.ndarray:
    """bfloat16 bit patterns of decode(code) * scale (float32 product, nearest even)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.uint16)
    _load().oracle_e4m3_dequant_bf16(_ptr(c), c.size, float(scale), _ptr(out))
    return out


def pool_write_e4m3(pool_k, pool_v, layer: int, k, v, cu_seqlens, past_lens, slot_ids, k_scale: float,
                    v_scale: float) -> None:
    """In-place CPU mirror of the pool write into an E4M3 pool (codes of k / k_scale, v / v_scale).

    The division is taken as a float32 multiply by 1 / scale, the reciprocal itself rounded to
    float32 once, as the library does."""
    for name, t in (("pool_k", pool_k), ("pool_v", pool_v)):
        if t.dtype != np.uint8 or not t.flags.c_contiguous:
            raise TypeError("%s must be a C-contiguous uint8 array" % name)
    L, S, H, n_cap, D = pool_k.shape
    k, v = _u16(k), _u16(v)
    cu, past, slots = _i32(cu_seqlens), _i32(past_lens), _i32(slot_ids)
    inv_k = float(np.float32(1.0) / np.float32(k_scale))
    inv_v = float(np.float32(1.0) / np.float32(v_scale))
    rc = _load().oracle_pool_write_e4m3(_ptr(pool_k), _ptr(pool_v), L, S, H, n_cap, D, int(layer), _ptr(k), _ptr(v),
                                        _ptr(cu), _ptr(past), _ptr(slots), past.shape[0], inv_k, inv_v)
    if rc != 0:
        raise ValueError("oracle_pool_write_e4m3 rejected its arguments")


def decode_e4m3(qc, kc, vc, cu_c, slot_ids, past_lens, pool_k8, pool_v8, layer: int, k_scale: float,
                v_scale: float, scale: Optional[float] = None):
    """Rank decode over an E4M3 pool: the pool rows read as bfloat16(decode(code) * scale), then the
    same decode as over a bfloat16 pool."""
    pk = e4m3_dequant_bf16(pool_k8, k_scale)
    pv = e4m3_dequant_bf16(pool_v8, v_scale)
    return decode(qc, kc, vc, cu_c, slot_ids, past_lens, pk, pv, layer, scale=scale)


def _bwd(fn, q, k, v, dout, cu_seqlens, past_lens, scale, cand_self):
    T, H, D = q.shape
    Hkv = _kv_heads(q, k, v)
    cu = _i32(cu_seqlens)
    past = _i32(past_lens)
    B = past.shape[0]
    if cu.shape[0] != B + 1 or int(cu[-1]) != T:
        raise ValueError("cu_seqlens does not match q")
    if dout.shape != q.shape:
        raise ValueError("dout must have the shape of q")
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    dq = np.zeros((T, H, D), dtype=np.float64)
    dk, dv = (np.zeros((T, Hkv, D), dtype=np.float64) for _ in range(2))
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(cu), _ptr(past), B, H, Hkv, D, scale,
            int(bool(cand_self)), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError("oracle backward rejected its arguments")
    return dq, dk, dv


def prefill_bwd(q, k, v, dout, cu_seqlens, past_lens, scale: Optional[float] = None, cand_self: bool = True):
    """Gradients of the masked prefill for upstream gradient dout (bf16 bits): dq float64 [T, H, D],
    dk and dv [T, Hkv, D] (with grouped heads a kv head sums its query heads' contributions)."""
    q, k, v, dout = _u16(q), _u16(k), _u16(v), _u16(dout)
    return _bwd(_load().oracle_prefill_bwd, q, k, v, dout, cu_seqlens, past_lens, scale, cand_self)


def prefill_bwd_f64(q, k, v, dout, cu_seqlens, past_lens, scale: Optional[float] = None, cand_self: bool = True):
    """As prefill_bwd on float64 inputs (e.g. for finite-difference checks)."""
    q, k, v, dout = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v, dout))
    return _bwd(_load().oracle_prefill_bwd_f64, q, k, v, dout, cu_seqlens, past_lens, scale, cand_self)
