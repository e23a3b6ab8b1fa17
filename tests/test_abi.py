"""CPU-only checks of the boundary: the library loads and exports what the header declares."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "unipin.h")
LIB = os.path.join(ROOT, "kv_cache_reuse_falcon_b200", "libunipin.so")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(unipin_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from kv_cache_reuse_falcon_b200 import build
    build.build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_three_hot_path_calls():
    names = declared_functions()
    for n in ("unipin_masked_prefill_attn", "unipin_kvpool_write", "unipin_rank_decode_attn"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    lib.unipin_status_string.restype = ctypes.c_char_p
    lib.unipin_status_string.argtypes = [ctypes.c_int]
    assert lib.unipin_status_string(0) == b"UNIPIN_OK"
    assert lib.unipin_status_string(-6) == b"UNIPIN_ERR_DEVICE_TIMEOUT"
    assert lib.unipin_status_string(42) == b"UNIPIN_ERR_UNKNOWN"


def test_host_validation_needs_no_device(lib):
    """Argument errors are found before any CUDA call, so they work without a GPU."""
    P, I = ctypes.c_void_p, ctypes.c_int
    f = lib.unipin_masked_prefill_attn
    SZ = ctypes.c_size_t
    f.argtypes = [P, P, P, P, I, P, P, P, I, I, I, I, I, I, ctypes.c_float, P, P, I, P, SZ, P, P]
    f.restype = I
    args = [None, None, None, None, 1, None, None, None]
    assert f(*args, 1, 1, 1, 48, 16, 16, 0.1, None, None, 0, None, 0, None, None) == -2
    assert f(*args, -1, 1, 1, 64, 16, 16, 0.1, None, None, 0, None, 0, None, None) == -1
    assert f(*args, 1, 1, 1, 64, 16, 16, -1.0, None, None, 0, None, 0, None, None) == -1
    assert f(*args, 1, 4, 3, 64, 16, 16, 0.1, None, None, 0, None, 0, None, None) == -1   # 4 heads over 3
    # nothing to do: B = 0 returns OK without touching the device
    assert f(*args, 0, 1, 1, 64, 16, 0, 0.1, None, None, 0, None, 0, None, None) == 0
    b = lib.unipin_masked_prefill_bwd
    b.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, ctypes.c_float, P, SZ, P, P]
    b.restype = I
    nul = [None] * 11
    assert b(*nul, 1, 1, 1, 96, 16, 16, 0.1, None, 0, None, None) == -2     # D = 96: not supported
    assert b(*nul, 1, 1, 1, 64, 16, 16, 0.0, None, 0, None, None) == -1     # scale must be positive
    assert b(*nul, 1, 1, 1, 64, 16, 16, 0.1, None, 0, None, None) == -1     # missing tensors
    assert b(*nul, 0, 1, 1, 64, 16, 0, 0.1, None, 0, None, None) == 0
    wb = lib.unipin_masked_prefill_bwd_workspace_size
    wb.argtypes = [I, I]
    wb.restype = SZ
    assert wb(1000, 8) == 32000 and wb(3, 1) == 16
    g = lib.unipin_rank_decode_workspace_size
    g.argtypes = [I, I, I, I, I, I, I]
    g.restype = SZ
    assert g(32, 8, 8, 64, 16, 512, 2048) > 256       # small k: split-n partials on top of the work counter
    assert g(32, 8, 8, 64, 1000, 32000, 2048) == 256  # large k: the work counter only
    assert g(32, 8, 2, 64, 16, 512, 2048) > 256       # grouped heads: 4 query heads per pool head
    assert g(32, 8, 3, 64, 16, 512, 2048) == 0        # 8 query heads over 3 key/value heads
    wp = lib.unipin_masked_prefill_workspace_size
    wp.restype = SZ
    assert wp() == 256


class Pool(ctypes.Structure):
    """unipin_kvpool as include/unipin.h declares it."""
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("L", ctypes.c_int), ("S", ctypes.c_int),
                ("H", ctypes.c_int), ("n_cap", ctypes.c_int), ("D", ctypes.c_int), ("dtype", ctypes.c_int),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


def test_e4m3_pool_host_rules_need_no_device(lib):
    """The E4M3 pool's workspace size and the calls that refuse it are host-side decisions."""
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    ws = lib.unipin_rank_decode_pool_workspace_size
    ws.argtypes = [P, I, I, I, I]
    ws.restype = SZ
    g = lib.unipin_rank_decode_workspace_size
    g.argtypes = [I, I, I, I, I, I, I]
    g.restype = SZ
    bf = Pool(16, 16, 1, 4, 2, 512, 64, 0, 1.0, 1.0)
    f8 = Pool(16, 16, 1, 4, 2, 512, 64, 1, 0.5, 0.25)
    base = g(3, 4, 2, 64, 16, 48, 512)
    assert ws(ctypes.byref(bf), 3, 4, 16, 48) == base
    # 16 candidates x 2 query heads per kv head = 32 columns: the small-k kernel reads the codes, no copy
    assert base <= ws(ctypes.byref(f8), 3, 4, 16, 48) < base + 2 * 3 * 2 * 512 * 64
    # 32 candidates x 2 = 64 columns at D=64: the dequantized copy (measured faster there)
    base32 = g(3, 4, 2, 64, 32, 96, 512)
    assert ws(ctypes.byref(f8), 3, 4, 32, 96) >= base32 + 2 * 3 * 2 * 512 * 64 * 2 + 3 * 4
    # ... when both scales are bfloat16 values in its range; otherwise the dequantized copy
    for ks, vs in ((0.3, 0.25), (0.5, 2.0 ** -120), (0.5, 2.0 ** 119)):
        odd = Pool(16, 16, 1, 4, 2, 512, 64, 1, ks, vs)
        assert ws(ctypes.byref(odd), 3, 4, 16, 48) >= base + 2 * 3 * 2 * 512 * 64 * 2 + 3 * 4
    # 100 candidates: the engine reads dequantized rows, 3 requests x 2 heads x 512 rows x 64 bf16 for
    # K and V, and the slot ids
    base100 = g(3, 4, 2, 64, 100, 300, 512)
    assert ws(ctypes.byref(f8), 3, 4, 100, 300) >= base100 + 2 * 3 * 2 * 512 * 64 * 2 + 3 * 4
    assert ws(ctypes.byref(f8), 3, 3, 16, 48) == 0          # query heads not a multiple of the pool's
    na = lib.unipin_rank_decode_attn_noalloc
    na.argtypes = [P, P, P, P, I, P, P, P, I, I, I, I, I, ctypes.c_float, P, I, P, P]
    na.restype = I
    assert na(P(16), P(16), P(16), P(16), 1, P(16), P(16), P(16), 3, 4, 64, 100, 300, 0.1, ctypes.byref(f8), 0,
              None, None) == -2                              # nor by the no-alloc call beyond 64 columns
    dec = lib.unipin_rank_decode_attn
    dec.argtypes = [P, P, P, P, I, P, P, P, I, I, I, I, I, ctypes.c_float, P, I, P, SZ, P, P]
    dec.restype = I
    for bad in (Pool(16, 16, 1, 4, 2, 512, 64, 2, 1.0, 1.0), Pool(16, 16, 1, 4, 2, 512, 64, 1, 0.0, 1.0),
                Pool(16, 16, 1, 4, 2, 512, 64, 1, 1.0, float("inf"))):
        assert dec(P(16), P(16), P(16), P(16), 1, P(16), P(16), P(16), 3, 4, 64, 16, 48, 0.1, ctypes.byref(bad), 0,
                   None, 0, None, None) == -1                # unknown dtype, scales not finite and positive


def test_binding_refuses_to_load_without_library(tmp_path):
    from kv_cache_reuse_falcon_b200 import binding
    with pytest.raises(ImportError):
        binding._load(str(tmp_path / "missing.so"))


def test_no_oracle_import_in_product_code():
    pkg = os.path.join(ROOT, "kv_cache_reuse_falcon_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src, fn
