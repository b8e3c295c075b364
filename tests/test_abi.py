"""CPU-only checks of the C-ABI library: it loads, exports every function the
header declares, and its host-side logic (threshold table, argument checks,
workspace sizing) behaves as documented.  No GPU call is made."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle.hstu_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hstu.h")


def _lib():
    from hstu_sequential_transducer_02_b200 import binding
    return binding


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_expected_entry_points():
    names = _declared_functions()
    for must in ("hstu_attn_fwd", "hstu_attn_bwd", "hstu_layer_fwd", "hstu_layer_bwd", "mfalcon_rank",
                 "hstu_stochastic_length", "hstu_build_time_thresholds"):
        assert must in names


def test_library_exports_every_declared_symbol():
    b = _lib()
    lib = ctypes.CDLL(b.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(b.EXPORTED) <= set(_declared_functions())


def test_status_strings_and_version():
    b = _lib()
    assert b.status_string(0) == "ok"
    assert "timed out" in b.status_string(b.ERR_TIMEOUT)
    assert b.status_string(999) == "unknown status"
    assert b.version() >= 10000


def test_threshold_table_reproduces_oracle_buckets():
    """The library's integer thresholds give the same bucket as the oracle's fp64
    formula for every dt probed (dense small range + around each threshold)."""
    b = _lib()
    thr = np.array(b.build_time_thresholds(0.301), dtype=np.int64)
    assert thr[0] == 0 and np.all(np.diff(thr) >= 0)
    probes = set(range(0, 5000))
    for t in thr[1:]:
        if t < 2 ** 62:
            probes.update([int(t) - 1, int(t), int(t) + 1])
    probes = np.array(sorted(p for p in probes if p >= 0), dtype=np.int64)
    lib_bucket = np.minimum(127, np.searchsorted(thr[1:], np.maximum(probes, 1), side="right"))
    assert np.array_equal(lib_bucket, O.time_bucket(probes))


def test_threshold_table_argument_checks():
    b = _lib()
    out = (ctypes.c_int64 * 128)()
    assert b._lib_thresholds(0.0, 128, out) == b.ERR_INVALID_ARG
    assert b._lib_thresholds(0.301, 1, out) == b.ERR_INVALID_ARG
    assert b._lib_thresholds(0.301, 128, None) == b.ERR_INVALID_ARG


def test_workspace_size_and_descriptor_checks():
    b = _lib()
    n = ctypes.c_size_t()
    d = b.attn_desc(4, 128, b.DTYPE_BF16)
    assert b._lib_attn_fwd_ws(ctypes.byref(d), 8, 49152, ctypes.byref(n)) == b.OK
    assert n.value > 0 and n.value % 256 == 0
    bad = b.attn_desc(4, 96, b.DTYPE_BF16)
    assert b._lib_attn_fwd_ws(ctypes.byref(bad), 8, 100, ctypes.byref(n)) == b.ERR_UNSUPPORTED
    bad = b.attn_desc(0, 64, b.DTYPE_BF16)
    assert b._lib_attn_fwd_ws(ctypes.byref(bad), 8, 100, ctypes.byref(n)) == b.ERR_INVALID_ARG
    bad = b.attn_desc(2, 64, 7)
    assert b._lib_attn_fwd_ws(ctypes.byref(bad), 8, 100, ctypes.byref(n)) == b.ERR_UNSUPPORTED
    ld = b.layer_desc(512, 4, 128, b.DTYPE_BF16)
    assert b._lib_layer_fwd_ws(ctypes.byref(ld), 8, 1000, ctypes.byref(n)) == b.OK
    assert b._lib_layer_bwd_ws(ctypes.byref(ld), 8, 1000, ctypes.byref(n)) == b.OK
    assert b._lib_mf_ws(ctypes.byref(ld), 1, 16, 32768, 512, ctypes.byref(n)) == b.OK
    assert b._lib_mf_ws(ctypes.byref(ld), 0, 16, 32768, 512, ctypes.byref(n)) == b.ERR_INVALID_ARG


def test_null_arguments_rejected_before_any_launch():
    b = _lib()
    d = b.attn_desc(2, 64, b.DTYPE_BF16)
    assert b._lib_attn_fwd(None, None, None, 0, None, 0, None, 0, None, None, None, 0, None, 0, None) \
        == b.ERR_INVALID_ARG
    jb = b.Jagged(1, 10, None, None, None)
    assert b._lib_attn_fwd(ctypes.byref(d), ctypes.byref(jb), None, 0, None, 0, None, 0, None, None, None, 0, None,
                           0, None) == b.ERR_INVALID_ARG
    # misaligned row stride (bf16, ld = 129 elements is not a multiple of 16 bytes)
    jb = b.Jagged(1, 10, ctypes.c_void_p(256), None, ctypes.c_void_p(256))
    p = ctypes.c_void_p(1 << 20)
    assert b._lib_attn_fwd(ctypes.byref(d), ctypes.byref(jb), p, 129, p, 128, p, 128, p, p, p, 128, p, 1 << 20,
                           None) == b.ERR_INVALID_ARG
    # workspace too small
    assert b._lib_attn_fwd(ctypes.byref(d), ctypes.byref(jb), p, 128, p, 128, p, 128, p, p, p, 128, p, 16,
                           None) == b.ERR_WORKSPACE
    assert b._lib_dbg_timeout(0, None, None) == b.ERR_INVALID_ARG
    assert b._lib_gather(p, p, 6, p, p, 1, None) == b.ERR_INVALID_ARG


def test_host_memory_forward_argument_checks():
    """hstu_layer_fwd_host validates its host offsets and sizes before it
    touches the GPU: offsets must start at 0 and not decrease, x and y must be
    given, num_chunks >= 1, and the workspace must be large enough."""
    b = _lib()
    ld = b.layer_desc(64, 2, 32, b.DTYPE_BF16)
    n = ctypes.c_size_t()
    assert b._lib_layer_fwd_host_ws(ctypes.byref(ld), 3, 100, 4, ctypes.byref(n)) == b.OK
    assert n.value > 0 and n.value % 256 == 0
    assert b._lib_layer_fwd_host_ws(ctypes.byref(ld), 3, 100, 0, ctypes.byref(n)) == b.ERR_INVALID_ARG
    p = ctypes.c_void_p(1 << 20)     # never dereferenced: every call below fails its host checks
    w = b.LayerWeights(*([p] * 10))
    ts = (ctypes.c_int64 * 100)()
    x = (ctypes.c_uint16 * 6400)()
    y = (ctypes.c_uint16 * 6400)()

    def call(offs, xx=x, chunks=2, ws_bytes=1 << 40):
        o = (ctypes.c_int32 * len(offs))(*offs)
        return b._lib_layer_fwd_host(ctypes.byref(ld), ctypes.byref(w), len(offs) - 1, o, None, ts, xx, y, chunks,
                                     p, ws_bytes, None)

    assert call([1, 40, 100]) == b.ERR_INVALID_ARG            # does not start at 0
    assert call([0, 60, 40]) == b.ERR_INVALID_ARG             # decreasing
    assert call([0, 40, 100], xx=None) == b.ERR_INVALID_ARG
    assert call([0, 40, 100], chunks=0) == b.ERR_INVALID_ARG
    assert call([0, 40, 100], ws_bytes=256) == b.ERR_WORKSPACE


def test_ranking_and_sl_argument_checks():
    """mfalcon_rank and hstu_stochastic_length refuse bad arguments on the host,
    before any launch: no layers, microbatch < 1, null or misaligned buffers,
    a workspace too small; SL with max_len < 1 or missing arrays."""
    b = _lib()
    ld = b.layer_desc(64, 2, 32, b.DTYPE_BF16)
    p = ctypes.c_void_p(1 << 20)      # never dereferenced: every call below fails its host checks
    odd = ctypes.c_void_p((1 << 20) + 8)
    w = b.LayerWeights(*([p] * 10))
    arr = (b.LayerWeights * 1)(w)

    def mf(layers=arr, L=1, bm=8, cand_x=p, cand_out=p, ws_bytes=1 << 40):
        return b._lib_mf(ctypes.byref(ld), layers, L, 2, 100, 16, bm, p, p, p, p, cand_x, p, cand_out, p, ws_bytes,
                         None)

    assert mf(layers=None) == b.ERR_INVALID_ARG
    assert mf(L=0) == b.ERR_INVALID_ARG
    assert mf(bm=0) == b.ERR_INVALID_ARG
    assert mf(cand_x=None) == b.ERR_INVALID_ARG
    assert mf(cand_out=odd) == b.ERR_INVALID_ARG
    assert mf(ws_bytes=256) == b.ERR_WORKSPACE
    assert b._lib_sl(4, 100, p, p, p, 0, 0, p, p, p, 1 << 20, None) == b.ERR_INVALID_ARG
    assert b._lib_sl(4, 100, None, p, p, 8, 0, p, p, p, 1 << 20, None) == b.ERR_INVALID_ARG
    assert b._lib_sl(4, 100, p, None, p, 8, 0, p, p, p, 1 << 20, None) == b.ERR_INVALID_ARG
    assert b._lib_sl(4, 100, p, p, p, 8, 0, p, p, p, 16, None) == b.ERR_WORKSPACE
