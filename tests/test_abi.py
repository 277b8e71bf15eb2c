"""C-ABI checks that need no GPU: the library loads, exports every declared symbol,
computes layouts on the host, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lbq.h")


@pytest.fixture(scope="module")
def L():
    from bit_weight_only_ternary_b200 import build
    build.build()
    from bit_weight_only_ternary_b200 import lbq
    return lbq


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lbq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("lbq_pack", "lbq_gemv", "lbq_gemm", "lbq_hadamard"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    lib = ctypes.CDLL(L.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(L.EXPORTS)


def test_status_strings(L):
    for st in range(8):
        assert L.lbq_status_string(st)
    assert L.lbq_status_string(99) == "unknown status"


def test_layout_matches_oracle_layout(L, orc):
    for fmt in (1, 2, 3):
        for K in (512, 1024, 5120, 17408):
            for N, N4 in ((3, 4), (4, 4), (9, 12)):  # rows are stored in groups of four
                cs, ss, cb, sb = L.lbq_packed_layout(fmt, K, N)
                ocs, oss, _ = orc.layout(fmt, K)
                assert (cs, ss, cb, sb) == (ocs, oss, N4 * ocs, N4 * oss * 2)
    assert L.lbq_packed_layout(1, 128, 1)[0] == 32
    assert L.lbq_packed_layout(1, 384, 1)[0] == 96  # 3 x 28 = 84 -> 96


@pytest.mark.parametrize("fmt,K,N,st", [(0, 512, 1, 4), (4, 512, 1, 4), (1, 100, 1, 2),
                                         (1, 0, 1, 2), (1, 512, 0, 2), (3, 640, 1, 2),
                                         (2, 640, 1, 0), (3, 1024, 1, 0)])
def test_layout_errors(L, fmt, K, N, st):
    cs = ctypes.c_int64()
    assert L.lib().lbq_packed_layout(fmt, K, N, ctypes.byref(cs), None, None, None) == st


def _desc(L, fmt=1, K=512, N=4, codes=0x10000, scales=None, cs=None, ss=0):
    if cs is None:
        cs = L.lbq_packed_layout(fmt if fmt in (1, 2, 3) else 1, K if K % 128 == 0 else 512, 1)[0]
    return L.lbq_weights(fmt, 0, K, N, codes, scales, cs, ss)


def test_validation_rejects_before_launch(L):
    lib = L.lib()
    x, y, ws = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000), ctypes.c_void_p(0x40000)
    D = ctypes.c_void_p(0x50000)
    ok = _desc(L)
    assert lib.lbq_gemv(None, x, None, y, None, 0, None) == L.LBQ_ERR_ARG
    bad = _desc(L, fmt=9)
    assert lib.lbq_gemv(ctypes.byref(bad), x, None, y, None, 0, None) == L.LBQ_ERR_FORMAT
    bad = _desc(L, K=500)
    assert lib.lbq_gemv(ctypes.byref(bad), x, None, y, None, 0, None) == L.LBQ_ERR_SHAPE
    bad = _desc(L, codes=0x10004)
    assert lib.lbq_gemv(ctypes.byref(bad), x, None, y, None, 0, None) == L.LBQ_ERR_ALIGN
    bad = _desc(L, cs=16)
    assert lib.lbq_gemv(ctypes.byref(bad), x, None, y, None, 0, None) == L.LBQ_ERR_SHAPE
    bad = _desc(L, codes=None)
    assert lib.lbq_gemv(ctypes.byref(bad), x, None, y, None, 0, None) == L.LBQ_ERR_ARG
    bad = _desc(L, scales=0x60000)  # ternary keeps its scales in-block
    assert lib.lbq_gemv(ctypes.byref(bad), x, None, y, None, 0, None) == L.LBQ_ERR_ARG
    assert lib.lbq_gemv(ctypes.byref(ok), None, None, y, None, 0, None) == L.LBQ_ERR_ARG
    assert lib.lbq_gemv(ctypes.byref(ok), ctypes.c_void_p(0x20008), None, y, None, 0,
                        None) == L.LBQ_ERR_ALIGN
    assert lib.lbq_gemv(ctypes.byref(ok), x, None, ctypes.c_void_p(0x30001), None, 0,
                        None) == L.LBQ_ERR_ALIGN
    assert lib.lbq_gemm(ctypes.byref(ok), x, 0, None, y, None, 0, None) == L.LBQ_ERR_SHAPE
    sign = _desc(L, fmt=2, scales=None, ss=8)
    assert lib.lbq_gemv(ctypes.byref(sign), x, None, y, None, 0, None) == L.LBQ_ERR_ARG
    sign = _desc(L, fmt=2, scales=0x60000, ss=3)
    assert lib.lbq_gemv(ctypes.byref(sign), x, None, y, None, 0, None) == L.LBQ_ERR_SHAPE
    sign = _desc(L, fmt=2, scales=0x60008, ss=8)
    assert lib.lbq_gemv(ctypes.byref(sign), x, None, y, None, 0, None) == L.LBQ_ERR_ALIGN
    q2 = _desc(L, fmt=3, scales=0x60000, ss=16)
    assert lib.lbq_gemv(ctypes.byref(q2), x, None, y, None, 0, None) == L.LBQ_ERR_ARG  # no D
    assert lib.lbq_gemv(ctypes.byref(q2), x, ctypes.c_void_p(0x50001), y, None, 0,
                        None) == L.LBQ_ERR_ALIGN
    need = lib.lbq_workspace_bytes(ctypes.byref(q2), 1)
    if need:
        assert lib.lbq_gemv(ctypes.byref(q2), x, D, y, None, 0, None) == L.LBQ_ERR_WORKSPACE
        assert lib.lbq_gemv(ctypes.byref(q2), x, D, y, ws, need - 1, None) == L.LBQ_ERR_WORKSPACE
    assert lib.lbq_workspace_bytes(None, 1) == 0
    assert lib.lbq_workspace_bytes(ctypes.byref(ok), 0) == 0
    # pack / hadamard / signs argument checks
    W = ctypes.c_void_p(0x70000)
    assert lib.lbq_pack(1, W, 512, 4, None, None, None) == L.LBQ_ERR_ARG
    assert lib.lbq_pack(1, W, 512, 4, ctypes.c_void_p(0x10000), ctypes.c_void_p(0x60000),
                        None) == L.LBQ_ERR_ARG
    assert lib.lbq_pack(2, W, 512, 4, ctypes.c_void_p(0x10000), None, None) == L.LBQ_ERR_ARG
    assert lib.lbq_pack(1, ctypes.c_void_p(0x70004), 512, 4, ctypes.c_void_p(0x10000), None,
                        None) == L.LBQ_ERR_ALIGN
    assert lib.lbq_pack(7, W, 512, 4, ctypes.c_void_p(0x10000), None, None) == L.LBQ_ERR_FORMAT
    assert lib.lbq_hadamard(x, D, 1, 500, y, None) == L.LBQ_ERR_SHAPE
    assert lib.lbq_hadamard(x, None, 1, 512, y, None) == L.LBQ_ERR_ARG
    assert lib.lbq_hadamard(x, D, 1, 512, ctypes.c_void_p(0x30004), None) == L.LBQ_ERR_ALIGN
    assert lib.lbq_rht_signs(1, 0, D, None) == L.LBQ_ERR_SHAPE
    assert lib.lbq_rht_signs(1, 5, None, None) == L.LBQ_ERR_ARG
    assert lib.lbq_device_fault(None) == L.LBQ_ERR_ARG
