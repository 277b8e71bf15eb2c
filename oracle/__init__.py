"""The oracle: a plain fp64 CPU reference of the low-bit formats and products.

TEST INFRASTRUCTURE ONLY. The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use it; the library under
``bit_weight_only_ternary_b200`` never imports it and shares no code with it.
The arithmetic lives in ``lbq_oracle.c`` (plain C, fp64); this module only
builds that file with gcc and marshals numpy arrays to it.

Every function is pinned by ``tests/test_oracle_pins.py`` against something other
than itself (numpy's float16 rounding, scipy's Hadamard matrix, brute force,
closed forms, published generator outputs). Parity is pinned for all functions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lbq_oracle.c")
_LIB = os.path.join(_HERE, "liblbq_oracle.so")

TERN5, SIGN1, Q2RHT = 1, 2, 3


def build(force: bool = False) -> str:
    """Compile lbq_oracle.c into liblbq_oracle.so next to it (strict IEEE flags)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-pthread", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        i64, u16, p = ctypes.c_int64, ctypes.c_uint16, ctypes.c_void_p
        _lib.orc_f16_from_f64.restype = u16
        _lib.orc_f16_from_f64.argtypes = [ctypes.c_double]
        _lib.orc_f16_to_f64.restype = ctypes.c_double
        _lib.orc_f16_to_f64.argtypes = [u16]
        _lib.orc_bf16_to_f64.restype = ctypes.c_double
        _lib.orc_bf16_to_f64.argtypes = [u16]
        _lib.orc_layout.argtypes = [ctypes.c_int, i64, p, p, p]
        _lib.orc_pack.argtypes = [ctypes.c_int, p, i64, i64, p, p]
        _lib.orc_unpack.argtypes = [ctypes.c_int, p, p, i64, i64, p, p]
        _lib.orc_dequant.argtypes = [ctypes.c_int, p, p, i64, i64, p]
        _lib.orc_rht_signs.argtypes = [ctypes.c_uint64, i64, p]
        _lib.orc_splitmix64.argtypes = [ctypes.c_uint64, i64, p]
        _lib.orc_hadamard.argtypes = [p, p, i64, i64, p]
        _lib.orc_gemm.argtypes = [ctypes.c_int, p, p, i64, i64, p, i64, p, p, p, ctypes.c_int]
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def f16_from_f64(v: float) -> int:
    return int(lib().orc_f16_from_f64(float(v)))


def f16_to_f64(h: int) -> float:
    return float(lib().orc_f16_to_f64(int(h)))


def layout(fmt: int, K: int):
    """(code_stride_bytes, scales_per_row, weights_per_scale)."""
    cs, ss, blk = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    _check(lib().orc_layout(fmt, K, ctypes.byref(cs), ctypes.byref(ss), ctypes.byref(blk)), "layout")
    return cs.value, ss.value, blk.value


def pack(fmt: int, W: np.ndarray):
    """W float32 [N][K] -> (codes uint8 [N][code_stride], scales uint16 [N][ss] or None)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    cs, ss, _ = layout(fmt, K)
    codes = np.zeros((N, cs), dtype=np.uint8)
    scales = np.zeros((N, ss), dtype=np.uint16) if ss else None
    _check(lib().orc_pack(fmt, _ptr(W), K, N, _ptr(codes), _ptr(scales)), "pack")
    return codes, scales


def unpack(fmt: int, codes: np.ndarray, scales, K: int):
    """-> (int8 codes [N][K], fp64 block scales [N][K/blk])."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N = codes.shape[0]
    _, _, blk = layout(fmt, K)
    out = np.zeros((N, K), dtype=np.int8)
    bs = np.zeros((N, K // blk), dtype=np.float64)
    sc = None if scales is None else np.ascontiguousarray(scales, dtype=np.uint16)
    _check(lib().orc_unpack(fmt, _ptr(codes), _ptr(sc), K, N, _ptr(out), _ptr(bs)), "unpack")
    return out, bs


def dequant(fmt: int, codes: np.ndarray, scales, K: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N = codes.shape[0]
    out = np.zeros((N, K), dtype=np.float64)
    sc = None if scales is None else np.ascontiguousarray(scales, dtype=np.uint16)
    _check(lib().orc_dequant(fmt, _ptr(codes), _ptr(sc), K, N, _ptr(out)), "dequant")
    return out


def splitmix64(seed: int, n: int) -> np.ndarray:
    out = np.zeros(n, dtype=np.uint64)
    _check(lib().orc_splitmix64(ctypes.c_uint64(seed), n, _ptr(out)), "splitmix64")
    return out


def rht_signs(seed: int, K: int) -> np.ndarray:
    D = np.zeros(K, dtype=np.int8)
    _check(lib().orc_rht_signs(ctypes.c_uint64(seed), K, _ptr(D)), "rht_signs")
    return D


def hadamard(x: np.ndarray, D: np.ndarray) -> np.ndarray:
    """x float64 [M][K] (or [K]) -> x' = H D x / sqrt(512) per 512-block, fp64."""
    x2 = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    M, K = x2.shape
    out = np.zeros_like(x2)
    D = np.ascontiguousarray(D, dtype=np.int8)
    _check(lib().orc_hadamard(_ptr(x2), _ptr(D), M, K, _ptr(out)), "hadamard")
    return out.reshape(np.shape(x))


def gemm(fmt: int, codes: np.ndarray, scales, K: int, X_bf16_bits: np.ndarray, D=None,
         nthreads: int = 1):
    """Y, Bnd fp64 [M][N] for bf16 X given as uint16 bits [M][K] (or [K])."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N = codes.shape[0]
    X2 = np.ascontiguousarray(np.atleast_2d(X_bf16_bits), dtype=np.uint16)
    M = X2.shape[0]
    Y = np.zeros((M, N), dtype=np.float64)
    B = np.zeros((M, N), dtype=np.float64)
    sc = None if scales is None else np.ascontiguousarray(scales, dtype=np.uint16)
    Dp = None if D is None else np.ascontiguousarray(D, dtype=np.int8)
    _check(lib().orc_gemm(fmt, _ptr(codes), _ptr(sc), K, N, _ptr(X2), M, _ptr(Dp), _ptr(Y),
                          _ptr(B), int(nthreads)), "gemm")
    return Y, B


def group4(a: np.ndarray) -> np.ndarray:
    """Device order of a per-row array: rows interleaved in groups of four.

    This is the library's own storage order (the pages fix no byte layout). Rows
    are padded with zero rows to a multiple of four; in group g (rows 4g .. 4g+3),
    element e of row 4g+q goes to position e*4 + q, where an "element" is one
    32-bit word of a code row (uint8 input, row length a multiple of 4 bytes) or
    one fp16 scale (uint16 input). Returns [ceil(N/4)][4 * row length] of the
    input dtype.
    """
    a = np.ascontiguousarray(a)
    N, R = a.shape
    G = (N + 3) // 4
    pad = np.zeros((4 * G, R), dtype=a.dtype)
    pad[:N] = a
    if a.dtype == np.uint8:
        assert R % 4 == 0, "code rows hold whole 32-bit words"
        return pad.reshape(G, 4, R // 4, 4).transpose(0, 2, 1, 3).reshape(G, 4 * R)
    assert a.dtype == np.uint16, "codes (uint8) or fp16 scale bits (uint16)"
    return pad.reshape(G, 4, R).transpose(0, 2, 1).reshape(G, 4 * R)


def ungroup4(g: np.ndarray, N: int) -> np.ndarray:
    """Inverse of group4: [ceil(N/4)][4 R] device order -> [N][R] rows."""
    g = np.ascontiguousarray(g)
    G, R4 = g.shape
    R = R4 // 4
    if g.dtype == np.uint8:
        return g.reshape(G, R // 4, 4, 4).transpose(0, 2, 1, 3).reshape(4 * G, R)[:N]
    return g.reshape(G, R, 4).transpose(0, 2, 1).reshape(4 * G, R)[:N]
