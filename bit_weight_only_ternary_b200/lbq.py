"""Thin ctypes binding of the C ABI in include/lbq.h (argument marshalling only).

Every function keeps the C name and hands torch tensors' device pointers and the
current CUDA stream to liblbq.so; all arithmetic runs in the library's kernels.
Importing this module fails loudly when the library has not been built: there
is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

LBQ_TERN5, LBQ_SIGN1, LBQ_Q2RHT = 1, 2, 3
FORMATS = {"tern": LBQ_TERN5, "sign": LBQ_SIGN1, "q2": LBQ_Q2RHT}

LBQ_OK, LBQ_ERR_ARG, LBQ_ERR_SHAPE, LBQ_ERR_ALIGN, LBQ_ERR_FORMAT, LBQ_ERR_CUDA, \
    LBQ_ERR_WORKSPACE, LBQ_ERR_DEVICE_WAIT = range(8)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblbq.so")
EXPORTS = ("lbq_status_string", "lbq_packed_layout", "lbq_pack", "lbq_unpack", "lbq_rht_signs",
           "lbq_hadamard", "lbq_workspace_bytes", "lbq_gemv", "lbq_gemm", "lbq_gemv_noalloc", "lbq_device_fault",
           "lbq_selftest_wait", "lbq_read_probe", "lbq_gemv_batch_workspace_bytes", "lbq_gemv_batch",
           "lbq_last_cuda_error", "lbq_last_cuda_error_string", "lbq_gemv_f32", "lbq_gemv_batch_plan")
LBQ_BATCH_MAX = 256
LBQ_BATCH_MAX_CTAS = 192
LBQ_NOALLOC_SCRATCH_BYTES = 4 << 20


class lbq_weights(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32), ("K", ctypes.c_int64),
                ("N", ctypes.c_int64), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("code_stride", ctypes.c_int64), ("scale_stride", ctypes.c_int64)]


class lbq_product(ctypes.Structure):
    _fields_ = [("w", lbq_weights), ("x", ctypes.c_void_p), ("D", ctypes.c_void_p),
                ("y", ctypes.c_void_p)]


class LbqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        extra = ""
        if status == LBQ_ERR_CUDA:
            extra = f": {_lib.lbq_last_cuda_error_string().decode()} ({_lib.lbq_last_cuda_error()})"
        super().__init__(f"{where}: {lbq_status_string(status)} (status {status}){extra}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m bit_weight_only_ternary_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    p, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    W = ctypes.POINTER(lbq_weights)
    sig = {
        "lbq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "lbq_packed_layout": (ctypes.c_int, [i32, i64, i64, p, p, p, p]),
        "lbq_pack": (ctypes.c_int, [i32, p, i64, i64, p, p, p]),
        "lbq_unpack": (ctypes.c_int, [W, p, p, p]),
        "lbq_rht_signs": (ctypes.c_int, [ctypes.c_uint64, i64, p, p]),
        "lbq_hadamard": (ctypes.c_int, [p, p, i64, i64, p, p]),
        "lbq_workspace_bytes": (sz, [W, i64]),
        "lbq_gemv": (ctypes.c_int, [W, p, p, p, p, sz, p]),
        "lbq_gemv_f32": (ctypes.c_int, [W, p, p, p, p, sz, p]),
        "lbq_gemm": (ctypes.c_int, [W, p, i64, p, p, p, sz, p]),
        "lbq_gemv_noalloc": (ctypes.c_int, [W, p, p, p, p]),
        "lbq_device_fault": (ctypes.c_int, [p]),
        "lbq_selftest_wait": (ctypes.c_int, [p]),
        "lbq_read_probe": (ctypes.c_int, [p, sz, p, p]),
        "lbq_gemv_batch_workspace_bytes": (sz, [ctypes.POINTER(lbq_product), i32]),
        "lbq_gemv_batch": (ctypes.c_int, [ctypes.POINTER(lbq_product), i32, p, sz, p]),
        "lbq_gemv_batch_plan": (ctypes.c_int, [ctypes.POINTER(lbq_product), i32, i32, p, p, p]),
        "lbq_last_cuda_error": (i32, []),
        "lbq_last_cuda_error_string": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


def lib():
    return _lib


def lbq_status_string(status: int) -> str:
    return _lib.lbq_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != LBQ_OK:
        raise LbqError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def lbq_packed_layout(fmt: int, K: int, N: int):
    """-> (code_stride bytes, scale_stride elements, code_bytes, scale_bytes)."""
    cs, ss = ctypes.c_int64(), ctypes.c_int64()
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.lbq_packed_layout(fmt, K, N, ctypes.byref(cs), ctypes.byref(ss), ctypes.byref(cb),
                                  ctypes.byref(sb)), "lbq_packed_layout")
    return cs.value, ss.value, cb.value, sb.value


@dataclass
class PackedWeights:
    """A packed matrix in the library's group-of-four row order: codes uint8
    [ceil(N/4)][4 * code_stride] and (sign, 2-bit) fp16 scales [ceil(N/4)][4 * scale_stride]."""
    fmt: int
    K: int
    N: int
    codes: torch.Tensor
    scales: torch.Tensor | None

    def desc(self) -> lbq_weights:
        return lbq_weights(self.fmt, 0, self.K, self.N, self.codes.data_ptr(),
                           None if self.scales is None else self.scales.data_ptr(),
                           self.codes.stride(0) // 4,
                           0 if self.scales is None else self.scales.stride(0) // 4)

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + (0 if self.scales is None else 2 * self.scales.numel())


def lbq_pack(fmt: int, W: torch.Tensor, stream=None) -> PackedWeights:
    """Quantise + pack fp32 W [N][K] (device) into freshly allocated device buffers."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    N, K = W.shape
    cs, ss, cb, sb = lbq_packed_layout(fmt, K, N)
    G = (N + 3) // 4  # rows are stored in groups of four
    codes = torch.empty((G, 4 * cs), dtype=torch.uint8, device=W.device)
    scales = torch.empty((G, 4 * ss), dtype=torch.int16, device=W.device) if ss else None
    # (torch's allocations are 256-byte aligned, as the scales' TMA rows require)
    _check(_lib.lbq_pack(fmt, _ptr(W), K, N, _ptr(codes), _ptr(scales), _stream(stream)),
           "lbq_pack")
    return PackedWeights(fmt, K, N, codes, scales)


def lbq_unpack(pw: PackedWeights, stream=None):
    """-> (int8 codes [N][K], fp32 block scales [N][K/blk]) on the device."""
    blk = 32 if pw.fmt == LBQ_Q2RHT else 128
    out = torch.empty((pw.N, pw.K), dtype=torch.int8, device=pw.codes.device)
    sc = torch.empty((pw.N, pw.K // blk), dtype=torch.float32, device=pw.codes.device)
    d = pw.desc()
    _check(_lib.lbq_unpack(ctypes.byref(d), _ptr(out), _ptr(sc), _stream(stream)), "lbq_unpack")
    return out, sc


def lbq_rht_signs(seed: int, K: int, device="cuda", stream=None) -> torch.Tensor:
    D = torch.empty(K, dtype=torch.int8, device=device)
    _check(_lib.lbq_rht_signs(ctypes.c_uint64(seed), K, _ptr(D), _stream(stream)), "lbq_rht_signs")
    return D


def lbq_hadamard(x: torch.Tensor, D: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """fp32 x' = H D x / sqrt(512) per 512-block for bf16 x [M][K] (or [K])."""
    x2 = x if x.dim() == 2 else x.view(1, -1)
    M, K = x2.shape
    if out is None:
        out = torch.empty((M, K), dtype=torch.float32, device=x.device)
    _check(_lib.lbq_hadamard(_ptr(x2), _ptr(D), M, K, _ptr(out), _stream(stream)), "lbq_hadamard")
    return out.view(x.shape)


def lbq_device_fault() -> int:
    """Code of a bounded in-kernel wait that gave up since the last query (0: none)."""
    code = ctypes.c_uint32()
    st = _lib.lbq_device_fault(ctypes.byref(code))
    if st != LBQ_ERR_DEVICE_WAIT:
        _check(st, "lbq_device_fault")
    return code.value


def lbq_selftest_wait(stream=None) -> None:
    """Enqueues the kernel whose bounded wait runs out on purpose (fault code 11)."""
    _check(_lib.lbq_selftest_wait(_stream(stream)), "lbq_selftest_wait")


def lbq_workspace_bytes(pw: PackedWeights, M: int = 1) -> int:
    d = pw.desc()
    return int(_lib.lbq_workspace_bytes(ctypes.byref(d), M))


def workspace_for(pw: PackedWeights, M: int = 1, device=None) -> torch.Tensor | None:
    """A zero-filled workspace of lbq_workspace_bytes(pw, M) bytes (None if 0)."""
    n = lbq_workspace_bytes(pw, M)
    if n == 0:
        return None
    return torch.zeros(((n + 15) // 16) * 16, dtype=torch.uint8,
                       device=device or pw.codes.device)


def lbq_gemv(pw: PackedWeights, x: torch.Tensor, D=None, y=None, workspace=None,
             stream=None) -> torch.Tensor:
    """bf16 y [N] = W_hat x for bf16 x [K] (device)."""
    if y is None:
        y = torch.empty(pw.N, dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = workspace_for(pw, 1, x.device)
    d = pw.desc()
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.lbq_gemv(ctypes.byref(d), _ptr(x), _ptr(D), _ptr(y), _ptr(workspace), wsb,
                         _stream(stream)), "lbq_gemv")
    return y


def lbq_gemv_f32(pw: PackedWeights, x: torch.Tensor, D=None, y=None, workspace=None,
                 stream=None) -> torch.Tensor:
    """fp32 y [N] = W_hat x for bf16 x [K] (device), without the final bf16 rounding."""
    if y is None:
        y = torch.empty(pw.N, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = workspace_for(pw, 1, x.device)
    d = pw.desc()
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.lbq_gemv_f32(ctypes.byref(d), _ptr(x), _ptr(D), _ptr(y), _ptr(workspace), wsb,
                             _stream(stream)), "lbq_gemv_f32")
    return y


def lbq_gemm(pw: PackedWeights, X: torch.Tensor, D=None, Y=None, workspace=None,
             stream=None) -> torch.Tensor:
    """bf16 Y [M][N] = X W_hat^T for bf16 X [M][K] (device)."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, pw.N), dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = workspace_for(pw, M, X.device)
    d = pw.desc()
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.lbq_gemm(ctypes.byref(d), _ptr(X), M, _ptr(D), _ptr(Y), _ptr(workspace), wsb,
                         _stream(stream)), "lbq_gemm")
    return Y


def lbq_gemv_noalloc(pw: PackedWeights, x: torch.Tensor, D=None, y=None,
                     stream=None) -> torch.Tensor:
    """lbq_gemv for callers that cannot allocate device memory: the library's own fixed
    scratch array replaces the workspace (see include/lbq.h). Only `y` is allocated
    here, and only when the caller passes none."""
    if y is None:
        y = torch.empty(pw.N, dtype=torch.bfloat16, device=x.device)
    d = pw.desc()
    _check(_lib.lbq_gemv_noalloc(ctypes.byref(d), _ptr(x), _ptr(D), _ptr(y), _stream(stream)),
           "lbq_gemv_noalloc")
    return y


def lbq_read_probe(buf: torch.Tensor, sink: torch.Tensor, nbytes: int | None = None,
                   stream=None) -> None:
    """Reads nbytes (default: all) of a device tensor once, XOR-folding the words into
    sink (an int32 device tensor): the plain read-stream rate, a bandwidth denominator."""
    n = buf.numel() * buf.element_size() if nbytes is None else int(nbytes)
    _check(_lib.lbq_read_probe(_ptr(buf), n, _ptr(sink), _stream(stream)), "lbq_read_probe")


class ProductList:
    """A host array of lbq_product records for lbq_gemv_batch, built once from
    (packed weights, x, D or None, y) tuples; the tensors must outlive its use."""

    def __init__(self, items):
        self.items = list(items)
        self.arr = (lbq_product * len(self.items))()
        for i, (pw, x, D, y) in enumerate(self.items):
            self.arr[i].w = pw.desc()
            self.arr[i].x = x.data_ptr()
            self.arr[i].D = None if D is None else D.data_ptr()
            self.arr[i].y = y.data_ptr()

    def __len__(self):
        return len(self.items)


def lbq_gemv_batch_plan(arr, n: int, ctas: int):
    """The schedule one launch of lbq_gemv_batch gives a list of one format (host only):
    (pieces per product, CTA boundaries [ctas + 1], total unit-slices). `arr` is a
    ctypes array of lbq_product (ProductList.arr, or records built by hand)."""
    pieces = (ctypes.c_int32 * n)()
    bound = (ctypes.c_int64 * (ctas + 1))()
    total = ctypes.c_int64()
    _check(_lib.lbq_gemv_batch_plan(arr, n, ctas, pieces, bound, ctypes.byref(total)),
           "lbq_gemv_batch_plan")
    return list(pieces), list(bound), int(total.value)


def lbq_gemv_batch_workspace_bytes(plist: ProductList) -> int:
    return int(_lib.lbq_gemv_batch_workspace_bytes(plist.arr, len(plist)))


def lbq_gemv_batch(plist: ProductList, workspace=None, stream=None) -> None:
    """Every product of the list (independent batch-1 products, see include/lbq.h), one
    launch per format present and LBQ_BATCH_MAX products of it. The workspace's first
    64 KB must be zero when it is first used (workspace_for_batch gives such a buffer)."""
    if workspace is None:
        workspace = workspace_for_batch(plist)
    wsb = workspace.numel() * workspace.element_size()
    _check(_lib.lbq_gemv_batch(plist.arr, len(plist), _ptr(workspace), wsb, _stream(stream)),
           "lbq_gemv_batch")


def workspace_for_batch(plist: ProductList, device=None) -> torch.Tensor:
    n = lbq_gemv_batch_workspace_bytes(plist)
    if n == 0:
        _check(LBQ_ERR_ARG, "lbq_gemv_batch_workspace_bytes")
    dev = device or plist.items[0][1].device
    return torch.zeros(((n + 15) // 16) * 16, dtype=torch.uint8, device=dev)
