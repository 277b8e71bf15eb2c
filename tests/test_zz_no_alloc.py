"""lbq_gemv_noalloc: the batch-1 product for callers that cannot allocate device memory.

Such a caller (a host that reaches the library only through its C interface and
has no device allocator, or one that must not call cudaMalloc once running) gets
its scratch from an array compiled into the library instead of a workspace it
passes in. These tests call that entry point through the C ABI and check it
against lbq_gemv, within the same 2^-8 * sum|w_hat x| bound every product test
uses, on two calls in a row (the second sees what the first left in the array).
The file is named to run last, and needs nothing from the other test files.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_weight_only_ternary_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 2.0 ** -8


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_only_ternary_b200 import build
    build.build()
    from bit_weight_only_ternary_b200 import lbq
    return lbq


def _bound(orc, fmt, W, x, D_orc):
    codes, scales = orc.pack(fmt, W.numpy())
    Y, B = orc.gemm(fmt, codes, scales, W.shape[1], synth.bf16_bits(x), D_orc)
    return Y[0], B[0]


@pytest.mark.parametrize("fmt", (1, 2, 3))
@pytest.mark.parametrize("N,K", [(300, 2048), (7168, 5120)])
def test_noalloc_matches_gemv_on_two_calls(L, orc, fmt, N, K):
    W = synth.weights(N, K, 600 + fmt + K)
    x = synth.activations(1, K, 700 + K)
    pw = L.lbq_pack(fmt, W.cuda())
    D = L.lbq_rht_signs(11, K) if fmt == 3 else None
    D_orc = orc.rht_signs(11, K) if fmt == 3 else None
    xd = x[0].cuda()
    y_ref = L.lbq_gemv(pw, xd, D).double().cpu().numpy()
    Y, B = _bound(orc, fmt, W, x, D_orc)
    lim = TOL * B
    for _ in range(2):
        y = torch.full((N,), 3.0, dtype=torch.bfloat16, device="cuda")
        d = pw.desc()
        st = L.lib().lbq_gemv_noalloc(ctypes.byref(d), ctypes.c_void_p(xd.data_ptr()),
                                      None if D is None else ctypes.c_void_p(D.data_ptr()),
                                      ctypes.c_void_p(y.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == L.LBQ_OK, L.lbq_status_string(st)
        got = y.double().cpu().numpy()
        assert np.all(np.abs(got - y_ref) <= lim), "differs from lbq_gemv beyond the bound"
        assert np.all(np.abs(got - Y) <= lim), "differs from the oracle beyond the bound"


def test_noalloc_rejects_products_needing_more_scratch(L):
    """A product whose scratch need exceeds the fixed array is refused before any launch
    (fake, well-aligned device addresses: nothing may be read or written)."""
    lib = L.lib()
    fake = ctypes.c_void_p(1 << 40)
    found = 0
    for fmt, K, N in [(3, 1 << 21, 1), (1, 5120, 1 << 19), (2, 5120, 1 << 19), (1, 17408, 1 << 19)]:
        cs, ss, _, _ = L.lbq_packed_layout(fmt, K, 1)
        d = L.lbq_weights(fmt, 0, K, N, fake.value, None if fmt == 1 else fake.value, cs, ss)
        need = lib.lbq_workspace_bytes(ctypes.byref(d), 1)
        if need > L.LBQ_NOALLOC_SCRATCH_BYTES:
            found += 1
            st = lib.lbq_gemv_noalloc(ctypes.byref(d), fake, fake, fake, None)
            assert st == L.LBQ_ERR_WORKSPACE
    assert found, "no test shape needs more than the fixed scratch"
    # invalid arguments are refused with the same statuses as lbq_gemv, checked before
    # the scratch size: a null x or y, or a misaligned x, on a product too large for the
    # array is an argument error, not a scratch error
    cs, _, _, _ = L.lbq_packed_layout(1, 5120, 1)
    big = L.lbq_weights(1, 0, 5120, 1 << 20, fake.value, None, cs, 0)
    assert lib.lbq_gemv_noalloc(ctypes.byref(big), None, None, fake, None) == L.LBQ_ERR_ARG
    assert lib.lbq_gemv_noalloc(ctypes.byref(big), fake, None, None, None) == L.LBQ_ERR_ARG
    assert lib.lbq_gemv_noalloc(ctypes.byref(big), ctypes.c_void_p(fake.value + 2), None, fake,
                                None) == L.LBQ_ERR_ALIGN
    # more rows than a split product may have: a shape error, as from lbq_gemv
    huge = L.lbq_weights(1, 0, 5120, (1 << 19) + 4, fake.value, None, cs, 0)
    assert lib.lbq_gemv_noalloc(ctypes.byref(huge), fake, None, fake, None) == L.LBQ_ERR_SHAPE
    assert lib.lbq_gemv(ctypes.byref(huge), fake, None, fake, fake, 1 << 30, None) == L.LBQ_ERR_SHAPE
    d = L.lbq_weights(1, 0, 500, 4, fake.value, None, 32, 0)
    assert lib.lbq_gemv_noalloc(ctypes.byref(d), fake, None, fake, None) == L.LBQ_ERR_SHAPE
    assert lib.lbq_gemv_noalloc(None, fake, None, fake, None) == L.LBQ_ERR_ARG
