"""lbq_gemv_batch: many independent batch-1 products in one launch.

Every product of a list must give what lbq_gemv gives it: codes are the same packed
bytes, outputs within 2^-8 * sum_k |w_hat x| of the fp64 oracle. Lists mix formats,
shapes (one K-slice or many, a partial last slice, N not a multiple of 16), repeat
(the workspace counters must come back to zero), and replay inside a CUDA graph.
"""
import os

import numpy as np
import pytest
import torch

from bit_weight_only_ternary_b200 import synth

pytestmark = pytest.mark.gpu
TERN5, SIGN1, Q2RHT = 1, 2, 3
TOL = 2.0 ** -8
NTHREADS = max(1, min(32, os.cpu_count() or 1))


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_only_ternary_b200 import build
    build.build()
    from bit_weight_only_ternary_b200 import lbq
    return lbq


def _make(L, orc, cases, seed):
    """Packed products (fmt, N, K) with their oracle results."""
    out = []
    for i, (fmt, N, K) in enumerate(cases):
        W = synth.weights(N, K, seed + 17 * i)
        x = synth.activations(1, K, seed + 17 * i + 1)
        pw = L.lbq_pack(fmt, W.cuda())
        codes, scales = orc.pack(fmt, W.numpy())
        D = L.lbq_rht_signs(seed + i, K) if fmt == Q2RHT else None
        Do = orc.rht_signs(seed + i, K) if fmt == Q2RHT else None
        Y, B = orc.gemm(fmt, codes, scales, K, synth.bf16_bits(x), Do, nthreads=NTHREADS)
        y = torch.full((N,), 5.0, dtype=torch.bfloat16, device="cuda")
        out.append(dict(fmt=fmt, N=N, K=K, pw=pw, x=x[0].cuda(), D=D, y=y, Y=Y[0], B=B[0]))
    return out


def _check(prods, what):
    for i, p in enumerate(prods):
        got = p["y"].double().cpu().numpy()
        err = np.abs(got - p["Y"])
        lim = TOL * p["B"]
        bad = err > lim
        assert not bad.any(), (f"{what}: product {i} (fmt {p['fmt']} {p['N']}x{p['K']}): "
                               f"{bad.sum()} outputs out of bound, first {np.argwhere(bad)[0]}")


MIXED = [(TERN5, 7168, 5120), (Q2RHT, 5120, 5120), (TERN5, 34816, 5120), (TERN5, 5120, 17408),
         (SIGN1, 300, 2048), (TERN5, 256, 512), (TERN5, 17, 1152), (Q2RHT, 130, 1024),
         (SIGN1, 1000, 1152), (TERN5, 1, 128), (TERN5, 4100, 640)]


def test_batch_mixed_list_matches_oracle(L, orc):
    prods = _make(L, orc, MIXED, 100)
    plist = L.ProductList([(p["pw"], p["x"], p["D"], p["y"]) for p in prods])
    ws = L.workspace_for_batch(plist)
    for rep in range(3):  # the counters are reset by every launch
        for p in prods:
            p["y"].fill_(5.0)
        L.lbq_gemv_batch(plist, ws)
        torch.cuda.synchronize()
        _check(prods, f"call {rep}")
        assert not ws[:65536].any(), "counters not left at zero"
    assert L.lbq_device_fault() == 0


@pytest.mark.parametrize("fmt", (TERN5, SIGN1, Q2RHT))
def test_batch_one_format_27b_layer_and_determinism(L, orc, fmt):
    """The four products of a 27B-shaped layer in one format (the kernel compiled for
    that format alone), twice: bit-identical results (fixed-order split-K sums)."""
    cases = [(fmt, N, K) for _, K, N in synth.LAYER_SHAPES]
    prods = _make(L, orc, cases, 300 + fmt)
    plist = L.ProductList([(p["pw"], p["x"], p["D"], p["y"]) for p in prods])
    ws = L.workspace_for_batch(plist)
    L.lbq_gemv_batch(plist, ws)
    torch.cuda.synchronize()
    _check(prods, f"fmt {fmt}")
    first = [p["y"].clone() for p in prods]
    L.lbq_gemv_batch(plist, ws)
    torch.cuda.synchronize()
    for a, p in zip(first, prods):
        assert torch.equal(a, p["y"])


def test_batch_matches_lbq_gemv_and_more_than_one_launch(L, orc):
    """A list longer than one launch takes (LBQ_BATCH_MAX): consecutive launches share
    the workspace; every output equals the single-product call's within the bound."""
    n = L.LBQ_BATCH_MAX + 9
    shapes = [(TERN5, 256 + 16 * (i % 5), 1024 + 512 * (i % 3)) for i in range(n)]
    prods = []
    for i, (fmt, N, K) in enumerate(shapes):
        W = synth.weights(N, K, 5000 + i)
        pw = L.lbq_pack(fmt, W.cuda())
        x = synth.activations(1, K, 6000 + i, device="cuda")[0]
        prods.append((pw, x, None, torch.empty(N, dtype=torch.bfloat16, device="cuda")))
    plist = L.ProductList(prods)
    L.lbq_gemv_batch(plist)
    torch.cuda.synchronize()
    for i in range(0, n, 23):
        pw, x, _, y = prods[i]
        ref = L.lbq_gemv(pw, x).double()
        W = synth.weights(pw.N, pw.K, 5000 + i)
        codes, scales = orc.pack(TERN5, W.numpy())
        Y, B = orc.gemm(TERN5, codes, scales, pw.K, synth.bf16_bits(x.view(1, -1)), None)
        lim = torch.from_numpy(TOL * B[0]).cuda()
        assert torch.all((y.double() - ref).abs() <= 2 * lim)
        assert torch.all((y.double() - torch.from_numpy(Y[0]).cuda()).abs() <= lim)


def test_batch_schedule_edges(L, orc):
    """Lists that reach the corners of the schedule: a one-row product alone (a CTA's
    share is empty on all but one CTA), products of few rows and many K-slices (split
    along K into up to one piece per slice, added by the second kernel), and such a
    product beside ordinary ones (split and whole-K products in one launch)."""
    lists = [
        [(TERN5, 1, 128)],
        [(TERN5, 16, 65536)],
        [(SIGN1, 5, 131072), (Q2RHT, 19, 32768)],
        [(TERN5, 7168, 5120), (TERN5, 16, 65536), (TERN5, 33, 2560), (TERN5, 3, 640)],
        [(Q2RHT, 1, 512), (Q2RHT, 4100, 1024), (Q2RHT, 2, 49152)],
    ]
    for li, cases in enumerate(lists):
        prods = _make(L, orc, cases, 3000 + 100 * li)
        plist = L.ProductList([(p["pw"], p["x"], p["D"], p["y"]) for p in prods])
        ws = L.workspace_for_batch(plist)
        for rep in range(2):
            for p in prods:
                p["y"].fill_(5.0)
            L.lbq_gemv_batch(plist, ws)
            torch.cuda.synchronize()
            _check(prods, f"list {li} call {rep}")
        assert not ws[:65536].any(), "counters not left at zero"
    assert L.lbq_device_fault() == 0


def test_batch_many_row_chunks(L, orc):
    """2.4 million rows of one product (150000 units, about 1014 a CTA): each CTA runs
    its rows in more than one chunk of running sums. The rows repeat a 1024-row block,
    so every output must equal its block row's exactly (a row's sum does not depend on
    where it falls), and the block rows must match the oracle."""
    Nb, K, reps = 1024, 512, 2344
    N = Nb * reps
    Wb = synth.weights(Nb, K, 4242)
    x = synth.activations(1, K, 4243)
    pw = L.lbq_pack(TERN5, Wb.cuda().repeat(reps, 1))
    y = torch.full((N,), 5.0, dtype=torch.bfloat16, device="cuda")
    L.lbq_gemv_batch(L.ProductList([(pw, x[0].cuda(), None, y)]))
    torch.cuda.synchronize()
    codes, scales = orc.pack(TERN5, Wb.numpy())
    Y, B = orc.gemm(TERN5, codes, scales, K, synth.bf16_bits(x), None, nthreads=NTHREADS)
    yb = y[:Nb].double().cpu().numpy()
    assert np.all(np.abs(yb - Y[0]) <= TOL * B[0])
    assert torch.equal(y.view(reps, Nb), y[:Nb].expand(reps, Nb)), "a repeated row differs"
    assert L.lbq_device_fault() == 0


def test_batch_in_cuda_graph(L, orc):
    prods = _make(L, orc, [(TERN5, 7168, 5120), (TERN5, 5120, 17408), (SIGN1, 512, 5120)], 900)
    plist = L.ProductList([(p["pw"], p["x"], p["D"], p["y"]) for p in prods])
    ws = L.workspace_for_batch(plist)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        L.lbq_gemv_batch(plist, ws, stream=s)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            L.lbq_gemv_batch(plist, ws, stream=s)
    for rep in range(3):
        for p in prods:
            p["y"].fill_(5.0)
        with torch.cuda.stream(s):
            g.replay()
        torch.cuda.synchronize()
        _check(prods, f"graph replay {rep}")


def test_batch_rejects_overlapping_and_bad_lists(L):
    N, K = 64, 512
    pw = L.lbq_pack(TERN5, synth.weights(N, K, 3).cuda())
    x = synth.activations(1, K, 4)[0].cuda()
    y = torch.empty(N, dtype=torch.bfloat16, device="cuda")
    big = torch.empty(K, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LbqError) as e:  # y of one product is x of another
        L.lbq_gemv_batch(L.ProductList([(pw, x, None, big[:N]), (pw, big, None, y)]))
    assert e.value.status == L.LBQ_ERR_ARG
    with pytest.raises(L.LbqError) as e:  # two outputs overlap
        L.lbq_gemv_batch(L.ProductList([(pw, x, None, big[:N]), (pw, x, None, big[8:8 + N])]))
    assert e.value.status == L.LBQ_ERR_ARG
    lib = L.lib()
    assert lib.lbq_gemv_batch(None, 1, None, 0, None) == L.LBQ_ERR_ARG
    pl = L.ProductList([(pw, x, None, y)])
    assert lib.lbq_gemv_batch(pl.arr, 0, None, 0, None) == L.LBQ_ERR_ARG
    assert lib.lbq_gemv_batch(pl.arr, 1, None, 0, None) == L.LBQ_ERR_WORKSPACE
