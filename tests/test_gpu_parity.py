"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Codes must be bit-exact; products must satisfy |y_gpu - y_ref| <= 2^-8 * sum_k |w_hat x|
per output element, the acceptance bound of the method (y_ref and the bound are the
oracle's, computed in fp64 from the oracle's own packing of the same seeded W).
"""
import os

import numpy as np
import pytest
import torch

from bit_weight_only_ternary_b200 import synth

pytestmark = pytest.mark.gpu
TERN5, SIGN1, Q2RHT = 1, 2, 3
FMTS = (TERN5, SIGN1, Q2RHT)
TOL = 2.0 ** -8
NTHREADS = max(1, min(32, os.cpu_count() or 1))


@pytest.fixture(scope="module")
def L():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_only_ternary_b200 import build
    build.build()
    from bit_weight_only_ternary_b200 import lbq
    return lbq


def _pack_both(L, orc, fmt, W_cpu):
    pw = L.lbq_pack(fmt, W_cpu.cuda())
    codes, scales = orc.pack(fmt, W_cpu.numpy())
    return pw, codes, scales


def _assert_codes_equal(orc, pw, codes, scales):
    """The library's buffers against the oracle's rows put in group-of-four order."""
    got = pw.codes.cpu().numpy()
    want = orc.group4(codes)
    assert got.shape == want.shape
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}"
    if scales is not None:
        gs = pw.scales.cpu().numpy().view(np.uint16)
        assert np.array_equal(gs, orc.group4(scales)), "scales differ"


def _check_products(y, Y, B, what=""):
    yg = y.float().cpu().double().numpy().reshape(Y.shape)
    err = np.abs(yg - Y)
    lim = TOL * B
    bad = err > lim
    if bad.any():
        i = np.argwhere(bad)[0]
        pytest.fail(f"{what}: {bad.sum()} of {bad.size} outputs out of bound; first {i.tolist()}: "
                    f"gpu {yg[tuple(i)]!r} ref {Y[tuple(i)]!r} bound {lim[tuple(i)]!r}")
    return float((err / np.maximum(lim, 1e-300)).max())


def _oracle_D(orc, fmt, K, seed=99):
    return orc.rht_signs(seed, K) if fmt == Q2RHT else None


def _gpu_D(L, fmt, K, seed=99):
    return L.lbq_rht_signs(seed, K) if fmt == Q2RHT else None


# ----------------------------------------------------------------------------- codes

SHAPES = [(256, 512), (37, 1536), (1, 512), (5, 1024)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", SHAPES)
def test_pack_bit_exact(L, orc, fmt, N, K):
    W = synth.weights(N, K, 1000 + N + K)
    pw, codes, scales = _pack_both(L, orc, fmt, W)
    _assert_codes_equal(orc, pw, codes, scales)


@pytest.mark.parametrize("fmt", (TERN5, SIGN1))
@pytest.mark.parametrize("K", (128, 384, 640))
def test_pack_ragged_k_and_row_padding(L, orc, fmt, K):
    W = synth.weights(9, K, 5 + K)
    pw, codes, scales = _pack_both(L, orc, fmt, W)
    _assert_codes_equal(orc, pw, codes, scales)


@pytest.mark.parametrize("fmt", FMTS)
def test_pack_adversarial_values(L, orc, fmt):
    K = 512
    W = synth.weights(8, K, 77)
    W[0] = 0.0                                   # all-zero row: scale 0
    W[1, :128] = 0.25                            # ties: |w| = s/2 and w = +-s, -0.0
    W[1, 0], W[1, 1], W[1, 2], W[1, 3] = 0.125, 0.375, -0.0, -0.25
    W[1, 4] = -0.125
    W[2] *= 1e7                                  # scale saturates at 65504
    W[3] *= 1e-12                                # tiny / subnormal fp16 scales
    W[4, ::2] = -W[4, 1::2]                      # exact +- pairs
    W[5, 32:64] = torch.tensor([-1.5, -1.0, -0.5, 0.0, 0.5, 1.0, 1.5, -1.0] * 4)  # 2-bit ties
    pw, codes, scales = _pack_both(L, orc, fmt, W)
    _assert_codes_equal(orc, pw, codes, scales)


@pytest.mark.parametrize("fmt", FMTS)
def test_unpack_bit_exact(L, orc, fmt):
    N, K = 33, 1024
    W = synth.weights(N, K, 4242)
    pw, codes, scales = _pack_both(L, orc, fmt, W)
    t, s = L.lbq_unpack(pw)
    ot, os_ = orc.unpack(fmt, codes, scales, K)
    assert np.array_equal(t.cpu().numpy(), ot)
    assert np.array_equal(s.cpu().double().numpy(), os_)


@pytest.mark.parametrize("fmt", FMTS)
def test_pack_sampled_rows_of_27b_gate_up(L, orc, fmt):
    N, K = 2 * synth.FFN, synth.HIDDEN
    Wd = synth.weights(N, K, 31337, device="cuda")
    pw = L.lbq_pack(fmt, Wd)
    groups = torch.tensor([0, 1, 777, 3000, N // 8, N // 4 - 2, N // 4 - 1])  # groups of 4 rows
    rows = (4 * groups[:, None] + torch.arange(4)[None, :]).reshape(-1)
    codes, scales = orc.pack(fmt, Wd[rows.cuda()].cpu().numpy())
    assert np.array_equal(pw.codes[groups.cuda()].cpu().numpy(), orc.group4(codes))
    if scales is not None:
        assert np.array_equal(pw.scales[groups.cuda()].cpu().numpy().view(np.uint16),
                              orc.group4(scales))


# ----------------------------------------------------------------------------- rotation

@pytest.mark.parametrize("K", (512, 5120, 17408))
def test_rht_signs_bit_exact(L, orc, K):
    for seed in (0, 1, 2 ** 63 + 5):
        assert np.array_equal(L.lbq_rht_signs(seed, K).cpu().numpy(), orc.rht_signs(seed, K))


@pytest.mark.parametrize("M,K", [(1, 512), (3, 5120), (2, 17408)])
def test_hadamard_parity(L, orc, M, K):
    x = synth.activations(M, K, 55)
    D = L.lbq_rht_signs(7, K)
    out = L.lbq_hadamard(x.cuda(), D).cpu().double().numpy()
    ref = orc.hadamard(x.double().numpy(), orc.rht_signs(7, K))
    # bound: 2^-8 * sum_{j in block} |x_j| / sqrt(512), per element
    bsum = np.abs(x.double().numpy()).reshape(M, K // 512, 512).sum(-1) / np.sqrt(512)
    lim = TOL * np.repeat(bsum, 512, axis=1)
    assert np.all(np.abs(out - ref) <= lim)


# ----------------------------------------------------------------------------- products

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", SHAPES + [(300, 2048)])
def test_gemv_parity(L, orc, fmt, N, K):
    W = synth.weights(N, K, 2000 + N + K)
    x = synth.activations(1, K, 3000 + K)
    pw, codes, scales = _pack_both(L, orc, fmt, W)
    y = L.lbq_gemv(pw, x[0].cuda(), _gpu_D(L, fmt, K))
    Y, B = orc.gemm(fmt, codes, scales, K, synth.bf16_bits(x), _oracle_D(orc, fmt, K))
    _check_products(y, Y[0], B[0], f"fmt {fmt} {N}x{K}")


@pytest.mark.parametrize("fmt", (TERN5, SIGN1))
@pytest.mark.parametrize("N,K", [(17, 1152), (130, 640), (1, 128)])
def test_gemv_partial_last_slice(L, orc, fmt, N, K):
    """K whose last slice holds fewer blocks than a full one (an odd number for the
    1-bit format: its scale copy rounds up into the row's padding), ragged N."""
    W = synth.weights(N, K, 2100 + N + K)
    x = synth.activations(1, K, 3100 + K)
    pw, codes, scales = _pack_both(L, orc, fmt, W)
    y = L.lbq_gemv(pw, x[0].cuda())
    Y, B = orc.gemm(fmt, codes, scales, K, synth.bf16_bits(x), None)
    _check_products(y, Y[0], B[0], f"fmt {fmt} {N}x{K}")


@pytest.mark.parametrize("fmt", FMTS)
def test_gemv_one_27b_layer(L, orc, fmt):
    """Every output of one 27B-shaped layer (QKV, O, gate+up, down), full oracle check."""
    for mi, (name, K, N) in enumerate(synth.LAYER_SHAPES):
        Wd = synth.weights(N, K, synth.seed_of(10, 0, mi), device="cuda")
        pw = L.lbq_pack(fmt, Wd)
        codes, scales = orc.pack(fmt, Wd.cpu().numpy())
        del Wd
        _assert_codes_equal(orc, pw, codes, scales)
        x = synth.activations(1, K, synth.seed_of(20, 0, mi), device="cuda")
        y = L.lbq_gemv(pw, x[0], _gpu_D(L, fmt, K))
        Y, B = orc.gemm(fmt, codes, scales, K, synth.bf16_bits(x), _oracle_D(orc, fmt, K),
                        nthreads=NTHREADS)
        _check_products(y, Y[0], B[0], f"fmt {fmt} {name}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", (2, 8, 13, 32, 100))
def test_gemm_parity(L, orc, fmt, M):
    N, K = 384, 1536
    W = synth.weights(N, K, 4000 + M)
    X = synth.activations(M, K, 5000 + M)
    pw, codes, scales = _pack_both(L, orc, fmt, W)
    Yg = L.lbq_gemm(pw, X.cuda(), _gpu_D(L, fmt, K))
    Y, B = orc.gemm(fmt, codes, scales, K, synth.bf16_bits(X), _oracle_D(orc, fmt, K),
                    nthreads=NTHREADS)
    _check_products(Yg, Y, B, f"fmt {fmt} M={M}")


@pytest.mark.parametrize("fmt", FMTS)
def test_zero_weights_and_zero_input_give_exact_zero(L, orc, fmt):
    N, K = 64, 1024
    W = synth.weights(N, K, 8)
    W[5:9] = 0.0
    pw = L.lbq_pack(fmt, W.cuda())
    x = synth.activations(1, K, 9)[0].cuda()
    y = L.lbq_gemv(pw, x, _gpu_D(L, fmt, K)).float().cpu()
    assert torch.all(y[5:9] == 0)
    y0 = L.lbq_gemv(pw, torch.zeros(K, dtype=torch.bfloat16, device="cuda"), _gpu_D(L, fmt, K))
    assert torch.all(y0.float() == 0)


@pytest.mark.parametrize("fmt", FMTS)
def test_repeated_calls_are_deterministic(L, fmt):
    N, K = 5120, 5120
    pw = L.lbq_pack(fmt, synth.weights(N, K, 12, device="cuda"))
    x = synth.activations(1, K, 13, device="cuda")[0]
    D = _gpu_D(L, fmt, K)
    ws = L.workspace_for(pw, 1)
    a = L.lbq_gemv(pw, x, D, workspace=ws).clone()
    for _ in range(3):
        b = L.lbq_gemv(pw, x, D, workspace=ws)
        assert torch.equal(a, b)


def test_errors_enqueue_nothing(L):
    N, K = 16, 512
    pw = L.lbq_pack(TERN5, synth.weights(N, K, 3).cuda())
    x = synth.activations(1, K, 4)[0].cuda()
    y = torch.full((N,), 7.0, dtype=torch.bfloat16, device="cuda")
    bad = L.PackedWeights(TERN5, K + 1, N, pw.codes, None)
    with pytest.raises(L.LbqError) as e:
        L.lbq_gemv(bad, x, None, y)
    assert e.value.status == L.LBQ_ERR_SHAPE
    xb = torch.zeros(K + 8, dtype=torch.bfloat16, device="cuda")[1:K + 1]  # 2-byte offset
    with pytest.raises(L.LbqError) as e:
        L.lbq_gemv(pw, xb, None, y)
    assert e.value.status == L.LBQ_ERR_ALIGN
    torch.cuda.synchronize()
    assert torch.all(y.float() == 7.0)


def test_one_workspace_serves_products_of_any_shape(L, orc):
    """One zero-filled workspace used in turn by products of different shapes, formats and M
    (the counters at its start must survive every other product's scratch data)."""
    cases = [(TERN5, 4352, 5120, 1), (TERN5, 640, 17408, 1), (SIGN1, 3000, 5120, 1),
             (Q2RHT, 700, 5120, 1), (TERN5, 2000, 1024, 1), (Q2RHT, 96, 1024, 4),
             (SIGN1, 5000, 2048, 1)]
    built = []
    for i, (fmt, N, K, M) in enumerate(cases):
        W = synth.weights(N, K, 9100 + i)
        X = synth.activations(M, K, 9200 + i)
        pw, codes, scales = _pack_both(L, orc, fmt, W)
        Y, B = orc.gemm(fmt, codes, scales, K, synth.bf16_bits(X), _oracle_D(orc, fmt, K),
                        nthreads=NTHREADS)
        built.append((pw, X.cuda(), _gpu_D(L, fmt, K), Y, B, M))
    need = max(L.lbq_workspace_bytes(pw, M) for pw, _, _, _, _, M in built)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for order in (built, built[::-1], built):
        for pw, X, D, Y, B, M in order:
            out = L.lbq_gemv(pw, X[0], D, workspace=ws) if M == 1 else \
                L.lbq_gemm(pw, X, D, workspace=ws)
            _check_products(out, Y if M > 1 else Y[0], B if M > 1 else B[0], f"shared ws {pw.N}x{pw.K}")
    torch.cuda.synchronize()
    assert not ws[:65536].any(), "counters not left at zero"


def test_no_bounded_device_wait_gave_up(L):
    """After every product above, no in-kernel wait ran out (the fault record is clear)."""
    torch.cuda.synchronize()
    assert L.lbq_device_fault() == 0


@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (3, 130, 640), (13, 130, 640), (16, 128, 128),
                                   (128, 384, 1024), (512, 256, 5120), (200, 1000, 2048)])
def test_ternary_gemm_tensor_cores(L, orc, M, N, K):
    """The ternary product: ragged M and N, K from one block to 40 (M <= 3 runs one
    batch-1 product per row, larger M the tensor cores)."""
    W = synth.weights(N, K, 6000 + M + N)
    X = synth.activations(M, K, 7000 + M)
    pw, codes, scales = _pack_both(L, orc, TERN5, W)
    Yg = L.lbq_gemm(pw, X.cuda())
    Y, B = orc.gemm(TERN5, codes, scales, K, synth.bf16_bits(X), None, nthreads=NTHREADS)
    _check_products(Yg, Y, B, f"tern gemm M={M} N={N} K={K}")


def test_ternary_gemm_large_activations_are_scaled_into_fp16(L, orc):
    """Rows of X beyond fp16's range (bf16 values up to 3e38 are finite) still come out right,
    including rows whose scale-back factor 2^e is itself outside fp32's normal range."""
    M, N, K = 6, 128, 512
    W = synth.weights(N, K, 61)
    X = synth.activations(M, K, 62)
    X[1] *= 2.0 ** 40
    X[2] *= 2.0 ** -30
    X[3] *= 2.0 ** -125   # e = ilogb(max|x|) - 14 < -126: the ldexpf branch
    X[4] *= 2.0 ** 100    # large e, still a normal power of two
    pw, codes, scales = _pack_both(L, orc, TERN5, W)
    Yg = L.lbq_gemm(pw, X.cuda())
    Y, B = orc.gemm(TERN5, codes, scales, K, synth.bf16_bits(X), None)
    _check_products(Yg, Y, B, "scaled rows")


def test_ternary_gemm_27b_gate_up_sampled(L, orc):
    """M = 512 tokens through a full 27B gate+up matrix; sampled rows checked exactly."""
    N, K, M = 2 * synth.FFN, synth.HIDDEN, 512
    Wd = synth.weights(N, K, 777, device="cuda")
    pw = L.lbq_pack(TERN5, Wd)
    X = synth.activations(M, K, 778, device="cuda")
    Yg = L.lbq_gemm(pw, X)
    rows = torch.tensor([0, 5, 127, 128, 9999, N - 129, N - 1], device="cuda")
    codes, scales = orc.pack(TERN5, Wd[rows].cpu().numpy())
    Y, B = orc.gemm(TERN5, codes, scales, K, synth.bf16_bits(X), None, nthreads=NTHREADS)
    _check_products(Yg[:, rows], Y, B, "27B gate+up, M=512")


def test_bounded_wait_gives_up_and_device_stays_usable(L, orc):
    """A kernel wait that runs out (an mbarrier nothing arrives on, 20 ms limit) records
    its code, returns instead of hanging, and the next product still runs correctly."""
    assert L.lbq_device_fault() == 0
    L.lbq_selftest_wait()
    torch.cuda.synchronize()
    assert L.lbq_device_fault() == 11
    assert L.lbq_device_fault() == 0  # the record is cleared by the query
    N, K = 64, 1024
    W = synth.weights(N, K, 91)
    x = synth.activations(1, K, 92)
    pw, codes, scales = _pack_both(L, orc, TERN5, W)
    y = L.lbq_gemv(pw, x[0].cuda())
    Y, B = orc.gemm(TERN5, codes, scales, K, synth.bf16_bits(x), None)
    _check_products(y, Y[0], B[0], "after a timed-out wait")
    assert L.lbq_device_fault() == 0


# ------------------------------------------------------- tensor-core product: edge cases

def _spread_rows(M, K, seed):
    """bf16 activation rows that fp16 cannot hold after one power-of-two scaling, next to
    ordinary ones: row 0 = [2^40, 1.0078125, ...], row 1 = [2^34, 1.0078125, ...], row 2 =
    random signs and exponents over 2^-60 .. 2^60, row 3 = N(0, 1), row 4 = zeros, the
    rest N(0, 1) with a few entries scaled by 2^-45."""
    assert M >= 4
    g = torch.Generator().manual_seed(seed)
    X = torch.randn((max(M, 5), K), generator=g)
    X[0] = 1.0078125
    X[0, 0] = 2.0 ** 40
    X[1] = 1.0078125
    X[1, 0] = 2.0 ** 34
    e = torch.randint(-60, 61, (K,), generator=g).double()
    X[2] = (torch.sign(torch.randn(K, generator=g)) * (1 + torch.rand(K, generator=g)) * 2.0 ** e).float()
    X[4] = 0.0
    X = X[:M]
    for r in range(5, M):
        X[r, r % K] *= 2.0 ** -45
    return X.to(torch.bfloat16)


def _spread_weights(N, K, seed):
    """Rows whose trit is 0 at k = 0 and +1 elsewhere (the large entry of rows 0 and 1
    meets a zero weight), every fourth row ordinary N(0, 0.02^2) weights."""
    W = torch.full((N, K), 0.02)
    W[:, 0] = 0.0
    R = synth.weights(N, K, seed)
    W[::4] = R[::4]
    return W


@pytest.mark.parametrize("M,N,K", [(6, 128, 512),      # one tile, Y through one TMA store
                                   (6, 256, 5120),     # K split over the grid: fp32 partials
                                   (4, 130, 512),      # N * 2 not 16-aligned: direct stores
                                   (20, 130, 1024),    # direct stores and a K split
                                   (300, 1000, 2048)]) # two token tiles
def test_ternary_gemm_rows_wider_than_fp16(L, orc, M, N, K):
    """Activation rows whose values span more than fp16 holds after a power-of-two scaling
    (2^40 beside 1.0078125, exponents over +-60) meet the bound like any other row."""
    W = _spread_weights(N, K, 8100 + N)
    X = _spread_rows(M, K, 8200 + M)
    pw, codes, scales = _pack_both(L, orc, TERN5, W)
    Yg = L.lbq_gemm(pw, X.cuda())
    Y, B = orc.gemm(TERN5, codes, scales, K, synth.bf16_bits(X), None, nthreads=NTHREADS)
    _check_products(Yg, Y, B, f"wide rows M={M} N={N} K={K}")
    assert L.lbq_device_fault() == 0


@pytest.mark.parametrize("M,N,K", [(8, 1, 512), (16, 129, 640), (5, 4 * 33 + 1, 1024)])
def test_ternary_gemm_tensor_core_ragged_n(L, orc, M, N, K):
    W = synth.weights(N, K, 8300 + N)
    X = synth.activations(M, K, 8400 + M)
    pw, codes, scales = _pack_both(L, orc, TERN5, W)
    Yg = L.lbq_gemm(pw, X.cuda())
    Y, B = orc.gemm(TERN5, codes, scales, K, synth.bf16_bits(X), None, nthreads=NTHREADS)
    _check_products(Yg, Y, B, f"ragged N={N} M={M}")


@pytest.mark.parametrize("M", (8, 64))
def test_ternary_gemm_zero_blocks_give_exact_zero(L, M):
    """An all-zero weight block contributes exactly nothing on the tensor cores too: rows
    whose every block is zero give exactly 0, and a zero activation matrix gives 0."""
    N, K = 256, 1024
    W = synth.weights(N, K, 8500)
    W[7:13] = 0.0
    W[100, 128:256] = 0.0   # one zero block in an otherwise ordinary row
    pw = L.lbq_pack(TERN5, W.cuda())
    X = synth.activations(M, K, 8600).cuda()
    Y = L.lbq_gemm(pw, X).float().cpu()
    assert torch.all(Y[:, 7:13] == 0)
    Y0 = L.lbq_gemm(pw, torch.zeros((M, K), dtype=torch.bfloat16, device="cuda"))
    assert torch.all(Y0.float() == 0)


@pytest.mark.parametrize("mi", (0, 3))
def test_ternary_gemm_m4096_27b_sampled(L, orc, mi):
    """M = 4096 tokens through the 27B QKV (K = 5120) and down (K = 17408) products, the
    bench's largest batch; sampled weight rows checked over every token."""
    name, K, N = synth.LAYER_SHAPES[mi]
    M = 4096
    Wd = synth.weights(N, K, 9900 + mi, device="cuda")
    pw = L.lbq_pack(TERN5, Wd)
    X = synth.activations(M, K, 9950 + mi, device="cuda")
    Yg = L.lbq_gemm(pw, X)
    rows = torch.tensor([0, 1, 2, 3, 127, 128, 2049, N - 130, N - 1], device="cuda")
    codes, scales = orc.pack(TERN5, Wd[rows].cpu().numpy())
    Y, B = orc.gemm(TERN5, codes, scales, K, synth.bf16_bits(X), None, nthreads=NTHREADS)
    _check_products(Yg[:, rows], Y, B, f"27B {name}, M=4096")


# ------------------------------------------------------- mixed-format layer, one graph

def test_mixed_format_layer_graph_chained(L, orc):
    """One 27B-shaped layer with 2-bit + rotation attention (QKV, O) and ternary FFN
    (gate+up, down), captured in one CUDA graph as the bench's mixed pass runs it: every
    product chained to the previous kernel by programmatic dependent launch. Gate+up
    reads the O product's output as its input, so a product that read its x before the
    previous kernel finished would see stale values; O's input is changed between
    replays to make such a read visible. Every output is checked against the oracle."""
    fmts = (Q2RHT, Q2RHT, TERN5, TERN5)
    prods = []
    for mi, (name, K, N) in enumerate(synth.LAYER_SHAPES):
        Wd = synth.weights(N, K, synth.seed_of(40, 0, mi), device="cuda")
        pw = L.lbq_pack(fmts[mi], Wd)
        codes, scales = orc.pack(fmts[mi], Wd.cpu().numpy())
        del Wd
        x = synth.activations(1, K, synth.seed_of(50, 0, mi), device="cuda")[0].clone()
        prods.append(dict(name=name, K=K, N=N, fmt=fmts[mi], pw=pw, codes=codes, scales=scales,
                          x=x, y=torch.empty(N, dtype=torch.bfloat16, device="cuda")))
    prods[2]["x"] = prods[1]["y"]  # gate+up reads O's output
    Dg = {K: L.lbq_rht_signs(31 + K, K) for K in (synth.HIDDEN, synth.FFN)}
    Do = {K: orc.rht_signs(31 + K, K) for K in (synth.HIDDEN, synth.FFN)}
    ws = torch.zeros(max(L.lbq_workspace_bytes(p["pw"], 1) for p in prods), dtype=torch.uint8,
                     device="cuda")
    stream = torch.cuda.Stream()

    def step():
        for p in prods:
            L.lbq_gemv(p["pw"], p["x"], Dg[p["K"]] if p["fmt"] == Q2RHT else None, p["y"], ws,
                       stream=stream)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        step()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            step()
    x_o = prods[1]["x"]
    for rep in range(3):
        with torch.cuda.stream(stream):
            x_o.copy_(synth.activations(1, synth.HIDDEN, 60 + rep, device="cuda")[0])
            g.replay()
        torch.cuda.synchronize()
        for p in prods:
            Xb = synth.bf16_bits(p["x"].view(1, -1))
            Y, B = orc.gemm(p["fmt"], p["codes"], p["scales"], p["K"], Xb,
                            Do[p["K"]] if p["fmt"] == Q2RHT else None, nthreads=NTHREADS)
            _check_products(p["y"], Y[0], B[0], f"mixed {p['name']} replay {rep}")
    assert L.lbq_device_fault() == 0
