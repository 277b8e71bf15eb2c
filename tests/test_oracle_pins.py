"""Pins of the oracle against things other than itself (CPU only).

Each test ties one oracle function to an independent fact: numpy's IEEE float16
rounding, torch's bf16, scipy's Sylvester Hadamard matrix, an exact (fsum)
mean, published SplitMix64 outputs, exhaustive code tables, brute-force dense
products and closed forms. A plausible slip in the oracle (a digit order, a
tie rule, a dropped scale, a transposed index, a wrong normalisation) fails at
least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from bit_weight_only_ternary_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TERN5, SIGN1, Q2RHT = 1, 2, 3


# ------------------------------------------------------------------ fp16 / bf16

def test_f16_all_patterns_decode_like_numpy(orc):
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_f16_rounding_matches_numpy(orc):
    rng = np.random.default_rng(1)
    vals = [0.0, -0.0, 65504.0, 65519.999, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25,
            2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 * (1 - 2 ** -12)]
    # exact midpoints between neighbouring fp16 values (ties -> even), both signs
    h = np.arange(0, 0x7bff, 37, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    vals += list((lo + hi) / 2) + list(-(lo + hi) / 2)
    vals += list(rng.normal(0, 1, 2000) * 10.0 ** rng.uniform(-9, 4.7, 2000))
    for v in vals:
        want = int(np.array(v, dtype=np.float64).astype(np.float16).view(np.uint16))
        assert orc.f16_from_f64(v) == want, v


def test_bf16_decode_matches_torch(orc):
    bits = np.arange(0, 65536, 7, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    got = np.array([orc.lib().orc_bf16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(got[~nan], ref[~nan]) and np.isnan(got[nan]).all()


# ------------------------------------------------------------------ layouts

def test_layout_sizes(orc):
    # bytes per 128 weights: ternary 26 codes + 2 scale, sign 16 + 2, q2 (4 x 8) + (4 x 2)
    assert orc.layout(TERN5, 5120) == (1120, 0, 128)
    assert orc.layout(TERN5, 17408) == (3808, 0, 128)
    assert orc.layout(TERN5, 128) == (32, 0, 128)  # 28 padded to 16
    assert orc.layout(SIGN1, 5120) == (640, 40, 128)
    assert orc.layout(Q2RHT, 5120) == (1280, 160, 32)
    with pytest.raises(ValueError):
        orc.layout(Q2RHT, 640)
    with pytest.raises(ValueError):
        orc.layout(TERN5, 100)


# ------------------------------------------------------------------ ternary

def _tern_weights_for(trits, s=0.25):
    """Weights s * t: every |w| is 0 or s, far from the s16/2 threshold."""
    return np.asarray(trits, dtype=np.float32) * np.float32(s)


def test_tern_golden_bytes(orc):
    rows = []
    for line in open(os.path.join(GOLDEN, "tern_bytes.txt")):
        if line.strip() and not line.startswith("#"):
            rows.append([int(v) for v in line.split()])
    for r in rows:
        t = np.zeros(128, np.int64)
        t[:5] = r[:5]
        t[5] = 1  # keep the block mean non-zero
        W = _tern_weights_for(t)[None, :]
        codes, _ = orc.pack(TERN5, W)
        assert codes[0, 0] == r[5], r


def test_tern_all_243_codes_roundtrip_and_biject(orc):
    tuples = list(itertools.product((-1, 0, 1), repeat=5))
    seen = set()
    for chunk in range(0, len(tuples), 25):
        t = np.zeros(128, np.int64)
        for j, tup in enumerate(tuples[chunk:chunk + 25]):
            t[5 * j:5 * j + 5] = tup
        t[125:128] = (1, -1, 0)
        # weights are the trits themselves: |w| in {0, 1} and 0 < s16 < 2, so |w| = 1 lies
        # above the s16/2 threshold and w/s16 rounds to +-1 (or beyond, then clipped)
        W = (t * 1.0).astype(np.float32)[None, :]
        s16 = orc.f16_to_f64(orc.f16_from_f64(np.abs(W).astype(np.float64).mean()))
        assert 0 < s16 < 2
        codes, _ = orc.pack(TERN5, W)
        back, bs = orc.unpack(TERN5, codes, None, 128)
        assert np.array_equal(back[0], t)
        assert bs[0, 0] == s16
        for j in range(min(25, len(tuples) - chunk)):
            seen.add(int(codes[0, j]))
        assert codes[0, 25] == 2 + 0 * 3 + 1 * 9 + 27 + 81
    assert seen == set(range(243))


def test_tern_scale_is_exact_absmean_rounded_once(orc):
    rng = np.random.default_rng(7)
    W = (rng.normal(0, 0.02, (16, 1024)) * rng.choice([1e-6, 1, 100], (16, 1))).astype(np.float32)
    W[3, :128] = 0.0
    codes, _ = orc.pack(TERN5, W)
    _, bs = orc.unpack(TERN5, codes, None, 1024)
    for n in range(16):
        for b in range(8):
            blk = W[n, 128 * b:128 * b + 128].astype(np.float64)
            exact = math.fsum(abs(v) for v in blk) / 128.0
            want = float(np.float16(exact))
            if bs[n, b] != want:  # only a last-bit-of-fp64 tie could explain a difference
                lo, hi = sorted([bs[n, b], want])
                assert abs(exact - (lo + hi) / 2) <= 1e-12 * exact
    assert bs[3, 0] == 0.0


def test_tern_trits_follow_round_clip_rule(orc):
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, (32, 512)).astype(np.float32)
    codes, _ = orc.pack(TERN5, W)
    t, bs = orc.unpack(TERN5, codes, None, 512)
    s = np.repeat(bs, 128, axis=1)
    want = np.clip(np.round(W.astype(np.float64) / s), -1, 1)  # numpy round: half to even
    assert np.array_equal(t, want.astype(np.int8))
    # fraction of non-zero trits for Gaussian weights: P(|w| > E|w|/2) = erfc(sqrt(2/pi)/(2 sqrt 2))
    assert abs((t != 0).mean() - math.erfc(math.sqrt(2 / math.pi) / (2 * math.sqrt(2)))) < 0.01


def test_tern_zero_block(orc):
    codes, _ = orc.pack(TERN5, np.zeros((1, 128), np.float32))
    t, bs = orc.unpack(TERN5, codes, None, 128)
    assert bs[0, 0] == 0 and not t.any() and codes[0, 0] == 121 and codes[0, 25] == 121


def test_tern_exact_tie_at_half_scale(orc):
    # w[0] = s/2 exactly (a tie, which rounds half to even -> 0); w[1] = 0.375 keeps the
    # block mean at exactly 0.25, so s16 = 0.25
    w = np.full(128, 0.25, np.float32)
    w[0] = 0.125
    w[1] = 0.375  # mean stays 0.25
    codes, _ = orc.pack(TERN5, w[None, :])
    t, bs = orc.unpack(TERN5, codes, None, 128)
    assert bs[0, 0] == 0.25
    assert t[0, 0] == 0 and t[0, 1] == 1 and t[0, 2] == 1
    w[0] = -0.125
    w[1] = 0.375
    w[2] = 0.0
    w[3] = 0.5
    codes, _ = orc.pack(TERN5, w[None, :])
    t, bs = orc.unpack(TERN5, codes, None, 128)
    assert bs[0, 0] == 0.25 and t[0, 0] == 0 and t[0, 2] == 0


def test_tern_padding_and_invalid_bytes_rejected(orc):
    W = synth.weights(2, 256, 5).numpy()
    codes, _ = orc.pack(TERN5, W)
    assert codes.shape[1] == 64 and not codes[:, 56:].any()  # 2 x 28 bytes, padded to 64
    bad = codes.copy()
    bad[0, 3] = 243
    with pytest.raises(ValueError):
        orc.unpack(TERN5, bad, None, 256)
    bad = codes.copy()
    bad[0, 25] = 0  # padding digits must be zero trits
    with pytest.raises(ValueError):
        orc.unpack(TERN5, bad, None, 256)


# ------------------------------------------------------------------ sign

def test_sign_all_256_bytes_roundtrip(orc):
    for start in range(0, 256, 16):
        bits = np.array([[(v >> i) & 1 for i in range(8)] for v in range(start, start + 16)]).ravel()
        w = np.where(bits == 1, 0.5, -0.5).astype(np.float32)
        codes, scales = orc.pack(SIGN1, w[None, :])
        assert list(codes[0]) == list(range(start, start + 16))
        t, bs = orc.unpack(SIGN1, codes, scales, 128)
        assert np.array_equal(t[0], 2 * bits - 1) and bs[0, 0] == 0.5


def test_sign_zero_is_positive_and_scale(orc):
    rng = np.random.default_rng(11)
    W = rng.normal(0, 0.02, (8, 256)).astype(np.float32)
    W[0, 0], W[0, 1] = 0.0, -0.0
    codes, scales = orc.pack(SIGN1, W)
    t, bs = orc.unpack(SIGN1, codes, scales, 256)
    assert t[0, 0] == 1 and t[0, 1] == 1
    assert np.array_equal(t[:, 2:], np.where(W[:, 2:] >= 0, 1, -1))
    for n in range(8):
        for b in range(2):
            exact = math.fsum(abs(float(v)) for v in W[n, 128 * b:128 * b + 128]) / 128
            assert bs[n, b] == float(np.float16(exact))


# ------------------------------------------------------------------ 2-bit

def test_q2_all_256_bytes_roundtrip(orc):
    levels = np.array([-1.5, -0.5, 0.5, 1.5])
    vals, rows = list(range(256)), []
    while vals:
        row = []
        for _ in range(16):  # 16 blocks of 8 bytes per 512-weight row
            chunk, vals = vals[:7], vals[7:]
            row += chunk + [0x55] * (7 - len(chunk)) + [0xFF]  # 0xFF: four 1.5s, so s = 1
        rows.append(row)
    want = np.array(rows, dtype=np.uint8)
    q = ((want[..., None] >> (2 * np.arange(4))) & 3).reshape(len(rows), 512)
    W = levels[q].astype(np.float32)
    codes, scales = orc.pack(Q2RHT, W)
    assert np.array_equal(codes, want)
    assert (scales == 0x3C00).all()  # fp16 1.0
    got_q, bs = orc.unpack(Q2RHT, codes, scales, 512)
    assert np.array_equal(got_q, q) and (bs == 1.0).all()


def test_q2_scale_and_nearest_level_ties_up(orc):
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.02, (16, 512)).astype(np.float32)
    codes, scales = orc.pack(Q2RHT, W)
    q, bs = orc.unpack(Q2RHT, codes, scales, 512)
    mx = np.abs(W.astype(np.float64)).reshape(16, 16, 32).max(-1)
    assert np.array_equal(bs, (mx / 1.5).astype(np.float16).astype(np.float64))
    s = np.repeat(bs, 32, axis=1)
    lv = (q - 1.5) * s
    # nearest of the four levels (distance check against all levels)
    d = np.abs(W[..., None] - np.stack([(i - 1.5) * s for i in range(4)], -1))
    assert np.all(np.abs(W - lv) <= d.min(-1) + 0)
    # ties: w = -s, 0, +s go to the upper level
    w = np.zeros(32, np.float32)
    w[0] = 1.5  # s = 1
    w[1], w[2], w[3], w[4] = -1.0, 0.0, 1.0, -1.5
    w[5] = np.nextafter(np.float32(-1.0), np.float32(-2))
    codes, scales = orc.pack(Q2RHT, np.tile(w, 16)[None, :])
    q, bs = orc.unpack(Q2RHT, codes, scales, 512)
    assert bs[0, 0] == 1.0
    assert list(q[0, :6]) == [3, 1, 2, 3, 0, 0]
    codes, scales = orc.pack(Q2RHT, np.zeros((1, 512), np.float32))
    q, bs = orc.unpack(Q2RHT, codes, scales, 512)
    assert not bs.any() and (q == 2).all()


# ------------------------------------------------------------------ rotation

def test_splitmix64_published_outputs(orc):
    want = [int(l, 16) for l in open(os.path.join(GOLDEN, "splitmix64_seed0.txt"))
            if l.strip() and not l.startswith("#")]
    assert [int(v) for v in orc.splitmix64(0, 3)] == want
    D = orc.rht_signs(0, 3)
    assert list(D) == [-1 if (v >> 63) else 1 for v in want]


def test_rht_signs_balanced_and_seeded(orc):
    D = orc.rht_signs(1234, 1 << 16)
    assert set(np.unique(D)) == {-1, 1}
    assert abs(D.astype(np.float64).mean()) < 4 / math.sqrt(1 << 16)  # 4 sigma
    assert not np.array_equal(D[:4096], orc.rht_signs(1235, 4096))
    assert np.array_equal(D[:100], orc.rht_signs(1234, 100))


def test_hadamard_matrix_is_sylvester(orc):
    eye = np.eye(512)
    cols = orc.hadamard(eye, np.ones(512, np.int8))  # row j of the output = H e_j / sqrt 512
    Hs = scipy.linalg.hadamard(512).astype(np.float64)
    assert np.allclose(cols.T * math.sqrt(512), Hs, rtol=0, atol=1e-12)
    Hi = np.rint(cols * math.sqrt(512)).astype(np.int64)
    assert np.array_equal(Hi @ Hi.T, 512 * np.eye(512, dtype=np.int64))


def test_hadamard_properties(orc):
    rng = np.random.default_rng(9)
    x = rng.normal(0, 1, (3, 1536))
    D = orc.rht_signs(77, 1536)
    y = orc.hadamard(x, D)
    # orthonormal per 512-block: Parseval
    for c in range(3):
        assert np.allclose(np.linalg.norm(y[:, 512 * c:512 * c + 512], axis=1),
                           np.linalg.norm(x[:, 512 * c:512 * c + 512], axis=1), rtol=1e-12)
    # D acts first: H D x = H (D x)
    assert np.allclose(y, orc.hadamard(x * D, np.ones(1536, np.int8)), rtol=0, atol=1e-12)
    # involution of the unsigned transform
    ones = np.ones(1536, np.int8)
    assert np.allclose(orc.hadamard(orc.hadamard(x, ones), ones), x, atol=1e-12)
    # against scipy's matrix, block by block
    Hs = scipy.linalg.hadamard(512) / math.sqrt(512)
    for c in range(3):
        want = (Hs @ (D[512 * c:512 * c + 512] * x[:, 512 * c:512 * c + 512]).T).T
        assert np.allclose(y[:, 512 * c:512 * c + 512], want, atol=1e-12)


# ------------------------------------------------------------------ products

def _bits(x):
    return synth.bf16_bits(x)


@pytest.mark.parametrize("fmt", [TERN5, SIGN1, Q2RHT])
def test_gemm_matches_dense_brute_force(orc, fmt):
    K, N, M = 1024, 6, 3
    W = synth.weights(N, K, 21).numpy()
    X = synth.activations(M, K, 22)
    codes, scales = orc.pack(fmt, W)
    D = orc.rht_signs(5, K) if fmt == Q2RHT else None
    Y, B = orc.gemm(fmt, codes, scales, K, _bits(X), D)
    What = orc.dequant(fmt, codes, scales, K)
    xin = X.double().numpy()
    if fmt == Q2RHT:  # rotate with scipy's matrix, not the oracle's transform
        Hs = scipy.linalg.hadamard(512) / math.sqrt(512)
        xin = np.concatenate([(Hs @ (D[512 * c:512 * c + 512] * xin[:, 512 * c:512 * c + 512]).T).T
                              for c in range(K // 512)], axis=1)
    assert np.allclose(Y, xin @ What.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(B, np.abs(xin[:, None, :] * What[None, :, :]).sum(-1), rtol=1e-12)
    # the dequantised weights are scale x code with the documented code meaning
    t, bs = orc.unpack(fmt, codes, scales, K)
    blk = 32 if fmt == Q2RHT else 128
    lvl = (t - 1.5) if fmt == Q2RHT else t
    assert np.array_equal(What, np.repeat(bs, blk, axis=1) * lvl)


@pytest.mark.parametrize("fmt", [TERN5, SIGN1, Q2RHT])
def test_gemm_closed_forms(orc, fmt):
    K, N = 512, 5
    W = synth.weights(N, K, 31).numpy()
    codes, scales = orc.pack(fmt, W)
    t, bs = orc.unpack(fmt, codes, scales, K)
    ones = np.full((1, K), 0x3F80, np.uint16)  # bf16 1.0
    if fmt == Q2RHT:
        # x' = H D x / sqrt 512 with x = D * e_0 * sqrt(512) is the all-ones vector: rotate back
        # is not bf16-exact, so use x = e_j instead: x' = D_j H[:, j] / sqrt 512
        D = orc.rht_signs(3, K)
        j = 7
        x = np.zeros((1, K), np.uint16)
        x[0, j] = 0x3F80
        Y, _ = orc.gemm(fmt, codes, scales, K, x, D)
        h = scipy.linalg.hadamard(512)[:, j] * D[j] / math.sqrt(512)
        xr = np.zeros(K)
        xr[:512] = h
        What = np.repeat(bs, 32, axis=1) * (t - 1.5)
        assert np.allclose(Y[0], What @ xr, rtol=1e-12, atol=1e-15)
        return
    Y, B = orc.gemm(fmt, codes, scales, K, ones)
    # x = 1: y_n = sum_b s_b * sum_{k in b} code_k   (spec closed form)
    want = (bs * t.reshape(N, K // 128, 128).sum(-1)).sum(-1)
    assert np.allclose(Y[0], want, rtol=1e-13)
    if fmt == SIGN1:
        pop = np.unpackbits(codes.reshape(N, K // 128, 16), axis=-1, bitorder="little").sum(-1).astype(np.int64)
        assert np.allclose(Y[0], (bs * (2 * pop - 128)).sum(-1), rtol=1e-13)
    # x = e_k: column k of W_hat
    k = 300
    x = np.zeros((1, K), np.uint16)
    x[0, k] = 0x3F80
    Y, _ = orc.gemm(fmt, codes, scales, K, x)
    assert np.array_equal(Y[0], bs[:, k // 128] * t[:, k])


def test_gemm_threads_do_not_change_results(orc):
    K, N = 512, 37
    W = synth.weights(N, K, 41).numpy()
    X = synth.activations(2, K, 42)
    codes, _ = orc.pack(TERN5, W)
    Y1, B1 = orc.gemm(TERN5, codes, None, K, _bits(X), nthreads=1)
    Y4, B4 = orc.gemm(TERN5, codes, None, K, _bits(X), nthreads=4)
    assert np.array_equal(Y1, Y4) and np.array_equal(B1, B4)


# ------------------------------------------------------------------ device row order

def _read_group4_golden():
    blocks, cur = {}, None
    for line in open(os.path.join(GOLDEN, "group4_example.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith(("codes", "scales")):
            cur = blocks.setdefault(line, [])
            continue
        cur.extend(int(v) for v in line.split())
    return blocks


def test_group4_worked_example(orc):
    gold = _read_group4_golden()
    codes = np.arange(80, dtype=np.uint8).reshape(5, 16)
    g = orc.group4(codes)
    assert g.shape == (2, 64)
    assert g[0].tolist() == gold["codes group 0"]
    assert g[1].tolist() == gold["codes group 1"]
    sc = (np.arange(3)[:, None] * 10 + np.arange(2)[None, :] + 1).astype(np.uint16)
    assert orc.group4(sc)[0].tolist() == gold["scales group 0"]


@pytest.mark.parametrize("N", [1, 3, 4, 9])
def test_group4_is_a_padded_permutation(orc, N):
    rng = np.random.default_rng(N)
    codes = rng.integers(0, 243, size=(N, 32), dtype=np.uint8)
    g = orc.group4(codes)
    assert g.shape == ((N + 3) // 4, 128)
    # same multiset of bytes plus the zero padding rows, and exactly invertible
    assert np.array_equal(np.sort(g.ravel()),
                          np.sort(np.concatenate([codes.ravel(),
                                                  np.zeros(g.size - codes.size, np.uint8)])))
    assert np.array_equal(orc.ungroup4(g, N), codes)
    sc = rng.integers(0, 1 << 16, size=(N, 5), dtype=np.uint16)
    assert np.array_equal(orc.ungroup4(orc.group4(sc), N), sc)
