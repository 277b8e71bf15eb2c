"""Tensor-parallel layer products (tp.py): shard planning and the all-reduce, on two
gloo ranks on the CPU (the local products are the fp64 oracle's, standing in for the
library's GPU kernels), and on one GPU the library's fp32-output product on each
shard of a split, summed as the all-reduce would."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from bit_weight_only_ternary_b200 import synth, tp  # noqa: E402

TOL = 2.0 ** -8


# ---- stand-ins for the GPU calls (module level: the ranks are spawned processes)
class OraclePacked:
    def __init__(self, fmt, W):
        import oracle
        self.fmt, self.K, self.N = fmt, W.shape[1], W.shape[0]
        self.codes, self.scales = oracle.pack(fmt, W.numpy())


def oracle_pack(fmt, W):
    return OraclePacked(fmt, W)


def oracle_product(pw, x, D):
    import oracle
    Y, _ = oracle.gemm(pw.fmt, pw.codes, pw.scales, pw.K, synth.bf16_bits(x.view(1, -1)),
                       None if D is None else D.numpy())
    return torch.from_numpy(Y[0])


def oracle_gemv(pw, x, D=None):
    return oracle_product(pw, x, D).to(torch.bfloat16)


def oracle_gemv_f32(pw, x, D=None):
    return oracle_product(pw, x, D).to(torch.float32)


def _rank(rank, world, port, fmt, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        K, N = 2048, 300
        W = synth.weights(N, K, 77 + fmt)
        x = synth.activations(1, K, 78)[0]
        D = torch.from_numpy(oracle.rht_signs(5, K)) if fmt == tp.Q2RHT else None
        # column split: this rank's rows, gathered
        col = tp.make_shard(W, fmt, "column", rank, world, oracle_pack)
        y_loc = tp.column_forward(col, x, D, gemv=oracle_gemv)
        parts = [None] * world
        dist.all_gather_object(parts, (col.lo, col.hi, y_loc))
        # row split: partial products in fp32, one all-reduce
        row = tp.make_shard(W, fmt, "row", rank, world, oracle_pack)
        y_row = tp.row_forward(row, x, D, gemv_f32=oracle_gemv_f32)
        out[rank] = (parts, y_row, (row.lo, row.hi), (col.lo, col.hi))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("fmt", (tp.TERN5, tp.SIGN1, tp.Q2RHT))
def test_two_rank_split_products_match_the_whole(fmt, orc):
    world, port = 2, 29541 + fmt
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank, args=(world, port, fmt, out), nprocs=world, join=True,
                       start_method="spawn")
    K, N = 2048, 300
    W = synth.weights(N, K, 77 + fmt)
    x = synth.activations(1, K, 78)
    D = orc.rht_signs(5, K) if fmt == tp.Q2RHT else None
    codes, scales = orc.pack(fmt, W.numpy())
    Y, B = orc.gemm(fmt, codes, scales, K, synth.bf16_bits(x), D)
    # column split: the gathered rows are exactly the whole product's (row by row)
    parts = out[0][0]
    ycol = torch.cat([p[2] for p in sorted(parts, key=lambda t: t[0])]).double().numpy()
    assert [(p[0], p[1]) for p in sorted(parts, key=lambda t: t[0])] == [(0, 148), (148, 300)]
    assert np.array_equal(ycol, torch.from_numpy(Y[0]).to(torch.bfloat16).double().numpy())
    # row split: every rank holds the same sum, within the bound of the whole product
    y0, y1 = out[0][1], out[1][1]
    assert torch.equal(y0, y1)
    assert np.all(np.abs(y0.double().numpy() - Y[0]) <= TOL * B[0])
    lo, hi = out[1][2]
    assert lo % tp.block_of(fmt) == 0 and hi == K


@pytest.mark.parametrize("fmt", (tp.TERN5, tp.SIGN1, tp.Q2RHT))
def test_shards_pack_to_the_whole_matrix_bytes(fmt, orc):
    """A row shard's blocks and a column shard's rows are the same bytes as in the
    packing of the whole matrix (scales are per block, blocks never straddle a split)."""
    K, N = 3072, 40
    W = synth.weights(N, K, 99)
    codes, scales = orc.pack(fmt, W.numpy())
    bpb = {tp.TERN5: 28, tp.SIGN1: 16, tp.Q2RHT: 8}[fmt]  # code bytes per block (ternary: with scale)
    blk = {tp.TERN5: 128, tp.SIGN1: 128, tp.Q2RHT: 32}[fmt]
    for world in (2, 3):
        for rank in range(world):
            r = tp.make_shard(W, fmt, "row", rank, world, oracle_pack)
            b0, b1 = r.lo // blk, r.hi // blk
            assert np.array_equal(r.weights.codes[:, :(b1 - b0) * bpb], codes[:, b0 * bpb:b1 * bpb])
            if scales is not None:
                assert np.array_equal(r.weights.scales[:, :b1 - b0], scales[:, b0:b1])
            c = tp.make_shard(W, fmt, "column", rank, world, oracle_pack)
            assert c.lo % 4 == 0 and np.array_equal(c.weights.codes, codes[c.lo:c.hi])


def test_split_ranges_cover_everything_in_whole_granules():
    for total, g in ((5120, 128), (17408, 512), (300, 4), (34816, 4)):
        for world in (1, 2, 3, 4, 8):
            spans = [tp.split_range(total, world, r, g) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert all(lo % g == 0 for lo, _ in spans)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", (tp.TERN5, tp.SIGN1, tp.Q2RHT))
def test_gpu_row_split_partials_sum_to_the_product(orc, fmt):
    """On one GPU, the fp32 partial products of a two-way input-feature split of a 27B
    down matrix (lbq_gemv_f32 on each shard), summed as the all-reduce does and rounded
    once, meet the bound of the whole product; lbq_gemv_f32 of the whole matrix too."""
    from bit_weight_only_ternary_b200 import build
    build.build()
    from bit_weight_only_ternary_b200 import lbq
    name, K, N = synth.LAYER_SHAPES[3]
    W = synth.weights(N, K, 4321)
    x = synth.activations(1, K, 4322)
    D = lbq.lbq_rht_signs(9, K) if fmt == tp.Q2RHT else None
    Do = orc.rht_signs(9, K) if fmt == tp.Q2RHT else None
    codes, scales = orc.pack(fmt, W.numpy())
    Y, B = orc.gemm(fmt, codes, scales, K, synth.bf16_bits(x), Do, nthreads=8)
    xd = x[0].cuda()
    total = torch.zeros(N, dtype=torch.float32, device="cuda")
    for rank in range(2):
        s = tp.make_shard(W.cuda(), fmt, "row", rank, 2, lbq.lbq_pack)
        total += lbq.lbq_gemv_f32(s.weights, xd[s.lo:s.hi], None if D is None else D[s.lo:s.hi])
    y = total.to(torch.bfloat16).double().cpu().numpy()
    assert np.all(np.abs(y - Y[0]) <= TOL * B[0])
    whole = lbq.lbq_gemv_f32(lbq.lbq_pack(fmt, W.cuda()), xd, D).double().cpu().numpy()
    assert np.all(np.abs(whole - Y[0]) <= TOL * B[0])
    col = tp.make_shard(W.cuda(), fmt, "column", 1, 2, lbq.lbq_pack)
    yc = tp.column_forward(col, xd, D).double().cpu().numpy()
    assert np.all(np.abs(yc - Y[0][col.lo:col.hi]) <= TOL * B[0][col.lo:col.hi])
