"""Host logic of the multi-GPU bench (replicas only): two gloo ranks on the CPU.

Every rank runs its own replica; the job's time is the slowest rank's, taken with one
all-reduce that every rank joins, and the job's rate counts the units of all ranks.
"""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _rank(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(local_ms[rank], world, dist, torch.device("cpu"), torch)
        out[rank] = ms
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, 29517
    local_ms = [3.25, 7.5]
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank, args=(world, port, local_ms, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1] == max(local_ms)


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(4.0, 1, None, None, None) == 4.0


def test_job_rate_counts_every_rank():
    # 2 ranks x 4.6e9 bytes in 2.5 ms of the slowest rank
    assert bench.job_rate(2, 4.6e9, 2.5) == pytest.approx(2 * 4.6e9 / 2.5e-3)
    assert bench.job_rate(1, 1, 1000.0) == pytest.approx(1.0)


def test_kernel_key_ignores_comments_but_not_code():
    src = 'int a = 1;  // one\n// a comment line\n\nconst char* s = "x // y";\n'
    assert bench._code_only(src) == 'int a = 1;\nconst char* s = "x // y";'
    assert bench._code_only(src) != bench._code_only(src.replace("a = 1", "a = 2"))


def test_mixed_workload_formats():
    # QKV and O in the 2-bit + rotation format, gate+up and down ternary
    assert [bench.product_fmt(0, mi) for mi in range(4)] == [3, 3, 1, 1]
    assert [bench.product_fmt(2, mi) for mi in range(4)] == [2, 2, 2, 2]
