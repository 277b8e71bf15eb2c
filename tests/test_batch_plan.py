"""The batched product's schedule, checked on the host (no GPU): lbq_gemv_batch_plan
returns the K-pieces of every product and the CTAs' ranges of unit-slices that one
launch of lbq_gemv_batch uses. The plan reads no device memory, so the records carry
made-up (aligned, disjoint) device addresses.

Checked: the total; the pieces rule the header states; the ranges start at 0, end at
the total, never decrease and only cut at the first unit-slice of a unit; every CTA's
load (its unit-slices plus the table builds its units need, counted as the kernel
walks them) stays close to the average; and the argument errors.
"""
import ctypes
import math
import random

import pytest

TERN5, SIGN1, Q2RHT = 1, 2, 3
LAYER = [(5120, 7168), (5120, 5120), (5120, 34816), (17408, 5120)]  # (K, N)
ACC_UNITS = 1008   # units a CTA keeps running sums for at once (one chunk)
BUILD_COST = 48    # unit-slices the cut charges per table build


@pytest.fixture(scope="module")
def L():
    from bit_weight_only_ternary_b200 import build
    build.build()
    from bit_weight_only_ternary_b200 import lbq
    return lbq


def records(L, cases):
    """lbq_product records for (fmt, K, N) cases, with made-up device addresses."""
    arr = (L.lbq_product * len(cases))()
    for i, (fmt, K, N) in enumerate(cases):
        cs, ss = ctypes.c_int64(), ctypes.c_int64()
        cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
        assert L._lib.lbq_packed_layout(fmt, K, N, ctypes.byref(cs), ctypes.byref(ss),
                                        ctypes.byref(cb), ctypes.byref(sb)) == 0
        base = (1 << 44) + i * (1 << 36)
        scales = None if fmt == TERN5 else base + (1 << 35)
        arr[i].w = L.lbq_weights(fmt, 0, K, N, base, scales, cs.value, ss.value)
        arr[i].x = (1 << 45) + i * (1 << 32)
        arr[i].y = (1 << 46) + i * (1 << 32)
        arr[i].D = (1 << 47) + i * (1 << 32) if fmt == Q2RHT else None
    return arr


def slices(fmt, K):
    return -(-K // (1024 if fmt == SIGN1 else 512))


def loads(cases, pieces, bound):
    """Each CTA's unit-slices and table builds: unit u of piece s goes to the CTA whose
    range holds its first unit-slice; a CTA builds one table per slice of the piece for
    every chunk of ACC_UNITS of its units of that piece."""
    ctas = len(bound) - 1
    work = [0] * ctas
    builds = [0] * ctas
    starts = set()
    c0 = 0
    for (fmt, K, N), S in zip(cases, pieces):
        KS, NU = slices(fmt, K), -(-N // 16)
        for s in range(S):
            j0, j1 = KS * s // S, KS * (s + 1) // S
            base, ln = c0 + NU * j0, j1 - j0
            per_cta = {}
            for u in range(NU):
                pos = base + u * ln
                starts.add(pos)
                c = max(i for i in range(ctas) if bound[i] <= pos) if ctas < 8 else None
                if c is None:  # binary search over the boundaries
                    lo, hi = 0, ctas - 1
                    while lo < hi:
                        mid = (lo + hi + 1) // 2
                        if bound[mid] <= pos:
                            lo = mid
                        else:
                            hi = mid - 1
                    c = lo
                assert bound[c] <= pos < bound[c + 1]
                work[c] += ln
                per_cta[c] = per_cta.get(c, 0) + 1
            for c, n_units in per_cta.items():
                builds[c] += math.ceil(n_units / ACC_UNITS) * ln
        c0 += KS * NU
    return work, builds, starts, c0


def check_plan(L, cases, ctas=148):
    arr = records(L, cases)
    pieces, bound, total = L.lbq_gemv_batch_plan(arr, len(cases), ctas)
    W = sum(slices(f, K) * -(-N // 16) for f, K, N in cases)
    assert total == W
    for (fmt, K, N), S in zip(cases, pieces):
        KS = slices(fmt, K)
        assert S == max(1, min(KS, -(-64 * ctas * KS // W))), (fmt, K, N, S)
    assert bound[0] == 0 and bound[-1] == W
    assert all(a <= b for a, b in zip(bound, bound[1:]))
    work, builds, starts, _ = loads(cases, pieces, bound)
    assert sum(work) == W
    for b in bound[1:-1]:
        assert b == W or b in starts, f"a range starts inside a unit ({b})"
    cost = [w + BUILD_COST * b for w, b in zip(work, builds)]
    busy = [c for c in cost if c > 0]
    max_len = max(slices(f, K) for f, K, _ in cases)
    # the cut is a greedy fill to the smallest feasible target: no CTA carries more than
    # the average plus one unit's charge (its slices and their table builds)
    assert max(cost) <= sum(cost) / len(busy) + (BUILD_COST + 1) * max_len * 2, (max(cost), sum(cost) / len(busy))
    return pieces, bound, cost


@pytest.mark.parametrize("fmt", [TERN5, SIGN1, Q2RHT])
def test_plan_of_a_27b_layer_and_of_a_64_layer_pass(L, fmt):
    pieces, _, _ = check_plan(L, [(fmt, K, N) for K, N in LAYER])
    assert max(pieces) > 1  # one layer is too short in rows for whole-K rows per CTA
    pieces, _, cost = check_plan(L, [(fmt, K, N) for _ in range(64) for K, N in LAYER])
    assert pieces == [1] * 256  # a 64-layer pass splits nothing
    assert max(cost) <= 1.01 * sum(cost) / len(cost)


def test_plan_corner_lists(L):
    check_plan(L, [(TERN5, 128, 1)])                       # one unit: 147 CTAs without work
    p, _, _ = check_plan(L, [(TERN5, 65536, 16)])          # one unit of 128 slices
    assert p == [128]
    check_plan(L, [(SIGN1, 131072, 5), (SIGN1, 1152, 1000)])
    check_plan(L, [(Q2RHT, 512, 1), (Q2RHT, 1024, 4100), (Q2RHT, 49152, 2)])
    check_plan(L, [(TERN5, 512, 2400256)])                 # more than one chunk per CTA
    check_plan(L, [(TERN5, 5120, 7168)], ctas=1)
    check_plan(L, [(TERN5, 5120, 7168)], ctas=L.LBQ_BATCH_MAX_CTAS)


def test_plan_random_lists(L):
    rng = random.Random(11)
    for _ in range(25):
        fmt = rng.choice([TERN5, SIGN1, Q2RHT])
        cases = []
        for _ in range(rng.randint(1, 24)):
            K = 512 * rng.randint(1, 12) if fmt == Q2RHT else 128 * rng.randint(1, 40)
            cases.append((fmt, K, rng.randint(1, 6000)))
        check_plan(L, cases, ctas=rng.choice([1, 7, 148, 192]))


def test_plan_rejects_bad_arguments(L):
    arr = records(L, [(TERN5, 512, 64), (SIGN1, 512, 64)])
    with pytest.raises(L.LbqError) as e:
        L.lbq_gemv_batch_plan(arr, 2, 148)             # two formats: two launches
    assert e.value.status == L.LBQ_ERR_ARG
    one = records(L, [(TERN5, 512, 64)])
    for ctas in (0, L.LBQ_BATCH_MAX_CTAS + 1):
        with pytest.raises(L.LbqError) as e:
            L.lbq_gemv_batch_plan(one, 1, ctas)
        assert e.value.status == L.LBQ_ERR_ARG
    pieces = (ctypes.c_int32 * 1)()
    total = ctypes.c_int64()
    assert L._lib.lbq_gemv_batch_plan(one, 1, 148, pieces, None, ctypes.byref(total)) == L.LBQ_ERR_ARG


def test_bench_counts_the_launches_the_library_makes(L):
    """bench.py claims its kernel launches from the library's split rule; that rule must
    agree with the plan (a launch adds the piece-sum kernel when any product splits)."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    rng = random.Random(5)
    lists = [[(TERN5, K, N) for K, N in LAYER], [(TERN5, K, N) for _ in range(64) for K, N in LAYER],
             [(SIGN1, 131072, 5)], [(Q2RHT, 1024, 4100)]]
    for _ in range(10):
        fmt = rng.choice([TERN5, SIGN1, Q2RHT])
        lists.append([(fmt, 512 * rng.randint(1, 12) if fmt == Q2RHT else 128 * rng.randint(1, 40),
                       rng.randint(1, 6000)) for _ in range(rng.randint(1, 30))])
    for cases in lists:
        for i in range(0, len(cases), L.LBQ_BATCH_MAX):
            chunk = cases[i:i + L.LBQ_BATCH_MAX]
            pieces, _, _ = L.lbq_gemv_batch_plan(records(L, chunk), len(chunk), 148)
            prods = [dict(fmt=f, K=K, N=N) for f, K, N in chunk]
            assert bench.launches_per_step(L, prods, "batch") == 1 + int(max(pieces) > 1)
