#!/usr/bin/env python3
"""Throughput of the low-bit weight GEMV on synthetic 27B-decoder-shaped layers.

One step = one batch-1 pass over all 64 layers x 4 products (QKV 5120->7168,
O 5120->5120, gate+up 5120->34816, down 17408->5120), i.e. one "token" of the
weight stream, every product a call of the C ABI (lbq_gemv). The default
workload is the ternary format; --workload selects the 1-bit or 2-bit+rotation
formats or the batched products (lbq_gemm with M activation rows).

Prints ONE JSON line (rank 0). `value` is packed-weight GB/s of the whole job with
all inputs resident in HBM (4.6 GB of ternary weights per step, far above the
126 MB L2, so no flush is needed); `e2e` repeats the measurement with each step's
activations copied in from pinned host memory and its outputs copied back.
Multi-GPU (torchrun): every rank runs an independent replica on its own weights
("replicas only": the path has no exchange step), the time is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload tern|sign|q2|gemm8|...]
    python bench.py --impl reference   # the fp64 CPU oracle on a bounded sample
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (format, M); format 0: a mixed-format layer (see product_fmt)
    "tern": (1, 1), "sign": (2, 1), "q2": (3, 1), "mixed": (0, 1),
    "gemm8": (1, 8), "gemm32": (1, 32), "gemm512": (1, 512), "gemm4096": (1, 4096),
}
FMT_NAME = {1: "ternary 5 trits/byte + fp16 scale per 128", 2: "1-bit sign + fp16 scale per 128",
            3: "2-bit 4-level + fp16 scale per 32, input rotated by 512-point RHT",
            0: "mixed: attention (QKV, O) 2-bit + RHT, FFN (gate+up, down) ternary"}


def product_fmt(fmt, mi):
    """The format of product mi (0 QKV, 1 O, 2 gate+up, 3 down) of a layer."""
    if fmt != 0:
        return fmt
    return 3 if mi < 2 else 1  # the mixed layer: 2-bit attention, ternary FFN
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
# dram bytes per launch of the dominant kernel from one ncu capture (one 27B layer, the
# four products, averaged per launch), keyed by the hash of the kernel source it was
# taken on; reported as null once that source changes.
NCU_TRAFFIC = {
    # profiles/gemv_tern_1layer_full.md: 72.42 MB read + 256 B written over the 4 launches
    ("tern", "6a683c1dec9b0cc5"): 18.104e6,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="tern")
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--cpu-sample-s", type=float, default=12.0,
                    help="target seconds of oracle work for the CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-parity", action="store_true")
    return ap.parse_args()


# ------------------------------------------------------------------------------ helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained",
                                                                          d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


GEMV_SOURCES = ("gemv.cu", "rht.cuh", "sm100_async.cuh", "lbq_common.cuh")
GEMM_SOURCES = ("gemm.cu", "gemm_tc.cu", "sm100_async.cuh", "lbq_common.cuh")


def _code_only(text):
    """The source without // comments and blank lines (comment edits keep the key)."""
    out = []
    for line in text.splitlines():
        i = line.find("//")
        while i >= 0 and line[:i].count('"') % 2 == 1:  # inside a string literal
            i = line.find("//", i + 2)
        code = (line if i < 0 else line[:i]).rstrip()
        if code:
            out.append(code)
    return "\n".join(out)


def kernel_source_hash(files=GEMV_SOURCES):
    """Hash of the kernel sources a workload runs, comments aside (keys the recorded
    ncu traffic: a figure stands only for the code it was measured on)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_weight_only_ternary_b200", "csrc")
    for f in files:
        p = os.path.join(csrc, f)
        if os.path.exists(p):
            h.update(_code_only(open(p).read()).encode())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of SM clock and throttle reasons."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.lines = index, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------ the model

def build_layers(L, synth, fmt, M, n_layers, seed, device, torch):
    """Packs n_layers x 4 seeded matrices on the device; returns per-product records."""
    prods = []
    for layer in range(n_layers):
        for mi, (name, K, N) in enumerate(synth.LAYER_SHAPES):
            W = synth.weights(N, K, synth.seed_of(seed * 1000, layer, mi), device=device)
            pw = L.lbq_pack(product_fmt(fmt, mi), W)
            del W
            X = synth.activations(M, K, synth.seed_of(seed * 1000 + 500, layer, mi), device=device)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            prods.append({"layer": layer, "mi": mi, "name": name, "K": K, "N": N, "pw": pw,
                          "X": X, "Y": Y, "fmt": product_fmt(fmt, mi)})
    return prods


def max_over_ranks(ms, world, dist, device, torch):
    """The slowest rank's time: every rank takes part (same collective on all ranks)."""
    if world <= 1:
        return ms
    tt = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_rate(world, units_per_rank, ms_step):
    """Whole-job rate: the units all ranks processed per second of the slowest rank."""
    return world * units_per_rank / (ms_step * 1e-3)


def run_step(L, prods, D, ws, M):
    for p in prods:
        Dp = D.get(p["K"]) if p["fmt"] == 3 else None
        if M == 1:
            L.lbq_gemv(p["pw"], p["X"][0], Dp, p["Y"][0], ws)
        else:
            L.lbq_gemm(p["pw"], p["X"], Dp, p["Y"], ws)


def ours(args):
    import torch
    import torch.distributed as dist

    from bit_weight_only_ternary_b200 import lbq as L
    from bit_weight_only_ternary_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    assert world == args.gpus or (world == 1 and args.gpus == 1), "--gpus must match WORLD_SIZE"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    fmt, M = WORKLOADS[args.workload]
    prods = build_layers(L, synth, fmt, M, args.layers, args.seed + 7919 * rank, dev, torch)
    D = {}
    if any(p["fmt"] == L.LBQ_Q2RHT for p in prods):
        for K in (synth.HIDDEN, synth.FFN):
            D[K] = L.lbq_rht_signs(args.seed * 31 + K, K, dev)
    ws_bytes = max(L.lbq_workspace_bytes(p["pw"], M) for p in prods)
    ws = torch.zeros(max(16, ws_bytes), dtype=torch.uint8, device=dev)
    weight_bytes = sum(p["pw"].nbytes for p in prods)
    act_bytes = sum(p["X"].numel() * 2 for p in prods)
    out_bytes = sum(p["Y"].numel() * 2 for p in prods)
    algo_bytes = weight_bytes + act_bytes + out_bytes
    flops = sum(2 * M * p["K"] * p["N"] for p in prods)
    torch.cuda.synchronize()

    # one CUDA graph per step: every product, stream-ordered
    stream = torch.cuda.Stream(device=dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        run_step(L, prods, D, ws, M)  # eager warm-up (and first-touch) on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            run_step(L, prods, D, ws, M)
    # kernels per product: the GEMV, plus the split-K sum when K spans several slices
    launches = (sum(1 + (p["K"] > (1024 if p["fmt"] == L.LBQ_SIGN1 else 512)) for p in prods)
                if M == 1 else len(prods))
    with torch.cuda.stream(stream):  # replays run on the stream the events are recorded on
        for _ in range(args.warmup):
            graph.replay()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- timed region: K replays, inputs resident in HBM
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        with torch.cuda.stream(stream):
            t0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            t1.record(stream)
        barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dist, dev, torch)
    ms_step = ms / args.steps
    gbs = job_rate(world, weight_bytes, ms_step) / 1e9
    tok_s = job_rate(world, M, ms_step)

    # ---- per-launch durations of the GEMV kernel (events between launches, queued ahead)
    per_launch_ms = []
    with torch.cuda.stream(stream):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(prods) + 1)]
        torch.cuda._sleep(50_000_000)  # hold the stream while the host queues every launch
        for i, p in enumerate(prods):
            evs[i].record(stream)
            run_step(L, [p], D, ws, M)
        evs[-1].record(stream)
    torch.cuda.synchronize()
    per_launch_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(len(prods))]
    iso_ms = sum(per_launch_ms)
    # The product's launch duration inside the timed region: the timed step (one graph
    # of every product, stream-ordered, each product's kernels chained by programmatic
    # dependent launch) divided by the products in it. The isolated figure (events
    # between launches, which breaks that chaining) is reported beside it.
    kern_ms = ms_step
    hbm_peak, tc_peak, tc_sust, peak_src = peaks()
    achieved = algo_bytes / (kern_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4), "peak_source": peak_src,
            "kernel": "lbq_gemv (%s)" % args.workload,
            "algorithmic_bytes_per_launch": algo_bytes / len(prods),
            "avg_launch_us": round(1e3 * kern_ms / len(prods), 3),
            "isolated_launch_us": round(1e3 * iso_ms / len(prods), 3)}
    key = kernel_source_hash(GEMV_SOURCES if M == 1 else GEMM_SOURCES)
    tr = NCU_TRAFFIC.get((args.workload, key))
    roof["traffic"] = tr
    if M >= 512:
        tf = flops / (kern_ms * 1e-3) / 1e12
        # frac against the burst peak; a pass of many products runs under the power cap,
        # so the sustained peak is given beside it
        roof.update({"bound": "tensor", "achieved": round(tf, 1), "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": round(tf / tc_peak, 4), "peak_sustained": tc_sust,
                     "frac_of_sustained": round(tf / tc_sust, 4)})

    # ---- end to end: activations in from pinned host memory, outputs back, every step
    xin_host = torch.cat([p["X"].reshape(-1) for p in prods]).cpu().pin_memory()
    xin_dev = torch.empty_like(xin_host, device=dev)
    y_host = torch.empty(sum(p["Y"].numel() for p in prods), dtype=torch.bfloat16).pin_memory()
    y_dev = torch.empty_like(y_host, device=dev)
    views_x, views_y, ox, oy = [], [], 0, 0
    for p in prods:
        views_x.append(xin_dev[ox:ox + p["X"].numel()].view(p["X"].shape))
        views_y.append(y_dev[oy:oy + p["Y"].numel()].view(p["Y"].shape))
        ox += p["X"].numel()
        oy += p["Y"].numel()
    e2e_prods = [dict(p, X=vx, Y=vy) for p, vx, vy in zip(prods, views_x, views_y)]
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g2, stream=stream):
            xin_dev.copy_(xin_host, non_blocking=True)
            run_step(L, e2e_prods, D, ws, M)
            y_host.copy_(y_dev, non_blocking=True)
    e_steps = max(10, args.steps // 4)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g2.replay()
    barrier()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(e_steps):
            g2.replay()
        t1.record(stream)
    barrier()
    ems = max_over_ranks(t0.elapsed_time(t1), world, dist, dev, torch)
    e_step = ems / e_steps
    e2e = {"value": round(job_rate(world, weight_bytes, e_step) / 1e9, 1), "unit": "GB/s",
           "tok_s_equiv": round(job_rate(world, M, e_step), 2),
           "h2d_bytes_per_step": xin_host.numel() * 2, "d2h_bytes_per_step": y_host.numel() * 2}

    # ---- sampled parity of the timed configuration against the oracle (rank 0)
    parity = None
    if rank == 0 and not args.no_parity:
        parity = sampled_parity(L, synth, prods, M, D, ws, args, dev, torch)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, fmt, M)

    if world > 1:
        del graph, g2
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    clocks = clk.summary()
    line = {
        "metric": "packed-weight HBM GB/s (% of peak) & tok/s-equiv, batch-1 27B-shape GEMV",
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        # the arithmetic: fp32 lookups and sums, or fp16 tensor-core MMAs into fp32
        "dtype": "f32" if M <= 3 or fmt != 1 else "f16 (f32 accumulate)",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) bf16 activations)",
        "tok_s_equiv": round(tok_s, 2), "pct_of_hbm_peak": round(100 * gbs / world / hbm_peak, 2),
        "config": {"workload": f"{args.layers} x 27B-shaped decoder layers (QKV 5120x7168, "
                               f"O 5120x5120, gate+up 5120x34816, down 17408x5120), "
                               f"{FMT_NAME[fmt]}, M={M}",
                   "format": args.workload, "M": M, "layers": args.layers,
                   "weight_bytes_per_step": weight_bytes, "launches_per_step": len(prods),
                   "l2": "inputs larger than L2 (no flush): %.2f GB of weights per step"
                         % (weight_bytes / 1e9),
                   "parallelism": f"replicas x{world}", "graph": "one CUDA graph per step"},
        "roofline": roof, "e2e": e2e, "gpu_launches": args.steps * launches,
        "clocks": clocks, "parity": parity, "cpu_baseline": cpu, "kernel_source": key,
    }
    if M > 1:
        line["tflops"] = round(world * flops / (ms_step * 1e-3) / 1e12, 2)
    print(json.dumps(line), flush=True)


def sampled_parity(L, synth, prods, M, D, ws, args, dev, torch):
    """Re-draws a few timed matrices' weights, checks sampled output rows with the oracle."""
    import numpy as np

    import oracle
    worst, checked = 0.0, 0
    picks = [prods[0], prods[1], prods[2], prods[-1]]
    rng = np.random.default_rng(0)
    for p in picks:
        fmt = p["fmt"]
        run_step(L, [p], D, ws, M)
        torch.cuda.synchronize()
        W = synth.weights(p["N"], p["K"], synth.seed_of(args.seed * 1000, p["layer"], p["mi"]),
                          device=dev)
        # whole groups of four rows (the library's storage order), 12 of them
        groups = np.sort(rng.choice(p["N"] // 4, size=min(12, p["N"] // 4), replace=False))
        rows = (4 * groups[:, None] + np.arange(4)[None, :]).ravel()
        Wr = W[torch.from_numpy(rows).to(dev)].cpu().numpy()
        del W
        codes, scales = oracle.pack(fmt, Wr)
        got_codes = p["pw"].codes[torch.from_numpy(groups).to(dev)].cpu().numpy()
        assert np.array_equal(oracle.group4(codes), got_codes), \
            "timed weights differ from the oracle's packing"
        Xs = p["X"][: min(M, 8)]
        Do = oracle.rht_signs(args.seed * 31 + p["K"], p["K"]) if fmt == 3 else None
        Y, B = oracle.gemm(fmt, codes, scales, p["K"], synth.bf16_bits(Xs), Do,
                           nthreads=os.cpu_count() or 1)
        yg = p["Y"][: Xs.shape[0]][:, torch.from_numpy(rows).to(dev)].float().cpu().double().numpy()
        ratio = np.abs(yg - Y) / np.maximum(2.0 ** -8 * B, 1e-300)
        assert np.all(ratio <= 1.0), f"{p['name']}: outputs outside 2^-8 sum|w x|"
        worst = max(worst, float(ratio.max()))
        checked += ratio.size
    return {"outputs_checked": checked, "max_err_over_bound": round(worst, 4), "codes_bit_exact": True}


def cpu_baseline(args, fmt, M, budget_s=None):
    """The oracle (fp64 C, all host cores) on a bounded sample of the same workload."""
    import numpy as np

    import oracle
    from bit_weight_only_ternary_b200 import synth
    budget_s = budget_s or args.cpu_sample_s
    threads = os.cpu_count() or 1
    # sample: the same fraction of rows of each of the four products of one layer
    total_w = sum(K * N for _, K, N in synth.LAYER_SHAPES)
    packed = []
    for mi, (name, K, N) in enumerate(synth.LAYER_SHAPES):
        n = max(threads, int(N * 0.02))
        W = synth.weights(n, K, 777 + mi).numpy()
        f = product_fmt(fmt, mi)
        codes, scales = oracle.pack(f, W)
        X = synth.bf16_bits(synth.activations(min(M, 8), K, 888 + mi))
        D = oracle.rht_signs(5, K) if f == 3 else None
        packed.append((f, K, n, codes, scales, X, D))
    # time one pass over the sample, then repeat to fill the budget
    reps, elapsed = 0, 0.0
    t0 = time.perf_counter()
    while elapsed < budget_s or reps == 0:
        for f, K, n, codes, scales, X, D in packed:
            oracle.gemm(f, codes, scales, K, X, D, nthreads=threads)
        reps += 1
        elapsed = time.perf_counter() - t0
    w_per_pass = sum(K * n for _, K, n, *_ in packed)
    bpw = {1: 28 / 128, 2: 18 / 128, 3: 10 / 32}
    bytes_per_w = sum(bpw[f] * K * n for f, K, n, *_ in packed) / w_per_pass
    m_eff = min(M, 8)
    w_per_s = w_per_pass * reps / elapsed          # weights x (m_eff activation rows) per second
    gbs = w_per_s * bytes_per_w / 1e9 * m_eff / M  # packed-weight bytes per second at M rows
    tok_s = w_per_s / (total_w * 64) * m_eff       # 64-layer passes per second, x rows each
    return {"value": round(gbs, 4), "unit": "GB/s", "tok_s_equiv": round(tok_s, 5),
            "cores": threads, "kind": "oracle",
            "sample": f"{reps} passes over 2% of the rows of each of the 4 products of one layer "
                      f"({w_per_pass} weights, M={m_eff}), {elapsed:.1f} s; scaled to a 64-layer step"}


def reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    fmt, M = WORKLOADS[args.workload]
    cpu = cpu_baseline(args, fmt, M, budget_s=max(5.0, min(60.0, 0.5 * args.steps)))
    line = {"metric": "packed-weight HBM GB/s (% of peak) & tok/s-equiv, batch-1 27B-shape GEMV",
            "value": cpu["value"], "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "tok_s_equiv": cpu["tok_s_equiv"],
            "config": {"workload": f"64 x 27B-shaped decoder layers, {FMT_NAME[fmt]}, M={M}",
                       "format": args.workload, "M": M},
            "cpu_baseline": cpu,
            "e2e": {"value": cpu["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
