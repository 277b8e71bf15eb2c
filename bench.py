#!/usr/bin/env python3
"""Throughput of the low-bit weight GEMV on synthetic 27B-decoder-shaped layers.

One step = one batch-1 pass over all 64 layers x 4 products (QKV 5120->7168,
O 5120->5120, gate+up 5120->34816, down 17408->5120), i.e. one "token" of the
weight stream, every product a call of the C ABI (lbq_gemv). The headline workload
is the ternary format; --workload selects another one for the headline.

Prints ONE JSON line (rank 0). `value` is packed-weight GB/s of the whole job with
all inputs resident in HBM (4.6 GB of ternary weights per step, far above the
126 MB L2, so no flush is needed); `e2e` repeats the measurement with each step's
activations copied in from pinned host memory and its outputs copied back.
On one GPU the same line carries `configs`: every other workload of the method
measured in the same run (1-bit, 2-bit + rotation, the mixed-format layer, the tiny
GEMV and the batched ternary products at M = 8, 32, 512 and 4096 tokens), each with
its time, rate, roofline, sampled oracle parity and SM clocks, and `load_only`, the
rate of a plain streaming read of a buffer of the same size.
Multi-GPU (torchrun): every rank runs an independent replica on its own weights
("replicas only": the path has no exchange step), the time is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload tern|sign|q2|gemm8|...]
    python bench.py --impl reference   # the fp64 CPU oracle on a bounded sample
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "packed-weight HBM GB/s (% of peak) & tok/s-equiv, batch-1 27B-shape GEMV"
WORKLOADS = {
    # name: (format, M, how the pass runs); format 0: a mixed-format layer (product_fmt).
    # "batch": the pass's independent products (each has its own seeded x) through
    # lbq_gemv_batch, one launch per format and 256 products; "chained": one lbq_gemv
    # call per product in stream order, each allowed to start only as its predecessor
    # finishes (a decoder's order, where a product's x comes from earlier results);
    # "gemm": one lbq_gemm call per product.
    "tern": (1, 1, "batch"), "sign": (2, 1, "batch"), "q2": (3, 1, "batch"), "mixed": (0, 1, "batch"),
    "tern_chained": (1, 1, "chained"), "sign_chained": (2, 1, "chained"),
    "q2_chained": (3, 1, "chained"), "mixed_chained": (0, 1, "chained"),
    "gemm8": (1, 8, "gemm"), "gemm32": (1, 32, "gemm"), "gemm512": (1, 512, "gemm"),
    "gemm4096": (1, 4096, "gemm"),
}
# the workloads measured beside the headline in a one-GPU run (plus the tiny GEMV)
CONFIG_ORDER = ("tern_chained", "sign", "q2", "mixed", "mixed_chained", "gemm8", "gemm32",
                "gemm512", "gemm4096")
MODE_TEXT = {"batch": "independent products, one lbq_gemv_batch call per pass (one launch per format)",
             "chained": "one lbq_gemv per product, each chained to the previous",
             "gemm": "one lbq_gemm per product"}
FMT_NAME = {1: "ternary 5 trits/byte + fp16 scale per 128", 2: "1-bit sign + fp16 scale per 128",
            3: "2-bit 4-level + fp16 scale per 32, input rotated by 512-point RHT",
            0: "mixed: attention (QKV, O) 2-bit + RHT, FFN (gate+up, down) ternary"}
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu capture of
# an 8-layer pass (one launch) scaled by 8 to the 64-layer launch (the traffic grows
# with the units processed), keyed by workload and by the hash of the kernel sources
# it was taken on: reported as null once that source changes. (The figures below were
# captured on hash ddad2f6d44495dbb; the sources changed since on the host side only: the
# plan introspection call and an include.)
NCU_TRAFFIC = {
    # profiles/gemv_batch_tern_8layer_full.md: 605.54 MB read + 3.60 MB written
    ("tern", "24bc8e389e0eaddf"): 8 * 609.143e6,
    # profiles/gemv_batch_sign_8layer_full.md: 388.97 MB read + 5.70 MB written
    ("sign", "24bc8e389e0eaddf"): 8 * 394.667e6,
    # profiles/gemv_batch_q2_8layer_full.md: 826.45 MB read + 3.56 MB written
    ("q2", "24bc8e389e0eaddf"): 8 * 830.004e6,
}


def product_fmt(fmt, mi):
    """The format of product mi (0 QKV, 1 O, 2 gate+up, 3 down) of a layer."""
    if fmt != 0:
        return fmt
    return 3 if mi < 2 else 1  # the mixed layer: 2-bit attention, ternary FFN


def workload_string(fmt, M, layers=64, mode="batch"):
    """The workload's name, shared by both arms of the bench."""
    return (f"{layers} x 27B-shaped decoder layers (QKV 5120x7168, O 5120x5120, "
            f"gate+up 5120x34816, down 17408x5120), {FMT_NAME[fmt]}, M={M}; {MODE_TEXT[mode]}")


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
    ap.add_argument("--no-configs", action="store_true",
                    help="measure the headline workload only")
    ap.add_argument("--configs", default=",".join(("tiny",) + CONFIG_ORDER),
                    help="comma-separated workloads measured beside the headline")
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


GEMV_SOURCES = ("gemv.cu", "lut.cuh", "rht.cuh", "sm100_async.cuh", "lbq_common.cuh")
BATCH_SOURCES = ("gemv_batch.cu", "lut.cuh", "rht.cuh", "sm100_async.cuh", "lbq_common.cuh")
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
    """SM clock and throttle reasons sampled every 5 ms through NVML (read-only queries),
    timestamped, so that each timed region can be summarised on its own; nvidia-smi
    (every 50 ms) when NVML is not usable."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index, pci_bus_id=None):
        self.index, self.pci, self.proc, self.samples = index, pci_bus_id, None, []
        self.stop, self.source = threading.Event(), None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByPciBusId(self.pci) if self.pci
                 else pynvml.nvmlDeviceGetHandleByIndex(self.index))
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            mx = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def poll():
                while not self.stop.is_set():
                    try:
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((time.monotonic(), sm, mx,
                                             [n for n, bit in bits.items() if r & bit]))
                    except Exception:
                        pass
                    time.sleep(0.005)
            self.t = threading.Thread(target=poll, daemon=True)
            self.t.start()
            self.source = "nvml, 5 ms"
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            self.source = "nvidia-smi, 50 ms"
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            f = [v.strip() for v in line.strip().split(",")]
            if len(f) < 9:
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            self.samples.append((time.monotonic(), sm, mx,
                                 [n for n, v in zip(self.NAMES, f[5:9]) if v.lower().startswith("active")]))

    def __exit__(self, *a):
        self.stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        sm, mx, reasons = [], None, set()
        for ts, clk, cmax, rs in list(self.samples):
            if (t0 is not None and ts < t0) or (t1 is not None and ts > t1):
                continue
            sm.append(clk)
            mx = cmax
            reasons.update(rs)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": self.source}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


def pci_bus_string(torch, index):
    """NVML's PCI bus id string of CUDA device `index` ("dddddddd:bb:dd.0"), or None."""
    try:
        p = torch.cuda.get_device_properties(index)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


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


# ------------------------------------------------------------------------------ the model

class WeightStore:
    """Packed 64-layer weight sets, one per format, packed once and shared by the
    workloads (the batched products reuse the ternary set, the mixed layer the 2-bit
    attention and ternary FFN matrices)."""

    def __init__(self, L, synth, n_layers, seed, device):
        self.L, self.synth, self.n, self.seed, self.dev = L, synth, n_layers, seed, device
        self.sets = {}

    def get(self, fmt, layer, mi):
        key = (fmt, layer, mi)
        if key not in self.sets:
            name, K, N = self.synth.LAYER_SHAPES[mi]
            W = self.synth.weights(N, K, self.w_seed(layer, mi), device=self.dev)
            self.sets[key] = self.L.lbq_pack(fmt, W)
            del W
        return self.sets[key]

    def w_seed(self, layer, mi):
        return self.synth.seed_of(self.seed * 1000, layer, mi)

    def drop(self, fmt):
        for k in [k for k in self.sets if k[0] == fmt]:
            del self.sets[k]


def build_products(store, fmt, M, torch, share_outputs=False):
    """Per-product records of one pass: packed weights, activations, outputs."""
    synth, dev = store.synth, store.dev
    prods, shared_y = [], {}
    for layer in range(store.n):
        for mi, (name, K, N) in enumerate(synth.LAYER_SHAPES):
            f = product_fmt(fmt, mi)
            pw = store.get(f, layer, mi)
            X = synth.activations(M, K, synth.seed_of(store.seed * 1000 + 500, layer, mi), device=dev)
            if share_outputs:  # large batches: one output buffer per product shape
                if mi not in shared_y:
                    shared_y[mi] = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                Y = shared_y[mi]
            else:
                Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            prods.append({"layer": layer, "mi": mi, "name": name, "K": K, "N": N, "pw": pw,
                          "X": X, "Y": Y, "fmt": f})
    return prods


class Pass:
    """How one pass runs: its products, the signs, the workspace and the mode."""

    def __init__(self, L, prods, D, M, mode, device, torch):
        self.L, self.prods, self.D, self.M, self.mode = L, prods, D, M, mode
        if mode == "batch":
            self.plist = L.ProductList([(p["pw"], p["X"][0], D.get(p["K"]) if p["fmt"] == 3 else None,
                                         p["Y"][0]) for p in prods])
            self.ws = L.workspace_for_batch(self.plist, device)
        else:
            n = max(L.lbq_workspace_bytes(p["pw"], M) for p in prods)
            self.ws = torch.zeros(max(16, n), dtype=torch.uint8, device=device)

    def run(self, prods=None):
        L, D, M = self.L, self.D, self.M
        if self.mode == "batch" and prods is None:
            L.lbq_gemv_batch(self.plist, self.ws)
            return
        for p in prods if prods is not None else self.prods:
            Dp = D.get(p["K"]) if p["fmt"] == 3 else None
            if M == 1:
                if self.mode == "batch":  # a single product, through the batched call
                    L.lbq_gemv_batch(L.ProductList([(p["pw"], p["X"][0], Dp, p["Y"][0])]), self.ws)
                else:
                    L.lbq_gemv(p["pw"], p["X"][0], Dp, p["Y"][0], self.ws)
            else:
                L.lbq_gemm(p["pw"], p["X"], Dp, p["Y"], self.ws)


def launches_per_step(L, prods, mode, sms=148):
    """Our kernels per pass: for lbq_gemv_batch one launch per format and 256 products of
    it, plus the piece-sum kernel where the library splits a product along K (its rule:
    pieces = ceil(64 * SMs * slices / total unit-slices of the launch), at most the
    slices; none for the 64-layer passes); for chained calls, per product the GEMV plus
    the split-K sum when K spans several slices."""
    if mode == "batch":
        per_fmt = {}
        for p in prods:
            per_fmt.setdefault(p["fmt"], []).append(p)
        n = 0
        for lst in per_fmt.values():
            for i in range(0, len(lst), L.LBQ_BATCH_MAX):
                chunk = lst[i:i + L.LBQ_BATCH_MAX]
                ks = [-(-p["K"] // (1024 if p["fmt"] == L.LBQ_SIGN1 else 512)) for p in chunk]
                W = sum(k * -(-p["N"] // 16) for k, p in zip(ks, chunk))
                split = any(min(k, -(-64 * sms * k // W)) > 1 for k in ks)
                n += 1 + int(split)
        return n
    if mode == "chained":
        return sum(1 + (p["K"] > (1024 if p["fmt"] == L.LBQ_SIGN1 else 512)) for p in prods)
    return None  # lbq_gemm: 2 or 3 kernels per product, as the tile planner decides


def capture(ps, stream, torch):
    """One CUDA graph of a whole pass, after one eager pass."""
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        ps.run()  # eager warm-up (and first-touch) on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            ps.run()
    return graph


def time_replays(graph, stream, steps, warmup, torch, barrier):
    """Device time (ms) of `steps` back-to-back replays after `warmup` untimed ones."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps):
            graph.replay()
        t1.record(stream)
    barrier()
    return t0.elapsed_time(t1)


def roofline(M, algo_bytes, flops, ms_step, n_launch, kernel):
    hbm_peak, tc_peak, tc_sust, peak_src = peaks()
    gbs = algo_bytes / (ms_step * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(gbs / hbm_peak, 4), "peak_source": peak_src,
            "frac_of_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4), "kernel": kernel,
            "algorithmic_bytes_per_launch": algo_bytes / n_launch,
            "avg_launch_us": round(1e3 * ms_step / n_launch, 3)}
    if M >= 512:
        tf = flops / (ms_step * 1e-3) / 1e12
        # frac against the burst peak; a pass of many products runs under the power cap,
        # so the sustained peak is given beside it
        roof.update({"bound": "tensor", "achieved": round(tf, 1), "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": round(tf / tc_peak, 4), "peak_sustained": tc_sust,
                     "frac_of_sustained": round(tf / tc_sust, 4), "hbm_gbs": round(gbs, 1)})
    elif M > 1:
        roof["tflops"] = round(flops / (ms_step * 1e-3) / 1e12, 2)
    return roof


def pass_bytes(prods):
    weight_bytes = sum(p["pw"].nbytes for p in prods)
    act_bytes = sum(p["X"].numel() * 2 for p in prods)
    out_bytes = sum(p["Y"].numel() * 2 for p in prods)
    return weight_bytes, weight_bytes + act_bytes + out_bytes


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

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    fmt, M, mode = WORKLOADS[args.workload]
    store = WeightStore(L, synth, args.layers, args.seed + 7919 * rank, dev)
    prods = build_products(store, fmt, M, torch, share_outputs=M >= 512)
    D = {}
    for K in (synth.HIDDEN, synth.FFN):
        D[K] = L.lbq_rht_signs(args.seed * 31 + K, K, dev)
    ps = Pass(L, prods, D, M, mode, dev, torch)
    weight_bytes, algo_bytes = pass_bytes(prods)
    flops = sum(2 * M * p["K"] * p["N"] for p in prods)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    graph = capture(ps, stream, torch)
    launches = launches_per_step(L, prods, mode)

    # ---- timed region: K replays, inputs resident in HBM
    with ClockSampler(local, pci_bus_string(torch, local)) as clk:
        tc0 = time.monotonic()
        ms = max_over_ranks(time_replays(graph, stream, args.steps, args.warmup, torch, barrier),
                            world, dist, dev, torch)
        tc1 = time.monotonic()
        ms_step = ms / args.steps
        gbs = job_rate(world, weight_bytes, ms_step) / 1e9
        tok_s = job_rate(world, M, ms_step)
        clocks = clk.summary(tc0, tc1)
        kernel = {"batch": "lbq_gemv_batch", "chained": "lbq_gemv", "gemm": "lbq_gemm"}[mode]
        # The dominant kernel's launch duration inside the timed region: the timed step
        # divided by the launches of that kernel in it (the batch kernel: one launch a
        # step per format; per-product calls: the step over the products).
        n_launch = launches if mode == "batch" else len(prods)
        roof = roofline(M, algo_bytes, flops, ms_step, n_launch, f"{kernel} ({args.workload})")
        key = kernel_source_hash(BATCH_SOURCES if mode == "batch" else
                                 GEMV_SOURCES if mode == "chained" else GEMM_SOURCES)
        roof["traffic"] = NCU_TRAFFIC.get((args.workload, key))

        # ---- end to end: activations in from pinned host memory, outputs back, every step
        e2e = end_to_end(L, prods, D, M, mode, stream, args, world, weight_bytes, dist, dev, torch,
                         barrier)

        # ---- sampled parity of the timed configuration against the oracle (rank 0)
        parity = None
        if rank == 0 and not args.no_parity:
            parity = sampled_parity(ps, synth, store, args, dev, torch)

        configs, load_only = None, None
        if world == 1 and not args.no_configs:
            del graph
            load_only = read_probe(L, weight_bytes, stream, torch, dev, barrier)
            configs = measure_configs(L, synth, store, args, D, stream, torch, dev, barrier, clk,
                                      skip=args.workload)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, fmt, M)
        cpu["one_core"] = cpu_baseline(args, fmt, M, budget_s=max(2.0, args.cpu_sample_s / 3),
                                       threads=1)

    if world > 1:
        del graph
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    hbm_peak = peaks()[0]
    line = {
        "metric": METRIC,
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        # the arithmetic: fp32 lookups and sums, or fp16 tensor-core MMAs into fp32
        "dtype": "f32" if M <= 3 or fmt != 1 else "f16 (f32 accumulate)",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) bf16 activations)",
        "tok_s_equiv": round(tok_s, 2), "pct_of_hbm_peak": round(100 * gbs / world / hbm_peak, 2),
        "config": {"workload": workload_string(fmt, M, args.layers, mode),
                   "format": args.workload, "M": M, "layers": args.layers, "mode": mode,
                   "weight_bytes_per_step": weight_bytes, "products_per_step": len(prods),
                   "l2": "inputs larger than L2 (no flush): %.2f GB of weights per step"
                         % (weight_bytes / 1e9),
                   "parallelism": f"replicas x{world}", "graph": "one CUDA graph per step"},
        "roofline": roof, "e2e": e2e,
        "gpu_launches": None if launches is None else args.steps * launches,
        "clocks": clocks, "parity": parity, "cpu_baseline": cpu, "kernel_source": key,
    }
    if load_only:
        line["load_only"] = load_only
        line["roofline"]["frac_of_load_only"] = round(roof["achieved"] / load_only["value"], 4) \
            if roof["unit"] == "GB/s" else None
    if configs:
        line["configs"] = configs
    if M > 1:
        line["tflops"] = round(world * flops / (ms_step * 1e-3) / 1e12, 2)
    print(json.dumps(line), flush=True)


def end_to_end(L, prods, D, M, mode, stream, args, world, weight_bytes, dist, dev, torch, barrier):
    """The pass through the public API with every step's activations copied in from pinned
    host memory and its outputs copied back, all inside the timed region. The steps are
    independent passes, so two sets of buffers alternate on two streams (double
    buffering, as a serving loop over independent requests would run them): one step's
    copies overlap the other set's kernels, and every step still moves its own bytes."""
    sets = []
    for k in range(2):
        xin_host = torch.cat([p["X"].reshape(-1) for p in prods]).cpu().pin_memory()
        xin_dev = torch.empty_like(xin_host, device=dev)
        y_host = torch.empty(sum(p["Y"].numel() for p in prods), dtype=torch.bfloat16).pin_memory()
        y_dev = torch.empty_like(y_host, device=dev)
        e2e_prods, ox, oy = [], 0, 0
        for p in prods:
            vx = xin_dev[ox:ox + p["X"].numel()].view(p["X"].shape)
            vy = y_dev[oy:oy + p["Y"].numel()].view(p["Y"].shape)
            e2e_prods.append(dict(p, X=vx, Y=vy))
            ox += p["X"].numel()
            oy += p["Y"].numel()
        ps = Pass(L, e2e_prods, D, M, mode, dev, torch)
        s = stream if k == 0 else torch.cuda.Stream(device=dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            ps.run()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s):
                xin_dev.copy_(xin_host, non_blocking=True)
                ps.run()
                y_host.copy_(y_dev, non_blocking=True)
        sets.append((g, s, ps, xin_host, xin_dev, y_host, y_dev))
    e_steps = max(10, args.steps // 4)
    for i in range(max(args.warmup, 2)):
        g, s = sets[i % 2][:2]
        with torch.cuda.stream(s):
            g.replay()
    torch.cuda.synchronize()
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    start.record(sets[0][1])
    sets[1][1].wait_event(start)
    for i in range(e_steps):
        g, s = sets[i % 2][:2]
        with torch.cuda.stream(s):
            g.replay()
    ends = []
    for _, s, *_ in sets:
        e = torch.cuda.Event(enable_timing=True)
        e.record(s)
        ends.append(e)
    barrier()
    torch.cuda.synchronize()
    ems = max_over_ranks(max(start.elapsed_time(e) for e in ends), world, dist, dev, torch)
    e_step = ems / e_steps
    h2d, d2h = sets[0][3].numel() * 2, sets[0][5].numel() * 2
    del sets
    return {"value": round(job_rate(world, weight_bytes, e_step) / 1e9, 1), "unit": "GB/s",
            "tok_s_equiv": round(job_rate(world, M, e_step), 2),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelining": "two streams, two buffer sets: a step's copies overlap the other set's kernels"}


def read_probe(L, nbytes, stream, torch, dev, barrier, reps=20):
    """The rate of lbq_read_probe, a plain streaming read, over a buffer as large as a
    pass's weights: the measured ceiling for a weight stream on this GPU."""
    n = (int(nbytes) + 15) // 16 * 16
    buf = torch.ones(n, dtype=torch.uint8, device=dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(3):
            L.lbq_read_probe(buf, sink)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(reps):
            L.lbq_read_probe(buf, sink)
        t1.record(stream)
    barrier()
    ms = t0.elapsed_time(t1) / reps
    del buf
    return {"value": round(n / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "bytes": n,
            "kernel": "lbq_read_probe (16-byte no-allocate loads, 4 CTAs per SM)",
            "frac_of_measured_copy": round(n / (ms * 1e-3) / 1e9 / peaks()[0], 4)}


def measure_configs(L, synth, store, args, D, stream, torch, dev, barrier, clk, skip):
    """Every other workload of the method, measured one after another in this run."""
    out = {}
    names = [c.strip() for c in args.configs.split(",") if c.strip()]
    for name in names:
        if name == skip:
            continue
        if name == "tiny":
            out["tiny"] = tiny_config(L, synth, stream, torch, dev, barrier, clk)
            continue
        if name not in WORKLOADS:
            continue
        fmt, M, mode = WORKLOADS[name]
        prods = build_products(store, fmt, M, torch, share_outputs=M >= 512)
        ps = Pass(L, prods, D, M, mode, dev, torch)
        weight_bytes, algo_bytes = pass_bytes(prods)
        flops = sum(2 * M * p["K"] * p["N"] for p in prods)
        graph = capture(ps, stream, torch)
        # a short timing fixes the step count: at least ~0.3 s of timed replays, so that
        # the clock samples cover the region
        est = time_replays(graph, stream, 2, 2, torch, barrier) / 2
        steps = int(min(400, max(5, math.ceil(300.0 / max(est, 1e-3)))))
        tc0 = time.monotonic()
        ms = time_replays(graph, stream, steps, 3, torch, barrier)
        tc1 = time.monotonic()
        del graph
        ms_step = ms / steps
        launches = launches_per_step(L, prods, mode)
        n_launch = launches if mode == "batch" else len(prods)
        kernel = {"batch": "lbq_gemv_batch", "chained": "lbq_gemv", "gemm": "lbq_gemm"}[mode]
        roof = roofline(M, algo_bytes, flops, ms_step, n_launch, f"{kernel} ({name})")
        src = kernel_source_hash(BATCH_SOURCES if mode == "batch" else
                                 GEMV_SOURCES if mode == "chained" else GEMM_SOURCES)
        roof["traffic"] = NCU_TRAFFIC.get((name, src))
        entry = {"workload": workload_string(fmt, M, args.layers, mode), "M": M, "mode": mode,
                 "ms_per_step": round(ms_step, 5), "steps": steps, "warmup": 3,
                 "weight_bytes_per_step": weight_bytes,
                 "value": round(weight_bytes / (ms_step * 1e-3) / 1e9, 1), "unit": "GB/s",
                 "tok_s_equiv": round(M / (ms_step * 1e-3), 2),
                 "pct_of_hbm_peak": round(100 * weight_bytes / (ms_step * 1e-3) / 1e9 / peaks()[0], 2),
                 "gpu_launches_per_step": launches,
                 "roofline": roof, "clocks": clk.summary(tc0, tc1)}
        if M > 1:
            entry["tflops"] = round(flops / (ms_step * 1e-3) / 1e12, 2)
            entry["tokens_per_s"] = entry.pop("tok_s_equiv")
        if not args.no_parity:
            entry["parity"] = sampled_parity(ps, synth, store, args, dev, torch)
        out[name] = entry
        del prods, ps
        torch.cuda.empty_cache()
    return out


def tiny_config(L, synth, stream, torch, dev, barrier, clk):
    """The tiny ternary GEMV (K = 512, N = 256): every output against the oracle, and its
    launch time (one product per step, launch-bound)."""
    import numpy as np

    import oracle
    K, N = 512, 256
    W = synth.weights(N, K, 0)
    x = synth.activations(1, K, 1)
    pw = L.lbq_pack(L.LBQ_TERN5, W.to(dev))
    xd = x[0].to(dev)
    y = torch.empty(N, dtype=torch.bfloat16, device=dev)
    prods = [{"K": K, "N": N, "fmt": 1, "pw": pw, "X": xd.view(1, K), "Y": y.view(1, N)}]
    graph = capture(Pass(L, prods, {}, 1, "chained", dev, torch), stream, torch)
    steps = 2000
    tc0 = time.monotonic()
    ms = time_replays(graph, stream, steps, 10, torch, barrier)
    tc1 = time.monotonic()
    del graph
    codes, scales = oracle.pack(1, W.numpy())
    codes_ok = bool(np.array_equal(pw.codes.cpu().numpy(), oracle.group4(codes)))
    Y, B = oracle.gemm(1, codes, scales, K, synth.bf16_bits(x), None)
    err = np.abs(y.float().cpu().double().numpy() - Y[0]) / np.maximum(2.0 ** -8 * B[0], 1e-300)
    assert codes_ok and np.all(err <= 1.0), "tiny GEMV differs from the oracle"
    return {"workload": "tiny ternary GEMV K=512 x N=256, batch 1 (every output checked), lbq_gemv",
            "us_per_product": round(1e3 * ms / steps, 3), "steps": steps,
            "parity": {"outputs_checked": int(N), "max_err_over_bound": round(float(err.max()), 4),
                       "codes_bit_exact": codes_ok},
            "clocks": clk.summary(tc0, tc1)}


def sampled_parity(ps, synth, store, args, dev, torch):
    """Re-draws a few timed matrices' weights, checks sampled outputs with the oracle:
    12 groups of four weight rows of four products, over up to 8 token rows spread
    across the batch. The outputs are those of a whole pass run as timed."""
    import numpy as np

    import oracle
    prods, M = ps.prods, ps.M
    worst, checked = 0.0, 0
    picks = [prods[0], prods[1], prods[2], prods[-1]]
    rng = np.random.default_rng(0)
    toks = np.unique(np.linspace(0, M - 1, min(M, 8)).round().astype(int))
    if ps.M >= 512:
        ps.run(picks)  # shared output buffers: recompute the products checked below
    else:
        ps.run()
    torch.cuda.synchronize()
    for p in picks:
        fmt = p["fmt"]
        if ps.M >= 512:
            ps.run([p])
            torch.cuda.synchronize()
        W = synth.weights(p["N"], p["K"], store.w_seed(p["layer"], p["mi"]), device=dev)
        # whole groups of four rows (the library's storage order), 12 of them
        groups = np.sort(rng.choice(p["N"] // 4, size=min(12, p["N"] // 4), replace=False))
        rows = (4 * groups[:, None] + np.arange(4)[None, :]).ravel()
        Wr = W[torch.from_numpy(rows).to(dev)].cpu().numpy()
        del W
        codes, scales = oracle.pack(fmt, Wr)
        got_codes = p["pw"].codes[torch.from_numpy(groups).to(dev)].cpu().numpy()
        assert np.array_equal(oracle.group4(codes), got_codes), \
            "timed weights differ from the oracle's packing"
        Xs = p["X"][torch.from_numpy(toks).to(dev)]
        Do = oracle.rht_signs(args.seed * 31 + p["K"], p["K"]) if fmt == 3 else None
        Y, B = oracle.gemm(fmt, codes, scales, p["K"], synth.bf16_bits(Xs), Do,
                           nthreads=os.cpu_count() or 1)
        yg = p["Y"][torch.from_numpy(toks).to(dev)][:, torch.from_numpy(rows).to(dev)]
        yg = yg.float().cpu().double().numpy()
        ratio = np.abs(yg - Y) / np.maximum(2.0 ** -8 * B, 1e-300)
        assert np.all(ratio <= 1.0), f"{p['name']}: outputs outside 2^-8 sum|w x|"
        worst = max(worst, float(ratio.max()))
        checked += ratio.size
    return {"outputs_checked": checked, "max_err_over_bound": round(worst, 4), "codes_bit_exact": True}


def cpu_baseline(args, fmt, M, budget_s=None, threads=None):
    """The oracle (fp64 C, all host cores unless `threads`) on a bounded sample of the
    same workload."""
    import oracle
    from bit_weight_only_ternary_b200 import synth
    budget_s = budget_s or args.cpu_sample_s
    threads = threads or os.cpu_count() or 1
    # sample: the same fraction of rows of each of the four products of one layer
    total_w = sum(K * N for _, K, N in synth.LAYER_SHAPES)
    packed = []
    for mi, (name, K, N) in enumerate(synth.LAYER_SHAPES):
        n = max(os.cpu_count() or 1, int(N * 0.02))
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
                      f"({w_per_pass} weights, M={m_eff}), {elapsed:.1f} s on {threads} thread(s); "
                      f"scaled to a 64-layer step"}


def reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    fmt, M, mode = WORKLOADS[args.workload]
    cpu = cpu_baseline(args, fmt, M, budget_s=max(5.0, min(60.0, 0.5 * args.steps)))
    line = {"metric": METRIC,
            "value": cpu["value"], "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "tok_s_equiv": cpu["tok_s_equiv"],
            "config": {"workload": workload_string(fmt, M, args.layers, mode),
                       "format": args.workload, "M": M, "layers": args.layers, "mode": mode},
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
