#!/usr/bin/env python
"""Benchmark of the ConvLinear4bit (ConvRot W4A4) hot path on B200.

One step = the whole per-call path on one batch of synthetic FLUX-shaped input resident in
HBM: fused RHT + int4 quantisation + packing of the activations, then the tcgen05 W4A4 GEMM
with the fused dequantisation epilogue. Weights are prepacked once before timing (the
offline step of the method). Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config qkv] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): tokens are data-parallel; every rank runs its own
batch of M tokens against a replicated weight with no collective on the data path (weak
scaling). Timing: W untimed warm-up steps; then K steps back to back between two CUDA events
on the launching stream, barrier + synchronize on both sides, the slowest rank's time counts.
Instead of an L2 flush, each step runs on the next of several copies of all its operands
(activations, codes, weights, output), together several times the L2 size, so no step finds
its operands in L2. Events between the two kernels of every step give each kernel's time.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

NVSMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--config", default="qkv")
    p.add_argument("--group", type=int, default=None,
                   help="RHT group size (default: the workload's first group)")
    p.add_argument("--impl", default="ours", choices=("ours", "reference"))
    p.add_argument("--scaling", default="weak", choices=("weak", "strong"),
                   help="weak: every rank runs its own batch of M tokens; strong: one batch of M "
                        "tokens split over the ranks by rows (dp.run_sharded)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--record-traffic", metavar="NCU_CSV",
                   help="write profiles/ncu_traffic_<config>.json from ncu --csv captures "
                        "(comma-separated) of dram__bytes_read.sum and dram__bytes_write.sum, "
                        "then exit")
    p.add_argument("--variant", default="w4a4", choices=("w4a4", "w8a8", "nvfp4", "mxfp4", "fused"),
                   help="w4a4: the ConvLinear4bit layer (headline); w8a8: the int8 variant; "
                        "nvfp4: the floating-point (e2m1 + e4m3 block scales) variant; "
                        "mxfp4: e2m1 with a power-of-two (e8m0) scale per 32 K; fused: the W4A4 "
                        "layer through its one-call entry point (codes in a caller workspace)")
    return p.parse_args()


def metric_name(variant="w4a4"):
    if variant == "nvfp4":
        return "ConvRot NVFP4 layer TOPS and RHT+fp4-quant GB/s at FLUX-like M=4608 shapes"
    if variant == "mxfp4":
        return "ConvRot MXFP4 layer TOPS and RHT+fp4-quant GB/s at FLUX-like M=4608 shapes"
    if variant == "w8a8":
        return "ConvRot W8A8 layer TOPS and RHT+int8-quant GB/s at FLUX-like M=4608 shapes"
    if variant == "fused":
        return "ConvLinear4bit (fused call) TOPS and RHT+int4-quant GB/s at FLUX-like M=4608 shapes"
    return "ConvLinear4bit TOPS and RHT+int4-quant GB/s at FLUX-like M=4608 shapes"


def workload_desc(w, g, K_pad, variant="w4a4"):
    codes = {"w8a8": "int8 codes (W8A8)", "nvfp4": "NVFP4 codes (e2m1, e4m3 per 16 K, K4)",
             "mxfp4": "MXFP4 codes (e2m1, e8m0 per 32 K, K4)"}.get(
        variant, "packed int4 codes (W4A4)")
    return {
        "workload": f"{w.name}: X bf16 [{w.M},{w.K}] x W bf16 [{w.N},{w.K}], group {g}, {codes}",
        "M": w.M, "N": w.N, "K": w.K, "K_pad": K_pad, "group": g,
        "global_batch": w.M, "seq_len": w.M,
    }


# ~1 ms at 2 GHz of untimed device work before a timed run: the host enqueues the first steps
# meanwhile, and stays ahead of the device from then on (a step takes it far less time to
# enqueue than the device takes to run)
PRIME_CYCLES = 2_000_000


def l2_bytes(dev) -> int:
    import torch
    size = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0)
    return int(size) if size else 126 * 2**20


KERNEL_SOURCES = ("capi.cu", "internal.h", "ptx.cuh", "rht_quant.cuh", "rht_quant_ring.cuh",
                  "gemm_common.cuh",
                  "w4a4_gemm.cuh", "w8a8_gemm.cuh", "nvfp4_gemm.cuh", "mxfp4_gemm.cuh")


def kernel_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "rotation_w4a4_quantized_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_key(kernel_name: str):
    """The key a bench line uses for a kernel in ncu's report (None: not one of ours)."""
    import re
    for k in ("w4a4_gemm_kernel", "w8a8_gemm_kernel", "nvfp4_gemm_kernel", "mxfp4_gemm_kernel"):
        if k in kernel_name:
            return k
    m = (re.search(r"rht_quant_reg_kernel<\s*\d+,\s*(\d+)", kernel_name)       # <G, QM, ...>
         or re.search(r"rht_quant_ring_kernel<\s*\d+,\s*(\d+)", kernel_name))  # <G, QM>
    if m:   # code mode: 7 int4, 127 int8, 6 NVFP4, 5 MXFP4
        return {"7": "rht_quant_kernel", "127": "rht_quant_kernel_i8",
                "6": "rht_quant_kernel_fp4", "5": "rht_quant_kernel_mx"}.get(m.group(1))
    return None


UNIT_BYTES = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6,
              "GB": 1e9}


def record_traffic(csv_path: str, config: str, command: str):
    """Average DRAM bytes per launch, per kernel, from an ncu --csv capture; store them with
    the hash of the kernel sources they were taken from."""
    import csv
    sums = {}
    lines = []
    for one in csv_path.split(","):
        with open(one) as f:
            body = [ln for ln in f if ln.startswith('"')]
        lines += body if not lines else body[1:]          # one header row
    for row in csv.DictReader(lines):
        key = traffic_key(row.get("Kernel Name", ""))
        metric = row.get("Metric Name", "")
        if key is None or metric not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        val = float(row["Metric Value"].replace(",", "")) * UNIT_BYTES[row.get("Metric Unit", "byte")]
        d = sums.setdefault(key, {"dram__bytes_read.sum": [], "dram__bytes_write.sum": []})
        d[metric].append(val)
    kernels = {k: {"dram_read_bytes": int(round(statistics.mean(v["dram__bytes_read.sum"]))),
                   "dram_write_bytes": int(round(statistics.mean(v["dram__bytes_write.sum"]))),
                   "launches": len(v["dram__bytes_read.sum"])}
               for k, v in sums.items() if v["dram__bytes_read.sum"]}
    out = {"what": "DRAM bytes per launch (mean over the captured launches) from ncu; valid only "
                   "while the kernel sources hash to source_sha256",
           "command": command,
           "source_files": [f"rotation_w4a4_quantized_b200/csrc/{n}" for n in KERNEL_SOURCES],
           "source_sha256": kernel_sources_sha256(), "kernels": kernels}
    path = os.path.join(ROOT, "profiles", f"ncu_traffic_{config}.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out["kernels"]))


def profiled_traffic(kernel: str, config: str):
    """ncu DRAM bytes per launch for `kernel`, if profiles/ holds a capture of the current
    kernel sources on this workload; None otherwise (the counters no longer apply)."""
    path = os.path.join(ROOT, "profiles", f"ncu_traffic_{config}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if kernel_sources_sha256() != d.get("source_sha256"):
        return None
    k = d.get("kernels", {}).get(kernel)
    return None if k is None else k["dram_read_bytes"] + k["dram_write_bytes"]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu=timestamp,{NVSMI_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100", "-i", str(self.dev)],
                stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()

    def summary(self, t0: float, t1: float):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        smax = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        power = [float(r[4]) for r in rows if r[4].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i] == "Active"})
        loaded = [s for s, p in zip(sm, power) if p > 200.0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(rows), "reasons": reasons}


# ----------------------------------------------------------------------------- oracle leg
def oracle_step_fn(w, g, X, W, variant="w4a4"):
    """(step(rows), quant(rows), gemm(q)): the oracle's layer on the first `rows` token rows,
    its rotate + quantise of those rows alone, and its GEMM + dequantisation of quant's output."""
    import numpy as np
    from oracle import convrot_oracle as O
    X64 = X.float().numpy().astype(np.float64)
    W64 = W.float().numpy().astype(np.float64)
    if variant == "mxfp4":
        # the MXFP4 blocks span K4 (K_pad rounded up to 64): zero columns past K give whole zero
        # groups, as on the device
        K4 = -(-O.padded_k(w.K, g) // 64) * 64
        X64 = np.pad(X64, ((0, 0), (0, K4 - w.K)))
        _, _, ew, xw = O.rotate_quant_mxfp4(np.pad(W64, ((0, 0), (0, K4 - w.K))), g)

        def quant(rows: int):
            return O.rotate_quant_mxfp4(X64[:rows], g)

        def gemm(q):
            _, _, ex, xx = q
            return O.mxfp4_gemm(ex, xx, ew, xw)
    elif variant == "nvfp4":
        _, _, gw, ew, sbw = O.rotate_quant_nvfp4(W64, g)                    # offline prepack

        def quant(rows: int):
            return O.rotate_quant_nvfp4(X64[:rows], g)

        def gemm(q):
            _, _, gx, ex, sbx = q
            return O.dequant(O.nvfp4_gemm(ex, sbx, ew, sbw), gx, gw)
    elif variant == "w8a8":
        cw, sw = O.rotate_quant_int8(W64, g)                                # offline prepack

        def quant(rows: int):
            return O.rotate_quant_int8(X64[:rows], g)

        def gemm(q):
            cx, sx = q
            return O.dequant(O.int_gemm_fp64(cx, cw), sx, sw)
    else:
        _, sw, cw = O.rotate_quant(W64, g)                                  # offline prepack

        def quant(rows: int):
            return O.rotate_quant(X64[:rows], g)

        def gemm(q):
            _, sx, cx = q
            return O.dequant(O.int_gemm_fp64(cx, cw), sx, sw)

    def step(rows: int):
        return gemm(quant(rows))
    return step, quant, gemm


def oracle_steps(variant: str) -> str:
    if variant == "mxfp4":
        return ("fp64 RHT, power-of-two scales per 32 K and e2m1 codes by nearest-even rounding, "
                "fp64 block-scaled GEMM")
    if variant == "nvfp4":
        return ("fp64 RHT, e4m3 block scales and e2m1 codes by nearest-even rounding, fp64 "
                "block-scaled GEMM, fp64 dequant")
    return "fp64 RHT, rint, fp64-BLAS integer GEMM, fp64 dequant"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, g, K_pad, X, W, budget_s=12.0, variant="w4a4"):
    """Time the oracle (as it stands) on a bounded sample of the same workload: a row sample
    sized to about a quarter of the budget, repeated until the budget is spent (the whole
    workload is one row sample when it is cheap enough)."""
    step, quant, gemm = oracle_step_fn(w, g, X, W, variant)
    rows = 8
    t = 0.0
    while True:
        t0 = time.perf_counter()
        step(rows)
        t = time.perf_counter() - t0
        if t >= budget_s / 4 or rows >= w.M:
            break
        rows = min(w.M, max(rows * 2, int(rows * (budget_s / 4) / max(t, 1e-3))))
    runs, total = 1, t
    while total < budget_s:
        t0 = time.perf_counter()
        step(rows)
        total += time.perf_counter() - t0
        runs += 1
    tops = 2.0 * rows * w.N * K_pad * runs / total / 1e12
    # the oracle's rotate + quantise alone on the same rows (in the kernel's byte count), and its
    # GEMM + dequantisation alone
    t0 = time.perf_counter()
    q = quant(rows)
    tq = time.perf_counter() - t0
    t0 = time.perf_counter()
    gemm(q)
    tg = time.perf_counter() - t0
    q_bytes = rows * (2 * w.K + (K_pad if variant == "w8a8" else K_pad // 2)
                      + (K_pad // 32 if variant == "mxfp4" else 4))
    return {"value": tops, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} of {w.M} token rows x all {w.N} outputs ({oracle_steps(variant)}), "
                      f"{runs} runs in {total:.1f} s",
            "rht_quant_gbs": q_bytes / tq / 1e9,
            "gemm_tops": 2.0 * rows * w.N * K_pad / tg / 1e12}


def run_reference(args, w, g, K_pad, rank, world):
    from synthetic import make_inputs
    if rank != 0:
        return
    X, W, _ = make_inputs(w)
    step, _, _ = oracle_step_fn(w, g, X, W, args.variant)
    t0 = time.perf_counter()
    step(8)
    t8 = max(time.perf_counter() - t0, 1e-3)
    per_step_budget = 90.0 / max(args.steps + args.warmup, 1)
    rows = int(max(1, min(w.M, 8 * per_step_budget / t8)))
    for _ in range(args.warmup):
        step(rows)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step(rows)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    tops = 2.0 * rows * w.N * K_pad / (ms / 1e3) / 1e12
    cores = blas_threads()
    sample = (f"{rows} of {w.M} token rows per step x all {w.N} outputs (CPU oracle: "
              f"{oracle_steps(args.variant)})")
    line = {
        "metric": metric_name(args.variant), "value": tops, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_desc(w, g, K_pad, args.variant), "impl": "reference",
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU leg
def int8_library_reference(w, dev, stream, K):
    """cuBLASLt int8 x int8 -> int32 (torch._int_mm) as a measured reference for the INT8 tensor
    peak; None where the library call is unavailable."""
    import torch
    try:
        def timed(m, n, k, copies, launches):
            ops = [(torch.randint(-7, 8, (m, k), dtype=torch.int8, device=dev),
                    torch.randint(-7, 8, (n, k), dtype=torch.int8, device=dev))
                   for _ in range(copies)]
            for a, b in ops:
                torch._int_mm(a, b.t())
            torch.cuda.synchronize()
            if launches == 1:
                best = None
                for _ in range(10):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    torch._int_mm(ops[0][0], ops[0][1].t())
                    e1.record(stream)
                    e1.synchronize()
                    t = e0.elapsed_time(e1)
                    best = t if best is None else min(best, t)
                return 2.0 * m * n * k / (best / 1e3) / 1e12
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(PRIME_CYCLES)
            e0.record(stream)
            for i in range(launches):
                a, b = ops[i % copies]
                torch._int_mm(a, b.t())
            e1.record(stream)
            e1.synchronize()
            return 2.0 * m * n * k * launches / (e0.elapsed_time(e1) / 1e3) / 1e12

        peak = timed(8192, 8192, 8192, 1, 1)
        k = -(-w.K // 64) * 64
        shape = timed(w.M, w.N, k, 3, max(30, min(K, 300)))
        return {"what": "cuBLASLt int8 GEMM (torch._int_mm, int32 out), measured reference",
                "tops_8192_cubed_best_of_10": peak, f"tops_{w.M}x{w.N}x{k}": shape}
    except (RuntimeError, AttributeError) as e:
        return {"unavailable": str(e).splitlines()[0][:200]}


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from synthetic import CONFIGS, make_inputs
    w = CONFIGS[args.config]
    g = args.group if args.group is not None else w.group
    if g not in w.groups:
        raise SystemExit(f"group {g} is not one of {args.config}'s groups {w.groups}")
    K_pad = -(-w.K // g) * g

    if args.record_traffic:
        record_traffic(args.record_traffic, args.config, os.environ.get("TRAFFIC_COMMAND", ""))
        return
    if args.impl == "reference":
        run_reference(args, w, g, K_pad, rank, world)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from rotation_w4a4_quantized_b200 import binding as B
    from rotation_w4a4_quantized_b200.dp import (job_throughput, local_rows, run_sharded,
                                                 slowest_rank_ms)

    strong = args.scaling == "strong"
    # weak: each rank its own batch of M tokens (its own seed); strong: one global batch, the
    # same bytes on every rank, of which each rank takes its rows
    X, W, _ = make_inputs(w, seed=None if strong or not rank else w.seed + 1000 * rank)
    dev = torch.device("cuda", local_rank)
    Xg = X
    if strong:
        X = local_rows(Xg, rank, world).contiguous()
    Ml = X.shape[0]                               # token rows this rank runs per step
    Xd, Wd = X.to(dev), W.to(dev)
    int8 = args.variant == "w8a8"
    fused = args.variant == "fused"
    mx = args.variant == "mxfp4"
    fp4 = mx or args.variant == "nvfp4"
    u8, f32, bf16 = torch.uint8, torch.float32, torch.bfloat16
    gw0 = None
    if mx:
        K_pad = B.nvfp4_k(w.K, g)                 # the FP4 paths run over K4 (multiple of 64)
        qw0, sfw0 = B.prepack_weight_mxfp4(Wd, g)
        ldq = B.packed_stride(K_pad)
        sf_bytes = B.mxfp4_scale_bytes(Ml, w.K, g, False)

        def quant(st):
            B.rotate_quant_act_mxfp4(st["X"], g, q=st["qx"], sf=st["sfx"])

        def linear(st):
            B.mxfp4_linear(st["qx"], st["sfx"], st["qw"], st["sfw"], K_pad, out=st["Y"])

        def layer(X_):
            return B.conv_linear_mxfp4(X_, qw0, sfw0, g)
    elif fp4:
        K_pad = B.nvfp4_k(w.K, g)                 # the NVFP4 path runs over K4 (multiple of 64)
        qw0, sfw0, gw0 = B.prepack_weight_nvfp4(Wd, g)
        ldq = B.packed_stride(K_pad)
        sf_bytes = B.nvfp4_scale_bytes(Ml, w.K, g, False)

        def quant(st):
            B.rotate_quant_act_nvfp4(st["X"], g, q=st["qx"], sf=st["sfx"], g=st["sx"])

        def linear(st):
            B.nvfp4_linear(st["qx"], st["sfx"], st["sx"], st["qw"], st["sfw"], st["gw"], K_pad,
                           out=st["Y"])

        def layer(X_):
            return B.conv_linear_nvfp4(X_, qw0, sfw0, gw0, g)
    else:
        if int8:
            qw0, sw0 = B.rotate_quant_i8(Wd, g)
            ldq = B.int8_stride(K_pad)
            q_fn, l_fn, layer_fn = B.rotate_quant_i8, B.w8a8_linear, B.conv_linear_8bit
        else:
            qw0, sw0 = B.prepack_weight(Wd, g)
            ldq = B.packed_stride(K_pad)
            q_fn, l_fn, layer_fn = B.rotate_quant_act, B.w4a4_linear, B.conv_linear_4bit

        def quant(st):
            q_fn(st["X"], g, st["qx"], st["sx"])

        def linear(st):
            l_fn(st["qx"], st["sx"], st["qw"], st["sw"], K_pad, out=st["Y"])

        def layer(X_):
            if fused:
                return B.w4a4_linear_fused(X_, qw0, sw0, g)
            return layer_fn(X_, qw0, sw0, g, K_pad)

        def step_fused(st):
            B.w4a4_linear_fused(st["X"], st["qw"], st["sw"], g, out=st["Y"], workspace=st["ws"])

    def new_set():
        st = {"X": Xd.clone(), "qx": torch.empty(Ml, ldq, dtype=u8, device=dev),
              "Y": torch.empty(Ml, w.N, dtype=bf16, device=dev), "qw": qw0.clone()}
        if not mx:                                # MXFP4 has no per-row scale
            st["sx"] = torch.empty(Ml, dtype=f32, device=dev)
        if fp4:
            st.update(sfw=sfw0.clone(), sfx=torch.empty(sf_bytes, dtype=u8, device=dev))
            if not mx:
                st["gw"] = gw0.clone()
        else:
            st["sw"] = sw0.clone()
        if fused:
            st["ws"] = torch.empty(B.fused_workspace_bytes(Ml, w.K, g), dtype=u8, device=dev)
        return st

    # L2 policy: inputs larger than L2 instead of a flush inside the timed region. Each step
    # works on the next of S copies of all its operands (activations, codes, weights, output),
    # S chosen so that at least three L2 capacities stream through between two uses of a copy.
    sets = [new_set()]
    set_bytes = sum(t.numel() * t.element_size() for t in sets[0].values())
    n_sets = max(3, -(-3 * l2_bytes(dev) // set_bytes))
    sets += [new_set() for _ in range(n_sets - 1)]
    stream = torch.cuda.current_stream()

    def step(st):
        if fused:
            step_fused(st)
        else:
            quant(st)
            linear(st)

    for i in range(max(args.warmup, n_sets)):
        step(sets[i % n_sets])
    torch.cuda.synchronize()
    assert B.device_status() == 0
    if strong:
        # the split-and-gather of one global batch reproduces the unsplit layer bit for bit
        Xgd = Xg.to(dev)
        y_split = run_sharded(Xgd, layer, rank, world)
        assert torch.equal(y_split, layer(Xgd)), "row-split layer differs from the whole batch"
        del Xgd, y_split

    K = args.steps

    def timed_run(kernel_events: bool):
        """K steps back to back between two events (after an untimed device-side prime, so the
        host stays ahead). With kernel_events, events also sit between the two kernels of
        every step; each one drains the stream, so that run is a little slower overall."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)] if kernel_events else []
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        torch.cuda._sleep(PRIME_CYCLES)
        t0.record(stream)
        for i in range(K):
            st = sets[i % n_sets]
            if not kernel_events:
                step(st)
                continue
            ev[i][0].record(stream)
            quant(st)
            ev[i][1].record(stream)
            linear(st)
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        total = slowest_rank_ms(t0.elapsed_time(t1))      # max over ranks (device time)
        if not kernel_events:
            return total, None, None
        q = [a.elapsed_time(b) for a, b in ev]
        gm = [ev[i][1].elapsed_time(ev[i + 1][0] if i + 1 < K else t1) for i in range(K)]
        return total, q, gm

    def per_launch_ms(fn, operand_sets):
        """Average launch duration of one kernel: K launches back to back over rotating operand
        copies, between two events. The launches are captured once in a CUDA graph (each
        operand copy in turn) and the graph is replayed: a single quantisation launch takes the
        device less time than the Python binding takes the host to issue one call, so timing
        launches issued one by one from Python would time the host."""
        n = len(operand_sets)
        for i in range(n):
            fn(operand_sets[i])
        torch.cuda.synchronize()
        per_graph = n * max(1, min(K, 200) // n)
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(graph, stream=cap):
                for i in range(per_graph):
                    fn(operand_sets[i % n])
        torch.cuda.synchronize()
        replays = max(1, -(-K // per_graph))
        graph.replay()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(replays):
            graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        del graph
        return slowest_rank_ms(t0.elapsed_time(t1)) / (replays * per_graph)

    # the quantisation alone touches far fewer bytes per launch than a step: rotate over more
    # copies of its operands (sharing the step's code and scale buffers)
    q_bytes = sum(sets[0][k].numel() * sets[0][k].element_size()
                  for k in ("X", "qx", "sx", "sfx") if k in sets[0])
    n_q = max(n_sets, -(-3 * l2_bytes(dev) // q_bytes))
    q_sets = [dict(sets[i % n_sets], X=Xd.clone()) if i >= n_sets else sets[i]
              for i in range(n_q)]

    with ClockSampler(local_rank) as clk:
        t_wall0 = time.time()
        total_ms, _, _ = timed_run(kernel_events=False)          # the headline: K plain steps
        if fused:
            # the fused call's two kernels are not separable by events between calls: the GEMM's
            # time is the fused call's minus its quantisation's, each timed alone
            ev_total_ms = ev_quant_ms = ev_gemm_ms = None
            quant_ms = per_launch_ms(quant, q_sets)
            gemm_ms = per_launch_ms(step_fused, sets) - quant_ms
        else:
            ev_total_ms, ev_quant_ms, ev_gemm_ms = timed_run(kernel_events=True)
            quant_ms = per_launch_ms(quant, q_sets)
            gemm_ms = per_launch_ms(linear, sets)
        t_wall1 = time.time()
    del q_sets
    ms_per_step = total_ms / K
    ops = 2.0 * Ml * w.N * K_pad

    def job_rate(ms):
        """Whole-job ops/s: strong scaling divides the one global batch by the slowest rank."""
        if strong:
            return 2.0 * w.M * w.N * K_pad / (ms * 1e-3)
        return job_throughput(ops, world, ms)

    value = job_rate(ms_per_step) / 1e12
    clocks = clk.summary(t_wall0, t_wall1)
    assert B.device_status() == 0

    hbm_gbs, bf16_tflops, peak_src = measured_peaks()
    # the contraction's own dtype: nominal dense INT8 / BF16 = 4.5 / 2.25, FP4 / BF16 = 9 / 2.25
    peak_ratio = 4.0 if fp4 else 2.0
    int8_peak = peak_ratio * bf16_tflops
    gemm_avg, quant_avg = gemm_ms, quant_ms
    quant_bytes = Ml * w.K * 2 + Ml * (K_pad if int8 else K_pad // 2)
    if mx:
        quant_bytes += Ml * K_pad // 32                  # one e8m0 scale per 32 K
    elif fp4:
        quant_bytes += Ml * K_pad // 16 + Ml * 4        # e4m3 per 16 K, fp32 row scale
    else:
        quant_bytes += Ml * 4                            # fp32 row scale
    quant_gbs = quant_bytes / (quant_avg / 1e3) / 1e9
    config = workload_desc(w, g, K_pad, args.variant)
    config["parallelism"] = (f"dp{world}: one batch of {w.M} tokens split by rows ({Ml} on rank "
                             f"0), replicated weights, no collective on the data path" if strong
                             else f"dp{world}: {w.M} tokens per rank, replicated weights, no "
                                  f"collective on the data path")
    config["l2"] = (f"inputs larger than L2: {n_sets} rotating copies of every operand "
                    f"({set_bytes / 1e6:.0f} MB each), no flush inside the timed region")
    del sets
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.int32, device=dev)   # 256 MiB > L2

    # ---------------------------------------------------------------- end to end (host buffers)
    # Through the public API with host buffers: every step copies its activations from pinned
    # host memory and its result back. "e2e" streams the steps with HostPipeline (copies in,
    # layer and copies out of consecutive steps overlap on three streams); "e2e_serial" runs
    # each step's copy in, layer and copy out one after the other.
    e2e = e2e_serial = None
    if not args.no_e2e:
        from rotation_w4a4_quantized_b200.pipeline import HostPipeline
        Xh = X.pin_memory()
        Yhs = [torch.empty(Ml, w.N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        h2d_bytes = Xh.numel() * Xh.element_size()
        d2h_bytes = Yhs[0].numel() * Yhs[0].element_size()
        ke = max(1, min(K, 200))
        for _ in range(3):
            Xd.copy_(Xh, non_blocking=True)
            Yhs[0].copy_(layer(Xd), non_blocking=True)
        torch.cuda.synchronize()

        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(ke)]
        for i in range(ke):
            flush.zero_()
            eev[i][0].record(stream)
            Xd.copy_(Xh, non_blocking=True)
            Yhs[0].copy_(layer(Xd), non_blocking=True)
            eev[i][1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s_ms = slowest_rank_ms(sum(a.elapsed_time(b) for a, b in eev)) / ke
        e2e_serial = {"value": job_rate(s_ms) / 1e12, "unit": "TOPS",
                      "ms_per_step": s_ms, "steps": ke, "h2d_bytes_per_step": h2d_bytes,
                      "d2h_bytes_per_step": d2h_bytes}

        pipe = HostPipeline(layer, Ml, w.K, device=dev, depth=2)
        pipe.run([Xh] * 4, [Yhs[i % 2] for i in range(4)])       # warm-up
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        p0.record(stream)
        pipe.run([Xh] * ke, [Yhs[i % 2] for i in range(ke)])
        stream.wait_stream(pipe.d2h)
        p1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_ms = slowest_rank_ms(p0.elapsed_time(p1)) / ke
        e2e = {"value": job_rate(e_ms) / 1e12, "unit": "TOPS",
               "ms_per_step": e_ms, "steps": ke, "h2d_bytes_per_step": h2d_bytes,
               "d2h_bytes_per_step": d2h_bytes,
               "how": "HostPipeline: per step, H2D of the activations from pinned host memory, "
                      "the layer, D2H of the bf16 output; consecutive steps overlap on three "
                      "streams (one event pair around all steps)"}

    # reported baseline (not the optimisation target): the unquantised bf16 linear of the same
    # shape through cuBLAS (X @ W^T, as F.linear), timed like the layer: back to back over
    # rotating copies of its operands larger than L2, one event pair around the whole run
    bf16_us = None
    if rank == 0:
        bsets = [(Xd.clone(), Wd.clone(), torch.empty(Ml, w.N, dtype=bf16, device=dev))]
        b_bytes = sum(t.numel() * t.element_size() for t in bsets[0])
        nb = max(3, -(-3 * l2_bytes(dev) // b_bytes))
        bsets += [(Xd.clone(), Wd.clone(), torch.empty(Ml, w.N, dtype=bf16, device=dev))
                  for _ in range(nb - 1)]
        for i in range(3 * nb):
            xb, wb, yb = bsets[i % nb]
            torch.matmul(xb, wb.t(), out=yb)
        kb = max(3 * nb, min(K, 300))
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        torch.cuda._sleep(PRIME_CYCLES)
        a.record(stream)
        for i in range(kb):
            xb, wb, yb = bsets[i % nb]
            torch.matmul(xb, wb.t(), out=yb)
        b_.record(stream)
        b_.synchronize()
        bf16_us = a.elapsed_time(b_) / kb * 1e3
        del bsets

    # context for the GEMM roofline: the library int8 GEMM (cuBLASLt through torch._int_mm,
    # int32 out) at 8192^3 (best of 10 single launches) and at this layer's shape (back to back
    # over rotating operand copies, like the layer)
    int8_lib = None
    if rank == 0:
        int8_lib = int8_library_reference(w, dev, stream, K)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, g, K_pad, X, W, variant=args.variant)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    gemm_kernel = ("mxfp4_gemm_kernel" if mx else "nvfp4_gemm_kernel" if fp4 else "w8a8_gemm_kernel" if int8
                   else "w4a4_gemm_kernel")
    quant_kernel = ("rht_quant_kernel_mx" if mx else "rht_quant_kernel_fp4" if fp4 else "rht_quant_kernel_i8" if int8
                    else "rht_quant_kernel")
    line = {
        "metric": metric_name(args.variant),
        "value": value,
        "unit": "TOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": args.scaling,
        "vs_baseline": None,
        "dtype": "e2m1" if fp4 else "s8",
        "data": "synthetic",
        "config": config,
        "impl": "ours",
        "quant_gbs": quant_gbs,
        "quant_us": quant_avg * 1e3,
        "gemm_us": gemm_avg * 1e3,
        "kernel_times": "quant_us and gemm_us (and both rooflines): average launch duration "
                        "of that kernel alone, launched back to back over rotating operand "
                        "copies larger than L2 (captured once in a CUDA graph, replayed to at "
                        "least K launches), between two CUDA events",
        "kernel_split": None if fused else {
            "ms_per_step": ev_total_ms / K,
            "quant_us": statistics.mean(ev_quant_ms) * 1e3,
            "gemm_us": statistics.mean(ev_gemm_ms) * 1e3,
            "how": "a second run of K steps with CUDA events between the two kernels of every "
                   "step (each event drains the stream, so these times include that drain)"},
        "roofline": {"bound": "tensor", "kernel": gemm_kernel,
                     "achieved": ops / (gemm_avg / 1e3) / 1e12,
                     "peak": int8_peak, "unit": "TFLOP/s",
                     "frac": ops / (gemm_avg / 1e3) / 1e12 / int8_peak,
                     "peak_source": f"{peak_src} bf16 burst {bf16_tflops} x {peak_ratio:g} "
                                    f"({'fp4' if fp4 else 'int8'}/bf16)",
                     "traffic": profiled_traffic(gemm_kernel, args.config)},
        "roofline_quant": {"bound": "hbm", "kernel": quant_kernel, "achieved": quant_gbs,
                           "peak": hbm_gbs, "unit": "GB/s", "frac": quant_gbs / hbm_gbs,
                           "frac_of_8000_nominal": quant_gbs / 8000.0,
                           "peak_source": peak_src,
                           "traffic": profiled_traffic(quant_kernel, args.config)},
        "gpu_launches": 2 * K,
        "clocks": clocks,
        "e2e": e2e,
        "e2e_serial": e2e_serial,
        "cpu_baseline": cpu,
        "int8_library_gemm": int8_lib,
        "bf16_linear": None if bf16_us is None else {
            "what": "unquantised bf16 X @ W^T (cuBLAS) of the same shape, reported baseline",
            "us": bf16_us, "tflops": 2.0 * Ml * w.N * w.K / (bf16_us / 1e6) / 1e12,
            "layer_speedup": bf16_us / (ms_per_step * 1e3)},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
