#!/usr/bin/env python3
"""Benchmark of the sparse-weight decode / prefill path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one decode pass over the seven pruned linear layers of one Llama-7B decoder
layer (q, k, v, o: 4096 x 4096; gate, up: 11008 x 4096; down: 4096 x 11008), fp16
weights from N(0, 0.02) with a 50% per-row magnitude mask, batch 1.  The inputs of q..up
are N(0, 1); the down projection's input is SiLU(g) * u with its smallest 50% of
entries zeroed.  Each linear is one spw_spmv launch (threshold selection fused in), so a
step is 7 launches, replayed from a CUDA graph.  Steps rotate over 4 such layers (about
0.9 GB of compressed weights, 7x the 126 MB L2), so weight bytes come from HBM.

value = algorithmic bytes / time (GB/s): per linear, the values and bitmap words of the
active columns plus the activations read and the outputs written.  Prefill (spw_spmm at
M = 2048) and the dense cuBLAS comparisons are extra keys of the same JSON line.

--impl reference times the fp64 CPU oracle (this path's reference implementation) on
the host, on a bounded sample of the same workload.  N > 1 GPUs run replicas (one
process per GPU via torchrun, no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402  (seeded inputs only)

METRIC = "spMspV HBM GB/s (% of peak) at batch 1; SpMM TFLOP/s at M=2048 vs dense"
LAYERS = ["q", "k", "v", "o", "gate", "up", "down"]
SPARSITY = 0.5
DOWN_ACT_SPARSITY = 0.5
N_ROTATE = 4
WORKLOAD = ("Llama-7B decoder-layer decode, batch 1: 7 pruned linears (q,k,v,o 4096x4096; "
            "gate,up 11008x4096; down 4096x11008), fp16 N(0,0.02) weights, 50% per-row "
            "magnitude mask, TCB v1; q..up inputs N(0,1); down input SiLU(g)*u with the "
            "smallest 50% zeroed; threshold selection fused into spw_spmv")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return (float(d.get("hbm_gbs", 6650.0)), float(d.get("bf16_tflops", 1590.0)),
                float(d.get("bf16_tflops_sustained", 1400.0)), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def measured_traffic():
    """Per-launch DRAM bytes of the decode kernel from the committed ncu summary, or None
    when the kernel source changed since those counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "spmv_decode_step_traffic.json")
    try:
        rec = json.load(open(path))
        src = open(os.path.join(ROOT, rec["kernel_source"]), "rb").read()
    except (OSError, ValueError, KeyError):
        return None
    if hashlib.sha256(src).hexdigest() != rec.get("kernel_source_sha256"):
        return None
    return int(rec["traffic_bytes_per_launch"])


def decode_bytes(W, mask, x, t):
    """Algorithmic bytes of one decode call: values + bitmap words of the active columns,
    activations read, outputs written."""
    N, K = W.shape
    B = x.shape[0]
    xf = x.astype(np.float64)
    keep = (xf != 0) & ~(np.abs(xf) < np.float64(np.float32(t)))
    active = keep.any(axis=0)
    nnz_active = int(mask[:, active].astype(bool).sum())
    return 2 * nnz_active + 8 * (-(-N // 64)) * int(active.sum()) + 2 * B * K + 2 * B * N


def make_layer():
    """[(name, W, mask, x, t)] for the 7 linears of one decoder layer (seeded)."""
    layer = []
    for name in LAYERS:
        N, K = workloads.LLAMA7B_LAYERS[name]
        lin = workloads.pruned_layer(name, N, K, SPARSITY, "bench")
        a = DOWN_ACT_SPARSITY if name == "down" else 0.0
        x, _ = workloads.decode_act(name, 1, K, a, "bench")
        layer.append((name, lin.W, lin.mask, x, 0.0))
    return layer


class _Rotated:
    """A device copy of a compressed weight at a different address (same header)."""

    def __init__(self, base):
        import spmm_tiled_column_b200 as spw
        self._spw = spw
        self.N, self.K, self.hdr = base.N, base.K, base.hdr
        self.buf = base.buf.clone()
        self.ws = base.workspace(1).clone()

    def spmv(self, x, t, act_bits, y):
        return self._spw.spw_spmv(self.hdr, self.buf, x, t, act_bits, y, self.ws)


class Clocks:
    """nvidia-smi sampler around the timed region (SM clock, throttle reasons)."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(self.NAMES, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle arm

def oracle_decode_sample(seconds=12.0, layers=None):
    """Time the fp64 oracle on whole decode steps of the same workload (one thread)."""
    import oracle
    layers = layers if layers is not None else make_layer()
    step_bytes = sum(decode_bytes(W, m, x, t) for _, W, m, x, t in layers)
    # warm the library once on the smallest linear
    name, W, m, x, t = layers[0]
    oracle.spmv(W, m, x, t)
    done, t0 = 0, time.perf_counter()
    while True:
        for _, W, m, x, t in layers:
            oracle.spmv(W, m, x, t)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": round(step_bytes * done / el / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{done} full decode steps (7 linears, batch 1) in {el:.1f} s, "
                      "single-threaded fp64 C oracle"}, el / done


# ------------------------------------------------------------------ GPU arm

def run_ours(args, rank, world, local_rank):
    import torch
    import spmm_tiled_column_b200 as spw

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, tc_sust, peak_src = peaks()

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.float16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.float16)
        return torch.from_numpy(a).to(dev)

    # Consecutive decode launches overlap (programmatic dependent launch): the weights
    # are compressed once here and never written again.
    spw.spw_set_launch_overlap(True)
    layer = make_layer()
    step_bytes = sum(decode_bytes(W, m, x, t) for _, W, m, x, t in layer)
    lin = [[] for _ in range(N_ROTATE)]  # per rotation: (weight, x_dev, y_dev, t)
    for name, W, m, x, t in layer:
        base = spw.SparseLinear(to_dev(W), to_dev(m))
        for r in range(N_ROTATE):
            sl = base if r == 0 else _Rotated(base)
            if r == 0:
                sl.workspace(1)
            xd = to_dev(x)
            yd = torch.empty((1, base.N), dtype=torch.float16, device=dev)
            lin[r].append((sl, xd, yd, t))
    torch.cuda.synchronize()

    def step(r):
        for sl, xd, yd, t in lin[r]:
            sl.spmv(xd, t, None, yd)

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for r in range(N_ROTATE):   # warm up outside capture: attributes, status word
            step(r)
    stream.synchronize()
    graphs = []
    for r in range(N_ROTATE):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(r)
        graphs.append(g)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % N_ROTATE].replay()
    stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with Clocks(local_rank) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(args.steps):
                graphs[i % N_ROTATE].replay()
            e1.record(stream)
        stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if world > 1:
        import torch.distributed as dist
        tt = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    total_bytes = step_bytes * args.steps * world
    gbs = total_bytes / (ms * 1e-3) / 1e9
    per_rank_gbs = gbs / world
    assert spw.spw_last_device_status() == spw.SPW_OK

    # per-linear kernel timing (dominant kernel = spw_spmv) for the roofline, on the
    # launching stream, over graph replays of single linears
    per_linear = {}
    for j, name in enumerate(LAYERS):
        gs = []
        for r in range(N_ROTATE):
            g = torch.cuda.CUDAGraph()
            sl, xd, yd, t = lin[r][j]
            with torch.cuda.graph(g, stream=stream):
                sl.spmv(xd, t, None, yd)
            gs.append(g)
        reps = 50
        with torch.cuda.stream(stream):
            for i in range(8):
                gs[i % N_ROTATE].replay()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(reps):
                gs[i % N_ROTATE].replay()
            b.record(stream)
        stream.synchronize()
        us = a.elapsed_time(b) * 1e3 / reps
        nb = decode_bytes(*layer[j][1:])
        per_linear[name] = {"us": round(us, 3), "GB/s": round(nb / (us * 1e-6) / 1e9, 1),
                            "bytes": int(nb)}
        del gs

    # dense cuBLAS comparison at the same shapes (fp16 in, fp32 accumulate)
    dense = {}
    for j, name in enumerate(LAYERS[:: 1]):
        if name in dense or name in ("k", "v", "up"):
            continue
        N, K = workloads.LLAMA7B_LAYERS[name]
        Ws = [torch.randn((N, K), device=dev, dtype=torch.float16) * 0.02 for _ in range(6)]
        xd = torch.randn((1, K), device=dev, dtype=torch.float16)
        reps = 60
        with torch.cuda.stream(stream):
            for i in range(6):
                torch.nn.functional.linear(xd, Ws[i % 6])
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(reps):
                torch.nn.functional.linear(xd, Ws[i % 6])
            b.record(stream)
        stream.synchronize()
        us = a.elapsed_time(b) * 1e3 / reps
        dense[name] = {"us": round(us, 3), "GB/s": round(2 * N * K / (us * 1e-6) / 1e9, 1),
                       "sparse_us": per_linear[name]["us"],
                       "speedup": round(us / per_linear[name]["us"], 3)}
        del Ws

    # end to end through the public API with host buffers (pinned), eager calls
    e2e = None
    if not args.no_e2e:
        hx = [[torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).pin_memory()
               for _, _, _, x, _ in layer] for _ in range(N_ROTATE)]
        hy = [[torch.empty((1, sl.N), dtype=torch.int16).pin_memory() for sl, _, _, _ in row]
              for row in lin]
        h2d = sum(2 * x.shape[1] for _, _, _, x, _ in layer)
        d2h = sum(2 * sl.N for sl, _, _, _ in lin[0])

        def e2e_step(r):
            for j, (sl, xd, yd, t) in enumerate(lin[r]):
                xd.view(torch.int16).copy_(hx[r][j], non_blocking=True)
                sl.spmv(xd, t, None, yd)
                hy[r][j].copy_(yd.view(torch.int16), non_blocking=True)

        e2e_steps = max(10, min(args.steps, 100))
        with torch.cuda.stream(stream):
            for i in range(3):
                e2e_step(i % N_ROTATE)
        stream.synchronize()
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for i in range(e2e_steps):
                e2e_step(i % N_ROTATE)
            b.record(stream)
        stream.synchronize()
        ems = a.elapsed_time(b)
        if world > 1:
            import torch.distributed as dist
            tt = torch.tensor([ems], dtype=torch.float64, device=dev)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            ems = float(tt.item())
        ebytes = step_bytes * e2e_steps * world
        e2e = {"value": round(ebytes / (ems * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(ems / e2e_steps, 4),
               "how": "per step: 7 x (pinned H2D of x, spw_spmv via the Python binding "
                      "and C-ABI, D2H of y), eager launches on one stream"}

    prefill = None
    try:
        prefill = run_prefill(args, dev, stream, tc_peak, peak_src)
    except Exception as exc:  # the prefill leg must not hide the decode number
        prefill = {"unavailable": f"{type(exc).__name__}: {exc}"[:300]}

    avg_launch_us = ms * 1e3 / (args.steps * len(LAYERS))
    achieved = per_rank_gbs
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4), "traffic": measured_traffic(),
            "traffic_source": "profiles/spmv_decode_step_traffic_llama7b_b1.md (ncu, per launch)",
            "kernel": "spw::spmv_kernel<1>", "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
            "avg_launch_us": round(avg_launch_us, 3),
            "per_linear": per_linear}
    result = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": world, "parallelism": "replicas",
                   "launch_overlap": "programmatic dependent launch between consecutive decode kernels",
                   "l2": f"inputs larger than L2: {N_ROTATE} device copies of the layer rotated "
                         f"({sum(s.buf.numel() for row in lin for s, _, _, _ in row) / 1e9:.2f} GB)"},
        "roofline": roof,
        "gpu_launches": args.steps * len(LAYERS),
        "clocks": clk.summary(),
        "e2e": e2e,
        "dense_cublas_decode": dense,
        "prefill": prefill,
    }
    return result, layer


def run_prefill(args, dev, stream, tc_peak, peak_src):
    import torch
    import spmm_tiled_column_b200 as spw
    M = 2048
    out = {}
    for name in ("q", "gate", "down"):
        N, K = workloads.LLAMA7B_LAYERS[name]
        lin = workloads.pruned_layer(name, N, K, SPARSITY, "bench-prefill")
        W = torch.from_numpy(lin.W.view(np.int16)).to(dev).view(torch.float16)
        mask = torch.from_numpy(lin.mask).to(dev)
        sl = spw.SparseLinear(W, mask)
        X = torch.randn((M, K), device=dev, dtype=torch.float16)
        Y = torch.empty((M, N), device=dev, dtype=torch.float16)
        sl.spmm(X, Y)
        torch.cuda.synchronize()
        reps = 20
        with torch.cuda.stream(stream):
            for _ in range(3):
                sl.spmm(X, Y)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                sl.spmm(X, Y)
            b.record(stream)
        stream.synchronize()
        us = a.elapsed_time(b) * 1e3 / reps
        Wd = W * mask.to(torch.float16)
        with torch.cuda.stream(stream):
            for _ in range(3):
                torch.nn.functional.linear(X, Wd)
            a.record(stream)
            for _ in range(reps):
                torch.nn.functional.linear(X, Wd)
            b.record(stream)
        stream.synchronize()
        dus = a.elapsed_time(b) * 1e3 / reps
        flops = 2.0 * M * N * K
        out[name] = {"M": M, "N": N, "K": K, "us": round(us, 2),
                     "TFLOP/s_executed": round(flops / (us * 1e-6) / 1e12, 1),
                     "TFLOP/s_useful": round(2.0 * M * lin.mask.sum() / (us * 1e-6) / 1e12, 1),
                     "tensor_frac": round(flops / (us * 1e-6) / 1e12 / tc_peak, 4),
                     "dense_cublas_us": round(dus, 2),
                     "dense_cublas_TFLOP/s": round(flops / (dus * 1e-6) / 1e12, 1),
                     "speedup_vs_dense": round(dus / us, 3)}
    out["peak"] = {"TFLOP/s": tc_peak, "source": f"{peak_src} bf16_tflops (fp16 dense rate equals bf16)"}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        steps = max(1, args.steps)
        per_step_s = None
        cpu, per_step_s = oracle_decode_sample(seconds=min(60.0, max(5.0, 0.06 * steps)))
        line = {"impl": "reference", "metric": METRIC, "value": cpu["value"], "unit": "GB/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(per_step_s * 1e3, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": WORKLOAD, "parallelism": "host, 1 thread"},
                "cpu_baseline": cpu,
                "e2e": {"value": cpu["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    result, layer = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1:
        cpu, _ = oracle_decode_sample(seconds=10.0, layers=layer)
        result["cpu_baseline"] = cpu
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
