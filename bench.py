#!/usr/bin/env python3
"""Benchmark of the sparse-weight decode / prefill path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --sweep decode|prefill|taxonomy [--quick] [--out FILE]
    python bench.py --case spmv|spmm|tc|ffn|spmm24|tokens [--layer L] [--batch B] [--act A] [--m M] ...

A step is one decode pass over the seven pruned linear layers of one Llama-7B decoder
layer (q, k, v, o: 4096 x 4096; gate, up: 11008 x 4096; down: 4096 x 11008), fp16
weights from N(0, 0.02) with a 50% per-row magnitude mask, batch 1.  As in a decoder
layer, q, k and v read one input (the attention input) and gate and up read one input
(the FFN input), all N(0, 1); o reads its own N(0, 1) input; the down projection's input
is SiLU(g) * u with its smallest 50% of entries zeroed.  The step is four decode
launches, one per group of linears that share an input: [q, k, v], [o], [gate, up],
[down] (spw_spmv_group; threshold selection fused in), replayed from a CUDA graph.
Steps rotate over 4 device copies of the layer (about 0.9 GB of compressed weights, 7x
the 126 MB L2), so weight bytes come from HBM.

value = algorithmic bytes / time (GB/s): per linear, the values and bitmap words of the
active columns plus the activations read and the outputs written.  Prefill (spw_spmm at
M = 2048, graph-replayed over rotated operands), the dense cuBLAS comparisons (fp32
accumulation, no fp16 reduced-precision reductions), the decode time against a plain
copy of the same bytes (the three-layer-format page's Fig. 5), the bytes per weight
of dense / CSR / TCB storage (its Fig. 3), prefill with per-token index sets and token
grouping (spw_spmm_tokens) and the 2:4 + residual prefill on sparse tensor cores
(spw_spmm24) are extra keys of the same JSON line.

--impl reference times the fp64 CPU oracle (this path's reference implementation) on
one pinned host core: each step is a bounded sample of the same workload (the decode of
one of the layer's linears, in turn).  N > 1 GPUs run replicas (one process per GPU via
torchrun, no collective on the data path).

--sweep times the parity-test configurations that are not bench lines (Llama-7B and
Llama-13B decode and prefill sweeps, the GEMM-taxonomy shapes), one JSON line per point.
--case runs one decode or prefill case in a loop, for profilers (ncu -s/-c select
launches) and quick timing.
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
GROUPS = [["q", "k", "v"], ["o"], ["gate", "up"], ["down"]]
WORKLOAD = ("Llama-7B decoder-layer decode, batch 1: 7 pruned linears (q,k,v,o 4096x4096; "
            "gate,up 11008x4096; down 4096x11008), fp16 N(0,0.02) weights, 50% per-row "
            "magnitude mask, TCB v1; q/k/v share an N(0,1) input, gate/up share an N(0,1) "
            "input, o has its own; down input SiLU(g)*u with the smallest 50% zeroed, decoded "
            "with its activation threshold (only the kept columns' bytes are read); one "
            "grouped decode launch per shared input ([q,k,v],[o],[gate,up],[down]) with the "
            "threshold selection fused in")


L2_BYTES = 126 * 2**20


def run_config(world: int) -> dict:
    """The workload description, identical on both arms."""
    return {"workload": WORKLOAD, "global_batch": world, "parallelism": "replicas",
            "launch_overlap": "programmatic dependent launch between consecutive decode kernels",
            "l2": f"inputs larger than L2: {N_ROTATE} device copies of the layer's compressed "
                  "weights rotated (about 7x the 126 MB L2)"}


def host_cpu_info() -> dict:
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


class pinned_one_core:
    """Run the block on one host core (the first one this process may use)."""

    def __enter__(self):
        self.old = None
        self.core = None
        try:
            self.old = os.sched_getaffinity(0)
            self.core = min(self.old)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            pass
        return self.core

    def __exit__(self, *exc):
        if self.old is not None:
            try:
                os.sched_setaffinity(0, self.old)
            except OSError:
                pass
        return False


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return (float(d.get("hbm_gbs", 6650.0)), float(d.get("bf16_tflops", 1590.0)),
                float(d.get("bf16_tflops_sustained", 1400.0)), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def code_sha256(src: bytes) -> str:
    """sha256 of C/C++ source with comments and whitespace removed (string literals kept),
    so that editing a comment does not invalidate counters taken on the same code."""
    import hashlib
    import re
    tok = re.compile(rb'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"|\'(?:\\.|[^\'\\])*\'', re.S)
    kept = tok.sub(lambda m: m.group(0) if m.group(0)[:1] in (b'"', b"'") else b" ", src)
    return hashlib.sha256(re.sub(rb"\s+", b"", kept)).hexdigest()


def measured_traffic():
    """Per-launch DRAM bytes of the decode kernel from the committed ncu summary, or None
    when the kernel's code (comments aside) changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "spmv_decode_step_traffic.json")
    try:
        rec = json.load(open(path))
        src = open(os.path.join(ROOT, rec["kernel_source"]), "rb").read()
    except (OSError, ValueError, KeyError):
        return None
    if code_sha256(src) != rec.get("kernel_code_sha256"):
        return None
    return int(rec["traffic_bytes_per_launch"])


def job_rate(ms_local: float, bytes_per_step: int, steps: int, world: int, device) -> tuple:
    """Whole-job rate of N replicas: the slowest rank's time (a MAX all-reduce over the
    process group when world > 1) and every rank's bytes.  Returns (ms, GB/s)."""
    ms = float(ms_local)
    if world > 1:
        import torch
        import torch.distributed as dist
        tt = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    return ms, bytes_per_step * steps * world / (ms * 1e-3) / 1e9


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
    """[(name, W, mask, x, t)] for the 7 linears of one decoder layer (seeded); the
    linears of one group share their input array."""
    inputs = {}
    layer = []
    for group in GROUPS:
        for name in group:
            N, K = workloads.LLAMA7B_LAYERS[name]
            lin = workloads.pruned_layer(name, N, K, SPARSITY, "bench")
            if group[0] not in inputs:
                a = DOWN_ACT_SPARSITY if name == "down" else 0.0
                x, tt = workloads.decode_act(name, 1, K, a, "bench", group[0])
                # the down projection runs with its activation threshold (the smallest kept
                # |v|): the same active set as the zeroed input, and the signal that selects
                # the column-fetch decode; the dense-input layers run with threshold 0
                inputs[group[0]] = (x, float(tt[0]) if a > 0 else 0.0)
            x, t = inputs[group[0]]
            layer.append((name, lin.W, lin.mask, x, t))
    return layer


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
    """Time the fp64 oracle on whole decode steps of the same workload (one thread,
    pinned to one host core)."""
    import oracle
    layers = layers if layers is not None else make_layer()
    step_bytes = sum(decode_bytes(W, m, x, t) for _, W, m, x, t in layers)
    info = host_cpu_info()
    with pinned_one_core() as core:
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
            "kind": "oracle", **info, "pinned_core": core,
            "sample": f"{done} full decode steps (7 linears, batch 1) in {el:.1f} s, "
                      f"single-threaded fp64 C oracle on host core {core} of {info['nproc']} "
                      f"({info['cpu_model']})"}, el / done


def reference_arm(args, world):
    """The oracle as it stands, timed on one pinned host core.  Step i is a bounded sample
    of the same workload: the oracle decode of linear i mod 7 of the layer (batch 1)."""
    import oracle
    layers = make_layer()
    info = host_cpu_info()
    with pinned_one_core() as core:
        for i in range(args.warmup):
            _, W, m, x, t = layers[i % len(layers)]
            oracle.spmv(W, m, x, t)
        total, nbytes = 0.0, 0
        for i in range(args.steps):
            _, W, m, x, t = layers[i % len(layers)]
            t0 = time.perf_counter()
            oracle.spmv(W, m, x, t)
            total += time.perf_counter() - t0
            nbytes += decode_bytes(W, m, x, t)
    value = nbytes / total / 1e9
    sample = (f"{args.steps} steps, each the fp64 C oracle's decode of one of the layer's 7 "
              f"linears in turn (batch 1), after {args.warmup} untimed; one thread on host core "
              f"{core} of {info['nproc']} ({info['cpu_model']})")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": run_config(world),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1,
                             "kind": "oracle", "sample": sample, **info, "pinned_core": core},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ GPU arm

def run_ours(args, rank, world, local_rank):
    import torch
    import spmm_tiled_column_b200 as spw

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, tc_sust, peak_src = peaks()
    # the dense cuBLAS bar accumulates in fp32 throughout (no fp16 split-K reductions)
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False

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
    idx = {name: i for i, (name, *_rest) in enumerate(layer)}
    base = [spw.SparseLinear(to_dev(W), to_dev(m)) for _, W, m, _, _ in layer]
    # per rotation, per group: (names, headers, weight buffers, shared input, outputs, ws)
    gdata = []
    for r in range(N_ROTATE):
        per = []
        for group in GROUPS:
            ls = [base[idx[n]] for n in group]
            hdrs = [l.hdr for l in ls]
            bufs = [l.buf if r == 0 else l.buf.clone() for l in ls]
            xd = to_dev(layer[idx[group[0]]][3])
            ys = [torch.empty((1, l.N), dtype=torch.float16, device=dev) for l in ls]
            ws = torch.zeros(max(16, spw.spw_spmv_group_workspace_bytes(hdrs, 1)),
                             dtype=torch.uint8, device=dev)
            per.append((group, hdrs, bufs, xd, ys, ws))
        gdata.append(per)
    torch.cuda.synchronize()

    group_t = [layer[idx[g[0]]][4] for g in GROUPS]  # per-group threshold

    def step(r):
        for gi, (_, hdrs, bufs, xd, ys, ws) in enumerate(gdata[r]):
            spw.spw_spmv_group(hdrs, bufs, [xd] * len(bufs), group_t[gi], None, ys, ws)

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
    ms, gbs = job_rate(e0.elapsed_time(e1), step_bytes, args.steps, world, dev)
    per_rank_gbs = gbs / world
    assert spw.spw_last_device_status() == spw.SPW_OK

    # per-linear kernel timing (dominant kernel = spw_spmv) for the roofline, on the
    # launching stream, over graph replays of single linears
    def time_graphs(make_call, reps=48):
        # one graph chains the call over all rotated copies (kernels back to back, as in
        # the step graph and in the plain-copy and cuBLAS timings); us per call
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(N_ROTATE):
                make_call(r)
        n_rep = max(1, reps // N_ROTATE)
        with torch.cuda.stream(stream):
            for _ in range(2):
                g.replay()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n_rep):
                g.replay()
            b.record(stream)
        stream.synchronize()
        return a.elapsed_time(b) * 1e3 / (n_rep * N_ROTATE)

    # each grouped launch on its own, and each linear as a single-layer launch
    per_group = {}
    for gi, group in enumerate(GROUPS):
        def call(r, gi=gi):
            _, hdrs, bufs, xd, ys, ws = gdata[r][gi]
            spw.spw_spmv_group(hdrs, bufs, [xd] * len(bufs), group_t[gi], None, ys, ws)
        us = time_graphs(call)
        nb = sum(decode_bytes(*layer[idx[n]][1:]) for n in group)
        per_group["+".join(group)] = {"us": round(us, 3), "GB/s": round(nb / (us * 1e-6) / 1e9, 1),
                                      "bytes": int(nb)}
    per_linear = {}
    for gi, group in enumerate(GROUPS):
        for pi, name in enumerate(group):
            j = idx[name]
            ws1 = base[j].workspace(1)
            def call(r, gi=gi, pi=pi, j=j, ws1=ws1):
                _, hdrs, bufs, xd, ys, _ws = gdata[r][gi]
                spw.spw_spmv(hdrs[pi], bufs[pi], xd, group_t[gi], None, ys[pi], ws1)
            us = time_graphs(call)
            nb = decode_bytes(*layer[j][1:])
            per_linear[name] = {"us": round(us, 3), "GB/s": round(nb / (us * 1e-6) / 1e9, 1),
                                "bytes": int(nb)}

    # Column fetch (spw_set_column_fetch): the down launch (50 % of its activations below
    # the threshold) reading only its active columns' bytes, against whole tiles
    dgi = GROUPS.index(["down"])

    def down_call(r):
        _, hdrs, bufs, xd, ys, ws = gdata[r][dgi]
        spw.spw_spmv_group(hdrs, bufs, [xd] * len(bufs), group_t[dgi], None, ys, ws)
    prev_fetch = spw.spw_set_column_fetch(1)
    try:
        fetch_us = time_graphs(down_call)
    finally:
        spw.spw_set_column_fetch(prev_fetch)
    down_bytes = decode_bytes(*layer[idx["down"]][1:])
    column_fetch = {"down_whole_tiles_us": per_group["down"]["us"], "down_column_fetch_us": round(fetch_us, 3),
                    "down_column_fetch_GB/s": round(down_bytes / (fetch_us * 1e-6) / 1e9, 1),
                    "how": "spw_set_column_fetch(1): the decode copies only the 16-byte chunks of "
                           "active columns (default 0: whole tiles)"}
    assert spw.spw_last_device_status() == spw.SPW_OK

    # Fused FFN activation (spw_spmv_ffn): the gate and up decode plus h = SiLU(g) * u and
    # its column set in one launch, against the same work as separate launches (grouped
    # decode, torch's SiLU and product, spw_select_threshold).  The threshold is the
    # median |h| of this input, so about half of the down projection's columns are kept.
    gu = GROUPS.index(["gate", "up"])
    _, hdrs_gu, _, xd_gu, _, _ = gdata[0][gu]
    fws = [torch.zeros(spw.spw_spmv_ffn_workspace_bytes(hdrs_gu[0], hdrs_gu[1], 1), dtype=torch.uint8,
                       device=dev) for _ in range(N_ROTATE)]
    h_out = torch.empty((1, hdrs_gu[0].N), dtype=torch.float16, device=dev)
    bits_out = torch.empty(((hdrs_gu[0].N + 31) // 32 + 3,), dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        h0, _ = spw.spw_spmv_ffn(hdrs_gu[0], gdata[0][gu][2][0], hdrs_gu[1], gdata[0][gu][2][1], xd_gu,
                                 0.0, h_out, bits_out, fws[0])
    stream.synchronize()
    t_ffn = float(h0.float().abs().median().item())

    def fused(r):
        _, hdrs, bufs, xd, _, _ = gdata[r][gu]
        spw.spw_spmv_ffn(hdrs[0], bufs[0], hdrs[1], bufs[1], xd, t_ffn, h_out, bits_out, fws[r])

    def unfused(r):
        _, hdrs, bufs, xd, ys, ws = gdata[r][gu]
        spw.spw_spmv_group(hdrs, bufs, [xd, xd], 0.0, None, ys, ws)
        torch.mul(torch.nn.functional.silu(ys[0]), ys[1], out=h_out)
        spw.spw_select_threshold(h_out, t_ffn, bits_out)

    fused_us = time_graphs(fused)
    unfused_us = time_graphs(unfused)
    gu_bytes = sum(decode_bytes(*layer[idx[n]][1:]) for n in ("gate", "up"))
    ffn_fused = {"us": round(fused_us, 3), "GB/s": round(gu_bytes / (fused_us * 1e-6) / 1e9, 1),
                 "separate_launches_us": round(unfused_us, 3),
                 "speedup": round(unfused_us / fused_us, 3), "threshold": round(t_ffn, 5),
                 "how": "spw_spmv_ffn (gate+up decode, h = SiLU(g)*u, column set of h) vs "
                        "spw_spmv_group + torch silu/mul + spw_select_threshold; graph replays"}
    assert spw.spw_last_device_status() == spw.SPW_OK

    # The decoder layer's step with the fused FFN activation: [q,k,v], [o], then the
    # gate/up pair emits h and its column set, which the down projection consumes (its
    # input is h of this layer rather than the synthetic SiLU(g)*u of the main step).
    dn = GROUPS.index(["down"])
    h_host = h_out.view(torch.int16).cpu().numpy().view(np.float16)
    down_j = idx["down"]
    ffn_step_bytes = (sum(decode_bytes(*layer[idx[n]][1:]) for n in ("q", "k", "v", "o", "gate", "up"))
                      + decode_bytes(layer[down_j][1], layer[down_j][2], h_host, t_ffn))

    def ffn_step(r):
        for gi in (GROUPS.index(["q", "k", "v"]), GROUPS.index(["o"])):
            _, hdrs, bufs, xd, ys, ws = gdata[r][gi]
            spw.spw_spmv_group(hdrs, bufs, [xd] * len(bufs), 0.0, None, ys, ws)
        fused(r)
        _, hdrs, bufs, _, ys, ws = gdata[r][dn]
        spw.spw_spmv_group(hdrs, bufs, [h_out], t_ffn, [bits_out], ys, ws)

    ffn_step_us = time_graphs(ffn_step)
    ffn_fused["layer_step"] = {
        "us": round(ffn_step_us, 3), "GB/s": round(ffn_step_bytes / (ffn_step_us * 1e-6) / 1e9, 1),
        "bytes": int(ffn_step_bytes),
        "how": "[q,k,v], [o], spw_spmv_ffn(gate, up), down on h with its column set; 4 launches"}
    assert spw.spw_last_device_status() == spw.SPW_OK

    # dense cuBLAS comparison at the same shapes (fp16 in, fp32 accumulate)
    dense = {}
    for j, name in enumerate(LAYERS[:: 1]):
        if name in dense or name in ("k", "v", "up"):
            continue
        N, K = workloads.LLAMA7B_LAYERS[name]
        Ws = [torch.randn((N, K), device=dev, dtype=torch.float16) * 0.02 for _ in range(6)]
        xd = torch.randn((1, K), device=dev, dtype=torch.float16)
        outs = [torch.empty((1, N), device=dev, dtype=torch.float16) for _ in range(6)]
        # the same chained-graph timing as the sparse launches: six rotated weights (> L2)
        us = graph_us([(lambda i=i: torch.matmul(xd, Ws[i].t(), out=outs[i])) for i in range(6)],
                      stream)
        dense[name] = {"us": round(us, 3), "GB/s": round(2 * N * K / (us * 1e-6) / 1e9, 1),
                       "sparse_us": per_linear[name]["us"],
                       "speedup": round(us / per_linear[name]["us"], 3)}
        del Ws

    # the same step done densely by cuBLAS, as an engine would: fused qkv and gate/up
    # weights, four GEMVs per step, graph-replayed over two rotated copies (> L2 each)
    dense_shapes = [(3 * 4096, 4096), (4096, 4096), (2 * 11008, 4096), (4096, 11008)]
    dW = [[torch.randn(sh, device=dev, dtype=torch.float16) * 0.02 for sh in dense_shapes]
          for _ in range(2)]
    dX = [torch.randn((1, sh[1]), device=dev, dtype=torch.float16) for sh in dense_shapes]
    dY = [torch.empty((1, sh[0]), device=dev, dtype=torch.float16) for sh in dense_shapes]
    dgs = []
    for r in range(2):
        with torch.cuda.stream(stream):
            for w, x, y in zip(dW[r], dX, dY):
                torch.matmul(x, w.t(), out=y)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for w, x, y in zip(dW[r], dX, dY):
                torch.matmul(x, w.t(), out=y)
        dgs.append(g)
    with torch.cuda.stream(stream):
        for i in range(6):
            dgs[i % 2].replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(40):
            dgs[i % 2].replay()
        b.record(stream)
    stream.synchronize()
    dense_step_us = a.elapsed_time(b) * 1e3 / 40
    dense_bytes = sum(2 * n * k for n, k in dense_shapes)
    dense_step = {"us": round(dense_step_us, 2),
                  "GB/s": round(dense_bytes / (dense_step_us * 1e-6) / 1e9, 1),
                  "sparse_step_us": round(ms * 1e3 / args.steps, 2),
                  "speedup": round(dense_step_us / (ms * 1e3 / args.steps), 3),
                  "how": "cuBLAS (torch.matmul) on the dense weights of the same layer: "
                         "fused qkv 12288x4096, o, fused gate/up 22016x4096, down; batch 1"}
    del dW, dgs

    # end to end through the public API with host buffers (pinned), eager calls: per step
    # one copy of the step's inputs to the device, the four grouped decodes through
    # prepared DecodeGroup calls, and one copy of all outputs back
    e2e = None
    if not args.no_e2e:
        in_k = [int(layer[idx[g[0]]][3].shape[1]) for g in GROUPS]
        out_n = [[int(h.N) for h in hdrs] for _, hdrs, *_ in gdata[0]]
        hx = torch.from_numpy(np.concatenate([np.ascontiguousarray(layer[idx[g[0]]][3][0]).view(np.int16)
                                              for g in GROUPS])).pin_memory()
        hy = torch.empty((sum(sum(n) for n in out_n),), dtype=torch.int16).pin_memory()
        dx = [torch.empty((sum(in_k),), dtype=torch.float16, device=dev) for _ in range(N_ROTATE)]
        dy = [torch.empty((hy.numel(),), dtype=torch.float16, device=dev) for _ in range(N_ROTATE)]
        e2e_calls = []
        for r in range(N_ROTATE):
            calls, xo, yo = [], 0, 0
            for gi, (_, hdrs, bufs, _xd, _ys, ws) in enumerate(gdata[r]):
                xv = dx[r][xo:xo + in_k[gi]].view(1, -1)
                yv = []
                for n in out_n[gi]:
                    yv.append(dy[r][yo:yo + n].view(1, -1))
                    yo += n
                calls.append((spw.DecodeGroup(hdrs, bufs, 1, ws), [xv] * len(bufs), yv, group_t[gi]))
                xo += in_k[gi]
            e2e_calls.append(calls)
        h2d = 2 * sum(in_k)
        d2h = 2 * hy.numel()

        def e2e_step(r):
            dx[r].view(torch.int16).copy_(hx, non_blocking=True)
            for call, xs, ys, tg in e2e_calls[r]:
                call(xs, ys, threshold=tg)
            hy.copy_(dy[r].view(torch.int16), non_blocking=True)

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
        ems, egbs = job_rate(a.elapsed_time(b), step_bytes, e2e_steps, world, dev)
        e2e = {"value": round(egbs, 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(ems / e2e_steps, 4),
               "how": "per step: one pinned H2D of the 4 group inputs, the 4 grouped decodes "
                      "through prepared DecodeGroup calls (Python binding -> C-ABI "
                      "spw_spmv_group), one D2H of the 7 outputs; eager launches on one stream"}

    prefill, prefill_detail = None, None
    try:
        prefill, prefill_detail = run_prefill(args, dev, stream, tc_peak, peak_src)
    except Exception as exc:  # the prefill leg must not hide the decode number
        prefill = {"unavailable": f"{type(exc).__name__}: {exc}"[:300]}
    try:
        prefill_tokens = run_prefill_tokens(dev, stream)
    except Exception as exc:
        prefill_tokens = {"unavailable": f"{type(exc).__name__}: {exc}"[:300]}
    try:
        prefill24 = run_prefill24(dev, stream, tc_peak)
    except Exception as exc:
        prefill24 = {"unavailable": f"{type(exc).__name__}: {exc}"[:300]}

    # Decode time against a plain copy of the same bytes (the launch's compressed
    # weights), per grouped launch: the three-layer-format page's comparison of global
    # memory access with on-chip decoding (Fig. 5).
    decode_vs_read = {}
    for gi, group in enumerate(GROUPS):
        _, hdrs, _, _, _, _ = gdata[0][gi]
        nb = sum(int(h.bytes_total) for h in hdrs)
        cus = copy_us(nb, dev, stream)
        key = "+".join(group)
        decode_vs_read[key] = {"weight_bytes": nb, "copy_us": round(cus, 3),
                               "decode_us": per_group[key]["us"],
                               "decode_over_copy": round(per_group[key]["us"] / cus, 3)}
    storage = storage_bytes_per_weight(dev)

    avg_launch_us = ms * 1e3 / (args.steps * len(GROUPS))
    achieved = per_rank_gbs
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4), "traffic": measured_traffic(),
            "traffic_source": "profiles/spmv_decode_step_traffic.json (ncu dram bytes per launch; "
                              "null when the decode kernel's code changed since the capture)",
            "kernel": "spw::spmv_kernel<1>", "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
            "avg_launch_us": round(avg_launch_us, 3),
            "per_group_launch": per_group,
            "per_linear_single_launch": per_linear}
    result = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": run_config(world),
        "roofline": roof,
        "gpu_launches": args.steps * len(GROUPS),
        "clocks": clk.summary(),
        "e2e": e2e,
        "dense_cublas_decode": dense,
        "ffn_fused": ffn_fused,
        "column_fetch": column_fetch,
        "dense_cublas_step": dense_step,
        "prefill": prefill,
        "prefill_detail": prefill_detail,
        "prefill_tokens": prefill_tokens,
        "prefill_2of4_residual": prefill24,
        "decode_vs_plain_copy": decode_vs_read,
        "storage_bytes_per_weight": storage,
    }
    return result, layer


def graph_us(calls, stream, reps=20, warm=3):
    """Median microseconds per call: one CUDA graph replays calls[0..R-1] (R rotated
    operand sets), timed with CUDA events on the launching stream."""
    import torch
    R = len(calls)
    with torch.cuda.stream(stream):
        for c in calls:
            c()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c()
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g.replay()
    times = []
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g.replay()
            b.record(stream)
        stream.synchronize()
        times.append(a.elapsed_time(b) * 1e3 / R)
    del g
    return float(statistics.median(times))


def run_prefill(args, dev, stream, tc_peak, peak_src):
    """spw_spmm at M = 2048 on the q, gate and down shapes against cuBLAS on the dense
    masked weight, both replayed from CUDA graphs over 3 rotated operand sets (weights,
    X and Y together exceed L2).  Returns (flat record, per-shape detail)."""
    import torch
    import spmm_tiled_column_b200 as spw
    M, R = 2048, 3
    flat, detail = {"M": M}, {}
    for name in ("q", "gate", "down"):
        N, K = workloads.LLAMA7B_LAYERS[name]
        lin = workloads.pruned_layer(name, N, K, SPARSITY, "bench-prefill")
        W = torch.from_numpy(lin.W.view(np.int16)).to(dev).view(torch.float16)
        mask = torch.from_numpy(lin.mask).to(dev)
        sl = spw.SparseLinear(W, mask)
        bufs = [sl.buf] + [sl.buf.clone() for _ in range(R - 1)]
        g = torch.Generator(device=dev).manual_seed(2048 + N + K)
        Xs = [torch.randn((M, K), device=dev, dtype=torch.float16, generator=g) for _ in range(R)]
        Ys = [torch.empty((M, N), device=dev, dtype=torch.float16) for _ in range(R)]
        need = spw.spw_spmm_workspace_bytes(sl.hdr, M)
        wss = [torch.zeros(need, dtype=torch.uint8, device=dev) if need else None for _ in range(R)]
        us = graph_us([(lambda r=r: spw.spw_spmm(sl.hdr, bufs[r], Xs[r], Ys[r], wss[r]))
                       for r in range(R)], stream)
        assert spw.spw_last_device_status() == spw.SPW_OK
        Wd0 = W * mask.to(torch.float16)
        Wds = [Wd0] + [Wd0.clone() for _ in range(R - 1)]
        dus = graph_us([(lambda r=r: torch.matmul(Xs[r], Wds[r].t(), out=Ys[r])) for r in range(R)],
                       stream)
        flops = 2.0 * M * N * K
        ex = flops / (us * 1e-6) / 1e12
        detail[name] = {"M": M, "N": N, "K": K, "us": round(us, 2),
                        "TFLOP/s_executed": round(ex, 1),
                        "TFLOP/s_useful": round(2.0 * M * int(lin.mask.sum()) / (us * 1e-6) / 1e12, 1),
                        "tensor_frac": round(ex / tc_peak, 4), "dense_cublas_us": round(dus, 2),
                        "dense_cublas_TFLOP/s": round(flops / (dus * 1e-6) / 1e12, 1),
                        "speedup_vs_dense": round(dus / us, 3)}
        flat.update({f"{name}_us": round(us, 2), f"{name}_tflops_executed": round(ex, 1),
                     f"{name}_tensor_frac": round(ex / tc_peak, 4),
                     f"{name}_cublas_us": round(dus, 2), f"{name}_vs_cublas": round(dus / us, 3)})
        del bufs, Xs, Ys, Wds, Wd0, sl, wss
        torch.cuda.empty_cache()
    detail["peak"] = {"TFLOP/s": tc_peak,
                      "source": f"{peak_src} bf16_tflops (fp16 dense rate equals bf16)",
                      "how": "graph replays over 3 rotated operand sets; cuBLAS via torch.matmul "
                             "with fp16 reduced-precision reductions disabled"}
    flat["peak_tflops"] = tc_peak
    return flat, detail


def run_prefill_tokens(dev, stream):
    """spw_spmm_tokens (per-token index sets, token grouping; "Reduced Matrix
    Multiplication" §6.1-§6.2) at M = 2048 on the down shape: tokens from D domains that
    each use a random half of the 64-column channel blocks, SiLU(g) * u values, threshold
    0.3.  Against spw_spmm and cuBLAS on the same thresholded input (no skipping); graph
    replays over 3 rotated operand sets."""
    import torch
    import spmm_tiled_column_b200 as spw
    M, R, t, name = 2048, 3, 0.3, "down"
    N, K = workloads.LLAMA7B_LAYERS[name]
    lin = workloads.pruned_layer(name, N, K, SPARSITY, "bench-tokens")
    W = torch.from_numpy(lin.W.view(np.int16)).to(dev).view(torch.float16)
    mask = torch.from_numpy(lin.mask).to(dev)
    sl = spw.SparseLinear(W, mask)
    bufs = [sl.buf] + [sl.buf.clone() for _ in range(R - 1)]
    Wd0 = W * mask.to(torch.float16)
    Wds = [Wd0] + [Wd0.clone() for _ in range(R - 1)]
    plan = spw.spw_spmm_tokens_plan(sl.hdr, M)
    out = {"layer": f"{name} {N}x{K}", "M": M, "threshold": t, "token_tile": plan["token_tile"]}
    for D in (1, 4):
        Xs, Xts = [], []
        for r in range(R):
            X, _ = workloads.domain_tokens(M, K, D, 0.5, "bench-tokens", r, silu=True)
            Xd = _dev(X)
            Xs.append(Xd)
            keep = (Xd != 0) & ~(Xd.abs() < t)
            Xts.append(torch.where(keep, Xd, torch.zeros_like(Xd)))
        Ys = [torch.empty((M, N), device=dev, dtype=torch.float16) for _ in range(R)]
        wss = [torch.zeros(plan["workspace_bytes"], dtype=torch.uint8, device=dev) for _ in range(R)]
        us = graph_us([(lambda r=r: spw.spw_spmm_tokens(sl.hdr, bufs[r], Xs[r], t, Ys[r], wss[r]))
                       for r in range(R)], stream)
        gws = [torch.empty(spw.spw_group_tokens_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
               for _ in range(R)]
        gus = graph_us([(lambda r=r: spw.spw_group_tokens(Xs[r], t, plan["token_tile"], gws[r]))
                        for r in range(R)], stream)
        _, _, tsig = spw.spw_group_tokens(Xs[0], t, plan["token_tile"], gws[0])
        ts = tsig.cpu().numpy().view(np.uint64)
        visited = [sum(bin(int(v)).count("1") for v in row) for row in ts]
        swss = [torch.zeros(max(spw.spw_spmm_workspace_bytes(sl.hdr, M), 16), dtype=torch.uint8,
                            device=dev) for _ in range(R)]
        sus = graph_us([(lambda r=r: spw.spw_spmm(sl.hdr, bufs[r], Xts[r], Ys[r], swss[r]))
                        for r in range(R)], stream)
        dus = graph_us([(lambda r=r: torch.matmul(Xts[r], Wds[r].t(), out=Ys[r])) for r in range(R)],
                       stream)
        assert spw.spw_last_device_status() == spw.SPW_OK
        nk = -(-K // 64)
        out[f"domains_{D}"] = {
            "us": round(us, 2), "grouping_us": round(gus, 2),
            "k_tiles_visited_per_token_tile": visited, "k_tiles": nk,
            "spw_spmm_same_input_us": round(sus, 2), "dense_cublas_same_input_us": round(dus, 2),
            "speedup_vs_spw_spmm": round(sus / us, 3), "speedup_vs_dense": round(dus / us, 3)}
        del Xs, Xts, Ys, wss, gws, swss
    out["how"] = ("spw_spmm_tokens = grouping (signature, rank, gather of x~) + the product over "
                  "each token tile's k-tiles; the kernel time follows the longest k-tile list")
    del bufs, Wds, Wd0, sl
    torch.cuda.empty_cache()
    return out


def run_prefill24(dev, stream, tc_peak):
    """spw_spmm24 (2:4 part on tcgen05.mma.sp + TCB residual; the three-layer-format
    page's layers (i) and (iii)) at M = 2048 on the q shape for three masks: the 50 %
    magnitude mask (residual = every kept weight beyond two per group of four), an exact
    2:4 mask (no residual) and 2:4 plus 0.5 % of the input channels kept whole (residual
    in those columns).  Against spw_spmm on the same mask and cuBLAS on the dense masked
    weight; graph replays over 3 rotated operand sets."""
    import torch
    import spmm_tiled_column_b200 as spw
    M, R, name = 2048, 3, "q"
    N, K = workloads.LLAMA7B_LAYERS[name]
    layer = workloads.pruned_layer(name, N, K, SPARSITY, "bench-24")
    masks = {"magnitude_50": layer.mask,
             "exact_2of4": workloads.structured24_mask(N, K, "bench-24", count=2),
             "2of4_plus_dense_channels_0.5pct": workloads.structured24_mask(
                 N, K, "bench-24", count=2, dense_channels=0.005)}
    W = _dev(layer.W)
    g = torch.Generator(device=dev).manual_seed(24)
    Xs = [torch.randn((M, K), device=dev, dtype=torch.float16, generator=g) for _ in range(R)]
    Ys = [torch.empty((M, N), device=dev, dtype=torch.float16) for _ in range(R)]
    out = {"layer": f"{name} {N}x{K}", "M": M}
    for key, mask in masks.items():
        md = _dev(mask)
        l24 = spw.SparseLinear24(W, md)
        sl = spw.SparseLinear(W, md)
        s24s = [l24.s24] + [l24.s24.clone() for _ in range(R - 1)]
        brs = [l24.buf_r] + [l24.buf_r.clone() for _ in range(R - 1)]
        need = spw.spw_spmm24_workspace_bytes(l24.hdr_r, M)
        wss = [torch.zeros(max(need, 16), dtype=torch.uint8, device=dev) for _ in range(R)]
        us24 = graph_us([(lambda r=r: spw.spw_spmm24(l24.hdr_r, brs[r], s24s[r], Xs[r], Ys[r], wss[r]))
                         for r in range(R)], stream)
        bufs = [sl.buf] + [sl.buf.clone() for _ in range(R - 1)]
        sneed = spw.spw_spmm_workspace_bytes(sl.hdr, M)
        swss = [torch.zeros(max(sneed, 16), dtype=torch.uint8, device=dev) for _ in range(R)]
        us = graph_us([(lambda r=r: spw.spw_spmm(sl.hdr, bufs[r], Xs[r], Ys[r], swss[r]))
                       for r in range(R)], stream)
        Wd0 = W * md.to(torch.float16)
        Wds = [Wd0] + [Wd0.clone() for _ in range(R - 1)]
        dus = graph_us([(lambda r=r: torch.matmul(Xs[r], Wds[r].t(), out=Ys[r])) for r in range(R)],
                       stream)
        assert spw.spw_last_device_status() == spw.SPW_OK
        nnz = int(mask.sum())
        nnz_r = int(l24.hdr_r.nnz)
        hr = l24.hdr_r
        tp = l24.buf_r[hr.off_tileptr:hr.off_tileptr + 4 * (hr.n_strips * hr.n_ktiles + 1)]
        tp = tp.view(torch.int32).cpu().numpy().astype(np.int64)
        nonempty = (np.diff(tp).reshape(hr.n_strips, hr.n_ktiles) > 0)
        pairs = nonempty.reshape(-1, 2, hr.n_ktiles).any(axis=1) if hr.n_strips % 2 == 0 else nonempty
        out[key] = {"density": round(nnz / (N * K), 4), "residual_share": round(nnz_r / max(nnz, 1), 4),
                    "k_steps_with_residual": round(float(pairs.mean()), 4),
                    "us": round(us24, 2), "TFLOP/s_useful": round(2.0 * M * nnz / (us24 * 1e-6) / 1e12, 1),
                    "dense_equivalent_tensor_frac": round(2.0 * M * N * K / (us24 * 1e-6) / 1e12 / tc_peak, 4),
                    "spw_spmm_us": round(us, 2), "dense_cublas_us": round(dus, 2),
                    "speedup_vs_spw_spmm": round(us / us24, 3), "speedup_vs_dense": round(dus / us24, 3)}
        del l24, sl, s24s, brs, wss, bufs, swss, Wds, Wd0, md
        torch.cuda.empty_cache()
    out["how"] = ("2:4 part: two tcgen05.mma.sp (K = 32) per 64-column k-step; residual: TCB decode "
                  "and dense MMA into the same accumulator, skipped for k-steps without residual "
                  "weights; at most 256 tokens per tile (tensor memory also holds the metadata)")
    return out


def storage_bytes_per_weight(dev):
    """Bytes per weight slot of a 4096 x 4096 layer stored dense (fp16), as CSR (fp16
    values, int32 column indices, int32 row pointers), as CSR with 16-bit column indices,
    and as TCB v1 (bytes_total from spw_format_query), at 40-80 % magnitude pruning: the
    three-layer-format page's storage comparison (Fig. 3) for this format."""
    import torch
    import spmm_tiled_column_b200 as spw
    N = K = 4096
    W = workloads.weight(N, K, "storage")
    out = {}
    for s in (0.4, 0.5, 0.6, 0.7, 0.8):
        mask = workloads.magnitude_mask(W, s)
        nnz = int(np.count_nonzero(mask))
        nbytes, _ = spw.spw_format_query(torch.from_numpy(mask).to(dev))
        out[f"{int(s * 100)}%"] = {"dense": 2.0,
                                   "csr_int32": round((6 * nnz + 4 * (N + 1)) / (N * K), 4),
                                   "csr_int16": round((4 * nnz + 4 * (N + 1)) / (N * K), 4),
                                   "tcb_v1": round(nbytes / (N * K), 4)}
    return out


def copy_us(nbytes, dev, stream):
    """Time of a plain device-to-device copy of nbytes (cudaMemcpyAsync through torch:
    reads nbytes and writes nbytes), over rotated buffers larger than L2."""
    import torch
    n = max(16, nbytes)
    R = max(2, -(-3 * L2_BYTES // (2 * n)))
    src = [torch.ones(n, dtype=torch.uint8, device=dev) for _ in range(R)]
    dst = [torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(R)]
    us = graph_us([(lambda r=r: dst[r].copy_(src[r])) for r in range(R)], stream)
    del src, dst
    return us


# ------------------------------------------------------------------ sweeps (--sweep)

def _dev(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.float16)
    return torch.from_numpy(a).cuda()


def _copies(nbytes: int, cap: int = 24) -> int:
    return max(2, min(cap, -(-3 * L2_BYTES // max(nbytes, 1))))


class _SweepLayer:
    """One pruned weight on the device: rotated compressed copies for the sparse side and
    dense masked copies for cuBLAS, each set together larger than 3x the L2."""

    def __init__(self, W: np.ndarray, mask: np.ndarray, dense: bool = True):
        import torch
        import spmm_tiled_column_b200 as spw
        self.W, self.mask = W, mask
        self.N, self.K = W.shape
        self.lin = spw.SparseLinear(_dev(W), _dev(mask))
        R = _copies(self.lin.buf.numel())
        self.bufs = [self.lin.buf] + [self.lin.buf.clone() for _ in range(R - 1)]
        self.dense = None
        if dense:
            d0 = _dev(np.where(mask.astype(bool), W, np.float16(0)).astype(np.float16))
            self.dense = [d0] + [d0.clone() for _ in range(_copies(d0.numel() * 2) - 1)]
        torch.cuda.synchronize()


def _sweep_decode_point(layer, x, t, stream, act_bits=None) -> dict:
    import torch
    import spmm_tiled_column_b200 as spw
    B = x.shape[0]
    xd = _dev(x)
    ws = [torch.zeros(max(16, spw.spw_spmv_workspace_bytes(layer.lin.hdr, B)), dtype=torch.uint8,
                      device="cuda") for _ in layer.bufs]
    ys = [torch.empty((B, layer.N), dtype=torch.float16, device="cuda") for _ in layer.bufs]
    us = graph_us([(lambda r=r: spw.spw_spmv(layer.lin.hdr, layer.bufs[r], xd, t, act_bits, ys[r],
                                             ws[r])) for r in range(len(layer.bufs))], stream)
    assert spw.spw_last_device_status() == spw.SPW_OK
    out = {"sparse_us": round(us, 3)}
    if B >= 4:  # the tensor-core decode path as well
        need = spw.spw_spmv_tc_workspace_bytes(layer.lin.hdr, B)
        tws = [torch.zeros(max(16, need), dtype=torch.uint8, device="cuda") for _ in layer.bufs]
        out["tc_us"] = round(graph_us([(lambda r=r: spw.spw_spmv_tc(
            layer.lin.hdr, layer.bufs[r], xd, t, act_bits, ys[r], tws[r]))
            for r in range(len(layer.bufs))], stream), 3)
        assert spw.spw_last_device_status() == spw.SPW_OK
    if layer.dense is not None:
        yd = [torch.empty((B, layer.N), dtype=torch.float16, device="cuda") for _ in layer.dense]
        dus = graph_us([(lambda r=r: torch.matmul(xd, layer.dense[r].t(), out=yd[r]))
                        for r in range(len(layer.dense))], stream)
        out.update({"dense_us": round(dus, 3), "speedup": round(dus / us, 3)})
    return out


def _sweep_prefill_point(layer, M, stream) -> dict:
    import torch
    import spmm_tiled_column_b200 as spw
    X = [_dev(workloads.normal_act(M, layer.K, "sweep-prefill", M, layer.K, r)) for r in range(2)]
    Y = [torch.empty((M, layer.N), dtype=torch.float16, device="cuda") for _ in range(2)]
    us = graph_us([(lambda r=r: spw.spw_spmm(layer.lin.hdr, layer.bufs[r % len(layer.bufs)], X[r],
                                             Y[r])) for r in range(2)], stream, reps=10)
    assert spw.spw_last_device_status() == spw.SPW_OK
    out = {"sparse_us": round(us, 2)}
    if layer.dense is not None:
        dus = graph_us([(lambda r=r: torch.matmul(X[r], layer.dense[r % len(layer.dense)].t(),
                                                  out=Y[r])) for r in range(2)], stream, reps=10)
        out.update({"dense_us": round(dus, 2), "speedup": round(dus / us, 3)})
    return out


def _emit(rec: dict, fh):
    line = json.dumps(rec)
    print(line, flush=True)
    if fh:
        fh.write(line + "\n")
        fh.flush()


def sweep_decode(quick: bool, fh, stream):
    """Llama-7B linears (q, gate, down) at 50 % and Llama-13B linears at 40-80 % weight
    sparsity, crossed with activation sparsity (the smallest floor(a K) entries of every
    batch row zeroed) and batch B in {1, 4, 16}; each point also reports the decode time
    against a plain copy of the compressed bytes (Fig. 5 of the three-layer-format page)."""
    import torch
    hbm = peaks()[0]
    cases = [("7b", n, workloads.LLAMA7B_LAYERS[n], [0.5], [0.0, 0.3, 0.5, 0.7])
             for n in ("q", "gate", "down")]
    s13 = [0.5] if quick else [0.4, 0.5, 0.6, 0.7, 0.8]
    cases += [("13b", n, sh, s13, [0.0, 0.5, 0.9] if not quick else [0.0, 0.5])
              for n, sh in workloads.LLAMA13B_SHAPES.items()]
    batches = [1, 16] if quick else [1, 4, 16]
    for fam, name, (N, K), sps, acts in cases:
        W = workloads.weight(N, K, "sweep", fam, name)
        for s in sps:
            mask = workloads.magnitude_mask(W, s)
            layer = _SweepLayer(W, mask)
            cp_us = copy_us(int(layer.lin.hdr.bytes_total), "cuda", stream)
            for B in batches:
                for a in acts:
                    x, t = workloads.decode_act(name, B, K, a, "sweep", fam, B)
                    r = _sweep_decode_point(layer, x, 0.0, stream)
                    byts = decode_bytes(W, mask, x, 0.0)
                    r.update({"kind": "decode", "family": fam, "layer": name, "N": N, "K": K,
                              "sparsity": s, "act_sparsity": a, "B": B, "bytes": byts,
                              "GB/s": round(byts / r["sparse_us"] / 1e3, 1),
                              "hbm_frac": round(byts / r["sparse_us"] / 1e3 / hbm, 4),
                              "copy_us": round(cp_us, 3),
                              "decode_over_copy": round(r["sparse_us"] / cp_us, 3)})
                    _emit(r, fh)
            del layer
            torch.cuda.empty_cache()


def sweep_prefill(quick: bool, fh, stream):
    """The same shapes at 50/60/70 % weight sparsity and M in {512, 2048}."""
    import torch
    tc = peaks()[1]
    shapes = [("7b", n, workloads.LLAMA7B_LAYERS[n]) for n in ("q", "gate", "down")]
    if not quick:
        shapes += [("13b", n, sh) for n, sh in workloads.LLAMA13B_SHAPES.items()]
    for fam, name, (N, K) in shapes:
        W = workloads.weight(N, K, "sweep", fam, name)
        for s in ([0.5] if quick else [0.5, 0.6, 0.7]):
            mask = workloads.magnitude_mask(W, s)
            layer = _SweepLayer(W, mask)
            nnz = int(np.count_nonzero(mask))
            for M in ([2048] if quick else [512, 2048]):
                r = _sweep_prefill_point(layer, M, stream)
                ex = 2.0 * M * N * K / r["sparse_us"] / 1e6
                r.update({"kind": "prefill", "family": fam, "layer": name, "N": N, "K": K,
                          "sparsity": s, "M": M, "TFLOP/s_executed": round(ex, 1),
                          "tensor_frac": round(ex / tc, 4),
                          "TFLOP/s_useful": round(2.0 * M * nnz / r["sparse_us"] / 1e6, 1)})
                _emit(r, fh)
            del layer
            torch.cuda.empty_cache()


def sweep_taxonomy(quick: bool, fh, stream):
    """The GEMM-centric taxonomy shapes of "Beyond FLOPs" on the Llama-7B FFN: width-pruned
    N (gate/up 11008 -> 8256, 5504; down's K likewise) in decode and prefill, token-reduced
    M in {2048, 1024, 512}, and the K-reduced down projection keeping 25/50/75 % of its
    inputs by top-k |activation| ("Reduced Matrix Multiplication" §4.2, §5.1): on the dense
    side a gather of the kept weight columns (timed separately) plus cuBLAS on the reduced
    K, on the sparse side top-k selection plus spw_spmv with that column set on the full
    compressed layer."""
    import torch
    import spmm_tiled_column_b200 as spw
    hbm, tc = peaks()[0], peaks()[1]
    for w in ([8256] if quick else [8256, 5504]):
        for name, (N, K) in (("gate", (w, 4096)), ("down", (4096, w))):
            W = workloads.weight(N, K, "sweep-width", name, w)
            mask = workloads.magnitude_mask(W, 0.5)
            layer = _SweepLayer(W, mask)
            x, _ = workloads.decode_act(name, 1, K, 0.0, "sweep-width", w)
            r = _sweep_decode_point(layer, x, 0.0, stream)
            byts = decode_bytes(W, mask, x, 0.0)
            r.update({"kind": "width_decode", "layer": name, "N": N, "K": K, "sparsity": 0.5,
                      "B": 1, "bytes": byts, "GB/s": round(byts / r["sparse_us"] / 1e3, 1),
                      "hbm_frac": round(byts / r["sparse_us"] / 1e3 / hbm, 4)})
            _emit(r, fh)
            for M in ([2048] if quick else [2048, 1024, 512]):
                r = _sweep_prefill_point(layer, M, stream)
                ex = 2.0 * M * N * K / r["sparse_us"] / 1e6
                r.update({"kind": "width_prefill", "layer": name, "N": N, "K": K,
                          "sparsity": 0.5, "M": M, "TFLOP/s_executed": round(ex, 1),
                          "tensor_frac": round(ex / tc, 4)})
                _emit(r, fh)
            del layer
            torch.cuda.empty_cache()
    N, K = workloads.LLAMA7B_LAYERS["down"]
    W = workloads.weight(N, K, "sweep-kred")
    mask = workloads.magnitude_mask(W, 0.5)
    layer = _SweepLayer(W, mask)
    x = workloads.silu_gate_up_act(1, K, "sweep-kred")
    xd = _dev(x)
    Wd = layer.dense[0]
    for keep in ([0.5] if quick else [0.25, 0.5, 0.75]):
        k = int(round(keep * K))
        bits = torch.empty((-(-K // 32)) + 3, dtype=torch.int32, device="cuda")
        idx = torch.empty(k, dtype=torch.int32, device="cuda")
        spw.spw_select_topk(xd, k, bits, idx)
        torch.cuda.synchronize()
        sel_us = graph_us([lambda: spw.spw_select_topk(xd, k, bits, idx)], stream)
        rec = _sweep_decode_point(layer, x, 0.0, stream, act_bits=bits)
        il = idx.long()
        Wg = [Wd.index_select(1, il).contiguous() for _ in range(_copies(N * k * 2))]
        xg = xd.index_select(1, il).contiguous()
        gather_us = graph_us([lambda r=r: Wd.index_select(1, il) for r in range(2)], stream)
        yg = [torch.empty((1, N), dtype=torch.float16, device="cuda") for _ in Wg]
        gemm_us = graph_us([(lambda r=r: torch.matmul(xg, Wg[r].t(), out=yg[r]))
                            for r in range(len(Wg))], stream)
        act = np.zeros(K, dtype=bool)
        act[idx.cpu().numpy()] = True
        xk = np.where(act[None, :], x, np.float16(0)).astype(np.float16)
        byts = decode_bytes(W, mask, xk, 0.0)
        rec.update({"kind": "k_reduced_down", "N": N, "K": K, "keep": keep, "k": k,
                    "topk_select_us": round(sel_us, 3), "dense_gather_us": round(gather_us, 3),
                    "dense_gemm_reduced_K_us": round(gemm_us, 3), "bytes": byts,
                    "GB/s": round(byts / rec["sparse_us"] / 1e3, 1),
                    "select_plus_decode_us": round(sel_us + rec["sparse_us"], 3)})
        rec["speedup_vs_gather_plus_gemm"] = round((gather_us + gemm_us) / rec["sparse_us"], 3)
        _emit(rec, fh)
        del Wg


def run_sweep(args):
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("the sweeps need a CUDA device")
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    fh = open(args.out, "a") if args.out else None
    stream = torch.cuda.Stream()
    {"decode": sweep_decode, "prefill": sweep_prefill, "taxonomy": sweep_taxonomy}[args.sweep](
        args.quick, fh, stream)
    return 0


# ------------------------------------------------------------------ one case (--case)

def run_case(args):
    """One decode or prefill case of the seeded Llama-7B layers in a loop: --warmup untimed
    calls, then --reps calls timed with CUDA events on the launching stream (L2-warm: the
    same operands every call).  Meant for profilers, which select launches with -s / -c."""
    import torch
    import spmm_tiled_column_b200 as spw
    N, K = workloads.LLAMA7B_LAYERS[args.layer]
    stream = torch.cuda.current_stream()
    if args.case == "ffn":  # the gate/up pair of one layer, whatever --layer says
        N, K = workloads.LLAMA7B_LAYERS["gate"]
        gate = workloads.pruned_layer("gate", N, K, args.sparsity, "profile")
        up = workloads.pruned_layer("up", N, K, args.sparsity, "profile")
        lg = spw.SparseLinear(_dev(gate.W), _dev(gate.mask))
        lu = spw.SparseLinear(_dev(up.W), _dev(up.mask))
        xd = _dev(workloads.normal_act(args.batch, K, "profile"))
        h = torch.empty((args.batch, N), dtype=torch.float16, device="cuda")
        bits = torch.empty(((N + 31) // 32,), dtype=torch.int32, device="cuda")
        ws = torch.zeros(spw.spw_spmv_ffn_workspace_bytes(lg.hdr, lu.hdr, args.batch),
                         dtype=torch.uint8, device="cuda")
        run = lambda: spw.spw_spmv_ffn(lg.hdr, lg.buf, lu.hdr, lu.buf, xd, args.t, h, bits, ws)  # noqa: E731
    else:
        layer = workloads.pruned_layer(args.layer, N, K, args.sparsity, "profile")
        lin = spw.SparseLinear(_dev(layer.W), _dev(layer.mask))
        if args.case == "spmm":
            X = _dev(workloads.normal_act(args.m, K, "profile"))
            Y = torch.empty((args.m, N), dtype=torch.float16, device="cuda")
            run = lambda: lin.spmm(X, Y)  # noqa: E731
        elif args.case == "spmm24":  # 2:4 + residual; --mask24 exact: an exact 2:4 mask
            mask = (workloads.structured24_mask(N, K, "profile", count=2) if args.mask24 == "exact"
                    else layer.mask)
            l24 = spw.SparseLinear24(_dev(layer.W), _dev(mask))
            X = _dev(workloads.normal_act(args.m, K, "profile"))
            Y = torch.empty((args.m, N), dtype=torch.float16, device="cuda")
            ws24 = torch.zeros(max(spw.spw_spmm24_workspace_bytes(l24.hdr_r, args.m), 16),
                               dtype=torch.uint8, device="cuda")
            run = lambda: l24.spmm(X, Y, ws24)  # noqa: E731
        elif args.case == "tokens":  # per-token index sets: 4 domains, SiLU(g) * u values
            X, _ = workloads.domain_tokens(args.m, K, 4, 0.5, "profile", silu=True)
            Xd = _dev(X)
            Y = torch.empty((args.m, N), dtype=torch.float16, device="cuda")
            wst = torch.zeros(spw.spw_spmm_tokens_workspace_bytes(lin.hdr, args.m), dtype=torch.uint8,
                              device="cuda")
            run = lambda: lin.spmm_tokens(Xd, args.t, Y, wst)  # noqa: E731
        else:
            x, t = workloads.decode_act(args.layer, args.batch, K, args.act, "profile")
            xd = _dev(x)
            y = torch.empty((args.batch, N), dtype=torch.float16, device="cuda")
            thr = t if args.use_threshold else 0.0
            if args.case == "tc":
                ws = torch.zeros(max(spw.spw_spmv_tc_workspace_bytes(lin.hdr, args.batch), 16),
                                 dtype=torch.uint8, device="cuda")
                run = lambda: spw.spw_spmv_tc(lin.hdr, lin.buf, xd, thr, None, y, ws)  # noqa: E731
            else:
                if args.fetch:  # decode copies only the active columns' 16-byte chunks
                    spw.spw_set_column_fetch(2)
                run = lambda: lin.spmv(xd, thr, None, y)  # noqa: E731
    for _ in range(args.warmup):
        run()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.reps):
        run()
    b.record(stream)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    print(f"{args.case} {args.layer} {N}x{K} sparsity={args.sparsity} B={args.batch} M={args.m} "
          f"act={args.act}: {a.elapsed_time(b) * 1e3 / args.reps:.2f} us per call (L2-warm loop)")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sweep", choices=["decode", "prefill", "taxonomy"], default=None)
    ap.add_argument("--quick", action="store_true", help="--sweep: a few points of each sweep")
    ap.add_argument("--out", default=None, help="--sweep: also append the JSON lines to this file")
    ap.add_argument("--case", choices=["spmv", "spmm", "tc", "ffn", "spmm24", "tokens"], default=None)
    ap.add_argument("--layer", default="q", choices=sorted(workloads.LLAMA7B_LAYERS))
    ap.add_argument("--sparsity", type=float, default=0.5)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--act", type=float, default=0.0, help="--case: activation sparsity")
    ap.add_argument("--use-threshold", action="store_true",
                    help="--case spmv/tc: pass the activation threshold instead of 0")
    ap.add_argument("--m", type=int, default=2048, help="--case spmm: tokens")
    ap.add_argument("--t", type=float, default=0.0, help="--case ffn: threshold on h; tokens: on X")
    ap.add_argument("--fetch", action="store_true",
                    help="--case spmv: active-column fetch (spw_set_column_fetch(2))")
    ap.add_argument("--mask24", choices=["magnitude", "exact"], default="magnitude",
                    help="--case spmm24: the 50 %% magnitude mask or an exact 2:4 mask")
    ap.add_argument("--reps", type=int, default=10, help="--case: timed calls")
    args = ap.parse_args()
    if args.sweep:
        return run_sweep(args)
    if args.case:
        return run_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(reference_arm(args, world)), flush=True)
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
