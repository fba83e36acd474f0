"""Run one decode or prefill case in a loop, for profilers (ncu) and quick timing.

    python -m spmm_tiled_column_b200.profile spmv --layer gate --batch 1 --act 0.0
    python -m spmm_tiled_column_b200.profile spmm --layer q --m 2048
    python -m spmm_tiled_column_b200.profile tc --layer q --batch 16      (spw_spmv_tc)
    python -m spmm_tiled_column_b200.profile ffn --batch 1 --t 0.2       (spw_spmv_ffn, gate/up)

Inputs are the seeded synthetic Llama-7B layers from `workloads` (fp16 N(0, 0.02)
weights, 50% per-row magnitude mask by default).  The case runs `--warmup` untimed
calls, then `--reps` calls timed with CUDA events on the launching stream, and prints
the mean time per call.  Under a profiler, select launches with -s/-c as usual.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402
import spmm_tiled_column_b200 as spw  # noqa: E402


def to_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.float16)
    return torch.from_numpy(a).cuda()


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["spmv", "spmm", "tc", "ffn"])
    ap.add_argument("--layer", default="q", choices=sorted(workloads.LLAMA7B_LAYERS))
    ap.add_argument("--sparsity", type=float, default=0.5)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--act", type=float, default=0.0, help="activation sparsity (decode)")
    ap.add_argument("--m", type=int, default=2048, help="tokens (prefill)")
    ap.add_argument("--t", type=float, default=0.0, help="threshold on h (ffn)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--reps", type=int, default=10)
    args = ap.parse_args()

    N, K = workloads.LLAMA7B_LAYERS[args.layer]
    if args.op != "ffn":
        layer = workloads.pruned_layer(args.layer, N, K, args.sparsity, "profile")
        lin = spw.SparseLinear(to_dev(layer.W), to_dev(layer.mask))
    if args.op == "ffn":  # the gate/up pair of one layer, whatever --layer says
        N, K = workloads.LLAMA7B_LAYERS["gate"]
        up = workloads.pruned_layer("up", N, K, args.sparsity, "profile")
        gate = workloads.pruned_layer("gate", N, K, args.sparsity, "profile")
        lin = spw.SparseLinear(to_dev(gate.W), to_dev(gate.mask))
        lin_up = spw.SparseLinear(to_dev(up.W), to_dev(up.mask))
        xd = to_dev(workloads.normal_act(args.batch, K, "profile"))
        h = torch.empty((args.batch, N), dtype=torch.float16, device="cuda")
        bits = torch.empty(((N + 31) // 32,), dtype=torch.int32, device="cuda")
        ws = torch.zeros(spw.spw_spmv_ffn_workspace_bytes(lin.hdr, lin_up.hdr, args.batch),
                         dtype=torch.uint8, device="cuda")
        run = lambda: spw.spw_spmv_ffn(lin.hdr, lin.buf, lin_up.hdr, lin_up.buf, xd,  # noqa: E731
                                       args.t, h, bits, ws)
        work = f"{(gate.mask.sum() + up.mask.sum()) * 2 / 1e6:.1f} MB of values"
    elif args.op == "tc":
        x, _ = workloads.decode_act(args.layer, args.batch, K, args.act, "profile")
        xd = to_dev(x)
        y = torch.empty((args.batch, N), dtype=torch.float16, device="cuda")
        ws = torch.zeros(max(spw.spw_spmv_tc_workspace_bytes(lin.hdr, args.batch), 16),
                         dtype=torch.uint8, device="cuda")
        run = lambda: spw.spw_spmv_tc(lin.hdr, lin.buf, xd, 0.0, None, y, ws)  # noqa: E731
        work = f"{2 * int(layer.mask.sum()) / 1e6:.1f} MB of values on tensor cores"
    elif args.op == "spmv":
        x, _ = workloads.decode_act(args.layer, args.batch, K, args.act, "profile")
        xd = to_dev(x)
        y = torch.empty((args.batch, N), dtype=torch.float16, device="cuda")
        run = lambda: lin.spmv(xd, 0.0, None, y)  # noqa: E731
        work = f"{2 * int(layer.mask[:, np.any(x != 0, axis=0)].sum()) / 1e6:.1f} MB of active values"
    else:
        X = to_dev(workloads.normal_act(args.m, K, "profile"))
        Y = torch.empty((args.m, N), dtype=torch.float16, device="cuda")
        run = lambda: lin.spmm(X, Y)  # noqa: E731
        work = f"{2.0 * args.m * N * K / 1e9:.1f} GFLOP executed"
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.reps):
        run()
    e.record()
    torch.cuda.synchronize()
    if spw.spw_last_device_status() != spw.SPW_OK:
        print("device status not OK", file=sys.stderr)
        return 1
    print(f"{args.op} {args.layer} {N}x{K} sparsity={args.sparsity} "
          f"{'M=%d' % args.m if args.op == 'spmm' else 'B=%d act=%.2f' % (args.batch, args.act)}: "
          f"{s.elapsed_time(e) * 1e3 / args.reps:.2f} us per call ({work}; L2-warm loop)")
    return 0


if __name__ == "__main__":
    sys.exit(main())
