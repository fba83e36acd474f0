"""Sweeps of the decode and prefill calls against dense cuBLAS at the same shapes.

    python -m spmm_tiled_column_b200.sweep decode   [--quick] [--out FILE]
    python -m spmm_tiled_column_b200.sweep prefill  [--quick] [--out FILE]
    python -m spmm_tiled_column_b200.sweep taxonomy [--quick] [--out FILE]

One JSON object per line, one line per point.  Workloads (seeded, synthetic):

* decode: Llama-7B linears (q 4096x4096, gate 11008x4096, down 4096x11008) at 50 % weight
  sparsity and Llama-13B linears (5120x5120, 13824x5120, 5120x13824) at 40-80 %, each
  crossed with activation sparsity a (the smallest floor(a K) entries of every batch row
  zeroed) and batch B in {1, 4, 16}.
* prefill: the same shapes at 50/60/70 % and M in {512, 2048}.
* taxonomy (the GEMM-centric taxonomy sweep of "Beyond FLOPs"): width-pruned FFN shapes
  (N 11008 -> 8256, 5504 for gate/up; K likewise for down) in decode and prefill; the
  K-reduced down projection keeping 25/50/75 % of its 11008 inputs by top-k |activation|
  ("Reduced Matrix Multiplication" §4.2, §5.1) -- on the dense side a gather of the kept
  weight columns plus cuBLAS on the reduced K, on the sparse side spw_spmv with the top-k
  column set on the full compressed layer; and token-reduced M in {2048, 1024, 512}.

Timing: CUDA events around CUDA-graph replays of R launches that cycle through R copies
of the operands, R chosen so the copies exceed three times the L2 size; the figure is
the median over replays of (graph time / R).  Decode GB/s count algorithmic bytes: values
and bitmap words of the active columns, activations and outputs.  Prefill TFLOP/s count
the executed dense-equivalent work 2 M N K (tensor fraction against the measured dense
peak) and the useful work 2 M nnz.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys

import numpy as np
import torch

from . import (SparseLinear, spw_last_device_status, spw_select_topk, spw_spmm, spw_spmv,
               spw_spmv_tc, spw_spmv_tc_workspace_bytes)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import workloads  # noqa: E402  (seeded input generators, no arithmetic of the method)

L2_BYTES = 126 * 2**20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d.get("hbm_gbs", 6650.0)), float(d.get("bf16_tflops", 1590.0))
    return 6650.0, 1590.0


def _dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.float16)
    return torch.from_numpy(a).cuda()


def _copies(nbytes: int, cap: int = 24) -> int:
    return max(2, min(cap, math.ceil(3 * L2_BYTES / max(nbytes, 1))))


def _time_rotating(calls, reps: int = 20) -> float:
    """Median microseconds per call over graph replays; calls[r]() issues rotation r."""
    R = len(calls)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for c in calls:
            c()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c()
    with torch.cuda.stream(stream):
        for _ in range(3):
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
    return float(np.median(times))


def _decode_bytes(mask: np.ndarray, x: np.ndarray, t: float) -> int:
    N, K = mask.shape
    B = x.shape[0]
    xf = x.astype(np.float64)
    keep = (xf != 0) & ~(np.abs(xf) < np.float64(np.float32(t)))
    active = keep.any(axis=0)
    nnz = int(np.count_nonzero(mask[:, active]))
    return 2 * nnz + 8 * (-(-N // 64)) * int(active.sum()) + 2 * B * K + 2 * B * N


class _Layer:
    """One pruned weight on the device: compressed copies for the sparse side and dense
    masked copies for cuBLAS."""

    def __init__(self, W: np.ndarray, mask: np.ndarray, dense: bool = True):
        self.W, self.mask = W, mask
        self.N, self.K = W.shape
        Wd = np.where(mask.astype(bool), W, np.float16(0)).astype(np.float16)
        self.lin = SparseLinear(_dev(W), _dev(mask))
        self.R = _copies(self.lin.buf.numel())
        self.bufs = [self.lin.buf] + [self.lin.buf.clone() for _ in range(self.R - 1)]
        self.dense = None
        if dense:
            d0 = _dev(Wd)
            Rd = _copies(d0.numel() * 2)
            self.dense = [d0] + [d0.clone() for _ in range(Rd - 1)]


def _decode_point(layer: _Layer, x: np.ndarray, t: float, act_bits=None) -> dict:
    B = x.shape[0]
    xd = _dev(x)
    # split-K counters start at zero (each call leaves them zero)
    ws = [torch.zeros(max(16, layer.lin.workspace(B).numel()), dtype=torch.uint8, device="cuda")
          for _ in layer.bufs]
    ys = [torch.empty((B, layer.N), dtype=torch.float16, device="cuda") for _ in layer.bufs]
    calls = [(lambda r=r: spw_spmv(layer.lin.hdr, layer.bufs[r], xd, t, act_bits, ys[r], ws[r]))
             for r in range(len(layer.bufs))]
    us = _time_rotating(calls)
    assert spw_last_device_status() == 0
    out = {"sparse_us": round(us, 3)}
    if B >= 4:  # the tensor-core decode path as well
        need = spw_spmv_tc_workspace_bytes(layer.lin.hdr, B)
        tws = [torch.zeros(max(16, need), dtype=torch.uint8, device="cuda") for _ in layer.bufs]
        tcalls = [(lambda r=r: spw_spmv_tc(layer.lin.hdr, layer.bufs[r], xd, t, act_bits, ys[r],
                                           tws[r])) for r in range(len(layer.bufs))]
        out["tc_us"] = round(_time_rotating(tcalls), 3)
        assert spw_last_device_status() == 0
    if layer.dense is not None:
        yd = [torch.empty((B, layer.N), dtype=torch.float16, device="cuda") for _ in layer.dense]
        dcalls = [(lambda r=r: torch.matmul(xd, layer.dense[r].t(), out=yd[r]))
                  for r in range(len(layer.dense))]
        dus = _time_rotating(dcalls)
        out.update({"dense_us": round(dus, 3), "speedup": round(dus / us, 3)})
    return out


def _prefill_point(layer: _Layer, M: int, hbm_peak_unused=None) -> dict:
    X = [_dev(workloads.normal_act(M, layer.K, "sweep-prefill", M, layer.K, r)) for r in range(2)]
    Y = [torch.empty((M, layer.N), dtype=torch.float16, device="cuda") for _ in range(2)]
    calls = [(lambda r=r: spw_spmm(layer.lin.hdr, layer.bufs[r % len(layer.bufs)], X[r], Y[r]))
             for r in range(2)]
    us = _time_rotating(calls, reps=10)
    assert spw_last_device_status() == 0
    out = {"sparse_us": round(us, 2)}
    if layer.dense is not None:
        dcalls = [(lambda r=r: torch.matmul(X[r], layer.dense[r % len(layer.dense)].t(), out=Y[r]))
                  for r in range(2)]
        dus = _time_rotating(dcalls, reps=10)
        out.update({"dense_us": round(dus, 2), "speedup": round(dus / us, 3)})
    return out


def _emit(rec: dict, fh):
    line = json.dumps(rec)
    print(line, flush=True)
    if fh:
        fh.write(line + "\n")
        fh.flush()


def sweep_decode(quick: bool, fh):
    hbm, _ = _peaks()
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
            layer = _Layer(W, mask)
            for B in batches:
                for a in acts:
                    act_name = "down" if name == "down" else name
                    x, t = workloads.decode_act(act_name, B, K, a, "sweep", fam, B)
                    r = _decode_point(layer, x, 0.0)
                    byts = _decode_bytes(mask, x, 0.0)
                    r.update({"kind": "decode", "family": fam, "layer": name, "N": N, "K": K,
                              "sparsity": s, "act_sparsity": a, "B": B, "bytes": byts,
                              "GB/s": round(byts / r["sparse_us"] / 1e3, 1),
                              "hbm_frac": round(byts / r["sparse_us"] / 1e3 / hbm, 4)})
                    _emit(r, fh)
            del layer
            torch.cuda.empty_cache()


def sweep_prefill(quick: bool, fh):
    _, tc = _peaks()
    shapes = [("7b", n, workloads.LLAMA7B_LAYERS[n]) for n in ("q", "gate", "down")]
    if not quick:
        shapes += [("13b", n, sh) for n, sh in workloads.LLAMA13B_SHAPES.items()]
    for fam, name, (N, K) in shapes:
        W = workloads.weight(N, K, "sweep", fam, name)
        for s in ([0.5] if quick else [0.5, 0.6, 0.7]):
            mask = workloads.magnitude_mask(W, s)
            layer = _Layer(W, mask)
            nnz = int(np.count_nonzero(mask))
            for M in ([2048] if quick else [512, 2048]):
                r = _prefill_point(layer, M)
                ex = 2.0 * M * N * K / r["sparse_us"] / 1e6
                r.update({"kind": "prefill", "family": fam, "layer": name, "N": N, "K": K,
                          "sparsity": s, "M": M, "TFLOP/s_executed": round(ex, 1),
                          "tensor_frac": round(ex / tc, 4),
                          "TFLOP/s_useful": round(2.0 * M * nnz / r["sparse_us"] / 1e6, 1)})
                _emit(r, fh)
            del layer
            torch.cuda.empty_cache()


def sweep_taxonomy(quick: bool, fh):
    hbm, tc = _peaks()
    # width-pruned FFN shapes: decode B=1 and prefill at M in {2048, 1024, 512}
    widths = [8256] if quick else [8256, 5504]
    for w in widths:
        for name, (N, K) in (("gate", (w, 4096)), ("down", (4096, w))):
            W = workloads.weight(N, K, "sweep-width", name, w)
            mask = workloads.magnitude_mask(W, 0.5)
            layer = _Layer(W, mask)
            x, _ = workloads.decode_act(name, 1, K, 0.0, "sweep-width", w)
            r = _decode_point(layer, x, 0.0)
            byts = _decode_bytes(mask, x, 0.0)
            r.update({"kind": "width_decode", "layer": name, "N": N, "K": K, "sparsity": 0.5,
                      "B": 1, "bytes": byts, "GB/s": round(byts / r["sparse_us"] / 1e3, 1),
                      "hbm_frac": round(byts / r["sparse_us"] / 1e3 / hbm, 4)})
            _emit(r, fh)
            for M in ([2048] if quick else [2048, 1024, 512]):
                r = _prefill_point(layer, M)
                ex = 2.0 * M * N * K / r["sparse_us"] / 1e6
                r.update({"kind": "width_prefill", "layer": name, "N": N, "K": K,
                          "sparsity": 0.5, "M": M, "TFLOP/s_executed": round(ex, 1),
                          "tensor_frac": round(ex / tc, 4)})
                _emit(r, fh)
            del layer
            torch.cuda.empty_cache()
    # K-reduced down projection: keep k of 11008 inputs by top-k |activation|
    N, K = workloads.LLAMA7B_LAYERS["down"]
    W = workloads.weight(N, K, "sweep-kred")
    mask = workloads.magnitude_mask(W, 0.5)
    layer = _Layer(W, mask)
    x = workloads.silu_gate_up_act(1, K, "sweep-kred")
    xd = _dev(x)
    Wd = layer.dense[0]
    for keep in ([0.5] if quick else [0.25, 0.5, 0.75]):
        k = int(round(keep * K))
        bits = torch.empty((-(-K // 32)) + 3, dtype=torch.int32, device="cuda")
        idx = torch.empty(k, dtype=torch.int32, device="cuda")
        spw_select_topk(xd, k, bits, idx)
        torch.cuda.synchronize()
        sel_us = _time_rotating([lambda: spw_select_topk(xd, k, bits, idx)])
        rec = _decode_point(layer, x, 0.0, act_bits=bits)
        # dense side: gather the kept columns (cost reported separately), then cuBLAS on K'
        il = idx.long()
        Wg = [Wd.index_select(1, il).contiguous() for _ in range(_copies(N * k * 2))]
        xg = xd.index_select(1, il).contiguous()
        gather_us = _time_rotating([lambda r=r: Wd.index_select(1, il) for r in range(2)])
        yg = [torch.empty((1, N), dtype=torch.float16, device="cuda") for _ in Wg]
        gemm_us = _time_rotating([(lambda r=r: torch.matmul(xg, Wg[r].t(), out=yg[r]))
                                  for r in range(len(Wg))])
        act = np.zeros(K, dtype=bool)
        act[idx.cpu().numpy()] = True
        xk = np.where(act[None, :], x, np.float16(0)).astype(np.float16)
        byts = _decode_bytes(mask, xk, 0.0)
        rec.update({"kind": "k_reduced_down", "N": N, "K": K, "keep": keep, "k": k,
                    "topk_select_us": round(sel_us, 3), "dense_gather_us": round(gather_us, 3),
                    "dense_gemm_reduced_K_us": round(gemm_us, 3), "bytes": byts,
                    "GB/s": round(byts / rec["sparse_us"] / 1e3, 1)})
        rec["speedup_vs_gather_plus_gemm"] = round((gather_us + gemm_us) / rec["sparse_us"], 3)
        _emit(rec, fh)
        del Wg


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("what", choices=["decode", "prefill", "taxonomy"])
    ap.add_argument("--quick", action="store_true", help="a few points of each sweep")
    ap.add_argument("--out", default=None, help="also append the JSON lines to this file")
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("the sweeps need a CUDA device")
    fh = open(args.out, "a") if args.out else None
    {"decode": sweep_decode, "prefill": sweep_prefill, "taxonomy": sweep_taxonomy}[args.what](
        args.quick, fh)


if __name__ == "__main__":
    main()
