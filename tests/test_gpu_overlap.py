"""GPU tests of spw_set_launch_overlap (programmatic dependent launch of spw_spmv).

With overlap on, a decode kernel may start streaming its weights while the previous
kernel on the stream finishes; activations, outputs and the workspace wait for it.  The
results must equal the oracle's exactly as without overlap: chained calls on different
layers, back-to-back calls on one layer and workspace, and the same inside a CUDA graph."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture
def overlap():
    prev = spw.spw_set_launch_overlap(True)
    yield
    spw.spw_set_launch_overlap(prev)


def layers():
    out = []
    for name in ("q", "gate", "down"):
        N, K = workloads.LLAMA7B_LAYERS[name]
        L = workloads.pruned_layer(name, N, K, 0.5, "overlap")
        out.append((L, spw.SparseLinear(dev(L.W), dev(L.mask))))
    return out


def test_chained_layers_and_repeats(overlap):
    Ls = layers()
    xs, ys, refs = [], [], []
    for rep in range(2):                       # the same layers twice: workspace reuse
        for L, lin in Ls:
            K = L.W.shape[1]
            x = workloads.normal_act(2, K, "overlap", rep)
            xs.append(dev(x))
            ys.append(torch.empty((2, L.W.shape[0]), dtype=torch.float16, device="cuda"))
            refs.append(oracle.spmv(L.W, L.mask, x))
    i = 0
    for rep in range(2):
        for L, lin in Ls:
            lin.spmv(xs[i], 0.0, None, ys[i])   # launched back to back, no sync
            i += 1
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    for y, ref in zip(ys, refs):
        assert oracle.rel_err(host(y).astype(np.float64), ref) <= TOL
    # bit-identical to the same calls without overlap
    spw.spw_set_launch_overlap(False)
    i = 0
    for rep in range(2):
        for L, lin in Ls:
            again = lin.spmv(xs[i])
            np.testing.assert_array_equal(host(again), host(ys[i]))
            i += 1


def test_overlap_inside_cuda_graph(overlap):
    Ls = layers()
    xs = [dev(workloads.normal_act(1, L.W.shape[1], "graph")) for L, _ in Ls]
    ys = [torch.empty((1, L.W.shape[0]), dtype=torch.float16, device="cuda") for L, _ in Ls]
    for (L, lin), x, y in zip(Ls, xs, ys):       # warm-up outside capture
        lin.spmv(x, 0.0, None, y)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        for (L, lin), x, y in zip(Ls, xs, ys):
            lin.spmv(x, 0.0, None, y)
    for (L, lin), x, y in zip(Ls, xs, ys):
        y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    for (L, lin), x, y in zip(Ls, xs, ys):
        ref = oracle.spmv(L.W, L.mask, host(x))
        assert oracle.rel_err(host(y).astype(np.float64), ref) <= TOL
