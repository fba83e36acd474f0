"""GPU parity of the decode with the path chosen by batch size (spw_spmv_auto).

Every batch from 1 to 16 against the fp64 oracle (max|y - y_ref| / max|y_ref| <= 5e-3
over the whole output), and bit-identical to the path the choice names: spw_spmv below
the boundary, spw_spmv_tc from it (both are deterministic)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def rows16(x):
    B, K = x.shape
    return dev(x) if B == 1 or K % 8 == 0 else padded_rows(x, -(-K // 8) * 8)


def ok():
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK


def bits16(y):
    return host(y).view(np.uint16)


@pytest.mark.parametrize("B", range(1, 17))
def test_every_batch_matches_oracle_and_the_path_taken(B):
    N, K = 700, 1100  # ragged in both: 10 strips + 60 rows, 17 k-tiles + 12 columns
    W = workloads.weight(N, K, "auto")
    mask = workloads.random_mask(N, K, 0.5, "auto")
    x = workloads.zero_random(workloads.normal_act(B, K, "auto", B), 0.5, "auto", B)
    lin = spw.SparseLinear(dev(W), dev(mask))
    xd = rows16(x)
    path = spw.spw_spmv_auto_path(B)
    assert path in (0, 1)
    for t in (0.0, 0.5):
        y = lin.spmv_auto(xd, t)
        ok()
        assert oracle.rel_err(host(y).astype(np.float64), oracle.spmv(W, mask, x, t)) <= TOL, (B, t)
        y_path = lin.spmv(xd, t) if path == 0 else spw.spw_spmv_tc(lin.hdr, lin.buf, xd, t)
        ok()
        np.testing.assert_array_equal(bits16(y), bits16(y_path))


def test_column_set_on_both_sides_of_the_boundary():
    N, K = 384, 2000
    W = workloads.weight(N, K, "auto-set")
    mask = workloads.random_mask(N, K, 0.5, "auto-set")
    lin = spw.SparseLinear(dev(W), dev(mask))
    first_tc = [spw.spw_spmv_auto_path(B) for B in range(1, 17)].index(1) + 1
    for B in sorted({max(1, first_tc - 1), first_tc, 16}):
        x = workloads.silu_gate_up_act(B, K, "auto-set", B)
        bits, _ = oracle.select_topk(x, 700)
        ab = dev(np.concatenate([bits, np.zeros(3, np.uint32)]))
        y = lin.spmv_auto(rows16(x), 0.0, ab)
        ok()
        ref = oracle.spmv(W, mask, x, 0.0, bits)
        assert oracle.rel_err(host(y).astype(np.float64), ref) <= TOL, B


def test_llama7b_gate_full_size_batch16():
    N, K = workloads.LLAMA7B_LAYERS["gate"]
    layer = workloads.pruned_layer("gate", N, K, 0.5, "auto-7b")
    x = workloads.normal_act(16, K, "auto-7b")
    lin = spw.SparseLinear(dev(layer.W), dev(layer.mask))
    ws = torch.zeros(max(16, spw.spw_spmv_auto_workspace_bytes(lin.hdr, 16)), dtype=torch.uint8,
                     device="cuda")
    y = spw.spw_spmv_auto(lin.hdr, lin.buf, dev(x), 0.0, None, None, ws)
    ok()
    assert oracle.rel_err(host(y).astype(np.float64), oracle.spmv(layer.W, layer.mask, x)) <= TOL
    y2 = spw.spw_spmv_auto(lin.hdr, lin.buf, dev(x), 0.0, None, None, ws)  # the workspace reused
    ok()
    np.testing.assert_array_equal(bits16(y), bits16(y2))
