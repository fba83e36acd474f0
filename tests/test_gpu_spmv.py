"""GPU parity of the decode spMspV kernel against the fp64 oracle.

Bar: max|y - y_ref| / max|y_ref| <= 5e-3 over each call's whole output (fp16 inputs,
fp32 accumulation, fp16 output), exact equality where the result is exact (identity,
diagonal, zero), exact batch consistency and run-to-run determinism."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def run(W, mask, x, t=0.0, act_bits=None, ldx=None, ldy=None):
    lin = spw.SparseLinear(dev(W), dev(mask))
    B, K = x.shape
    if ldx is None and B > 1 and K % 8:
        ldx = -(-K // 8) * 8          # spw_spmv copies x rows with 16-byte bulk copies
    xd = dev(x) if ldx is None else padded_rows(x, ldx)
    y = None
    if ldy is not None:
        y = torch.zeros((B, ldy), dtype=torch.float16, device="cuda")[:, :lin.N]
    ab = None if act_bits is None else dev(np.concatenate([act_bits, np.zeros(3, np.uint32)]))
    out = lin.spmv(xd, t, ab, y)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    ws = lin.workspace(B)
    n_strips = -(-lin.N // 64)
    assert int(ws[:4 * n_strips].count_nonzero()) == 0, "split-K counters must return to zero"
    return host(out).astype(np.float64), lin


@pytest.mark.parametrize("N,K", [(256, 512), (512, 256), (130, 70), (200, 1000), (64, 64),
                                 (65, 4097), (1, 300), (300, 1)])
@pytest.mark.parametrize("B", [1, 2, 3, 4, 8, 16])
def test_parity_small(N, K, B):
    W = workloads.weight(N, K, "gspmv")
    mask = workloads.random_mask(N, K, 0.5, "gspmv")
    x = workloads.zero_random(workloads.normal_act(B, K, "gspmv"), 0.5, "gspmv")
    for t in (0.0, 0.5):
        y, _ = run(W, mask, x, t)
        ref = oracle.spmv(W, mask, x, t)
        assert oracle.rel_err(y, ref) <= TOL, (N, K, B, t)


@pytest.mark.parametrize("B", [1, 4, 16])
def test_topk_column_set(B):
    N, K = 384, 2000
    W = workloads.weight(N, K, "gtopk")
    mask = workloads.random_mask(N, K, 0.5, "gtopk")
    x = workloads.silu_gate_up_act(B, K, "gtopk")
    bits, idx = oracle.select_topk(x, 700)
    y, _ = run(W, mask, x, 0.0, bits)
    ref = oracle.spmv(W, mask, x, 0.0, bits)
    assert oracle.rel_err(y, ref) <= TOL
    # same as multiplying the gathered columns (the reduced product)
    ref2 = x[:, idx].astype(np.float64) @ (W[:, idx].astype(np.float64) * mask[:, idx]).T
    assert oracle.rel_err(y, ref2) <= TOL


def test_identity_and_diagonal_exact():
    K = 300
    x = workloads.normal_act(3, K, "gid")
    y, _ = run(np.eye(K, dtype=np.float16), np.eye(K, dtype=np.uint8), x, 0.4)
    xt = np.where(np.abs(x.astype(np.float32)) < np.float32(0.4), np.float16(0), x)
    np.testing.assert_array_equal(y, xt.astype(np.float64))
    d = workloads.weight(1, K, "gdiag", std=3.0)[0]
    y, _ = run(np.diag(d).astype(np.float16), np.eye(K, dtype=np.uint8), x)
    want = (d.astype(np.float64)[None, :] * x.astype(np.float64)).astype(np.float16)
    np.testing.assert_array_equal(y, want.astype(np.float64))


def test_one_nonzero_per_row_exact():
    N, K = 200, 500
    cols = np.random.default_rng(1).integers(0, K, N)
    W = workloads.weight(N, K, "gone")
    mask = np.zeros((N, K), np.uint8)
    mask[np.arange(N), cols] = 1
    x = workloads.normal_act(2, K, "gone")
    y, _ = run(W, mask, x)
    want = (W[np.arange(N), cols].astype(np.float64)[None, :] *
            x[:, cols].astype(np.float64)).astype(np.float16)
    np.testing.assert_array_equal(y, want.astype(np.float64))


def test_zero_results_exact():
    N, K = 130, 700
    W = workloads.weight(N, K, "gzero")
    x = workloads.normal_act(4, K, "gzero")
    y, _ = run(W, np.zeros((N, K), np.uint8), x)
    assert not y.any()
    y, _ = run(W, np.ones((N, K), np.uint8), np.zeros((4, K), np.float16))
    assert not y.any()
    y, _ = run(W, np.ones((N, K), np.uint8), x, 100.0)
    assert not y.any()
    y, _ = run(W, np.ones((N, K), np.uint8), x, 0.0, np.zeros((K + 31) // 32, np.uint32))
    assert not y.any()


def test_dropped_columns_never_read():
    N, K = 256, 1024
    W = workloads.weight(N, K, "gdrop")
    mask = workloads.random_mask(N, K, 0.5, "gdrop")
    x, _ = workloads.zero_smallest(workloads.normal_act(2, K, "gdrop"), 0.5)
    dead = np.all(x == 0, axis=0)
    W2 = W.copy()
    W2[:, dead] = np.float16(np.nan)   # kept weights in dropped columns hold NaN
    y, _ = run(W2, mask, x)
    assert np.isfinite(y).all()
    assert oracle.rel_err(y, oracle.spmv(W, mask, x)) <= TOL


def test_nan_activation_propagates_like_oracle():
    N, K = 128, 256
    W = workloads.weight(N, K, "gnan")
    mask = workloads.random_mask(N, K, 0.5, "gnan")
    x = workloads.normal_act(1, K, "gnan")
    x[0, 7] = np.float16(np.nan)
    y, _ = run(W, mask, x)
    ref = oracle.spmv(W, mask, x)
    np.testing.assert_array_equal(np.isnan(y), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.max(np.abs(y[ok] - ref[ok])) <= TOL * np.max(np.abs(ref[ok]))


def test_batch_rows_equal_single_row_runs_and_determinism():
    N, K = 1000, 3000
    W = workloads.weight(N, K, "gbatch")
    mask = workloads.random_mask(N, K, 0.5, "gbatch")
    x = workloads.zero_random(workloads.normal_act(4, K, "gbatch"), 0.3, "gbatch")
    y4, lin = run(W, mask, x, 0.2)
    for b in range(4):
        y1 = host(lin.spmv(dev(x[b:b + 1]), 0.2)).astype(np.float64)
        np.testing.assert_array_equal(y1[0], y4[b])
    again = host(lin.spmv(dev(x), 0.2)).astype(np.float64)
    np.testing.assert_array_equal(again, y4)


def test_strided_operands():
    N, K = 300, 520
    W = workloads.weight(N, K, "gstride")
    mask = workloads.random_mask(N, K, 0.5, "gstride")
    x = workloads.normal_act(3, K, "gstride")
    y, _ = run(W, mask, x, 0.1, ldx=528, ldy=304)
    assert oracle.rel_err(y, oracle.spmv(W, mask, x, 0.1)) <= TOL


@pytest.mark.parametrize("name", ["q", "gate", "down"])
@pytest.mark.parametrize("B", [1, 4, 16])
def test_llama7b_full_size(name, B):
    N, K = workloads.LLAMA7B_LAYERS[name]
    layer = workloads.pruned_layer(name, N, K, 0.5, "cfg2")
    for a in (0.0, 0.5):
        x, t = workloads.decode_act(name, B, K, a, "cfg2")
        y, _ = run(layer.W, layer.mask, x)
        ref = oracle.spmv(layer.W, layer.mask, x)
        assert oracle.rel_err(y, ref) <= TOL, (name, B, a)


@pytest.mark.parametrize("shape,s", [((5120, 5120), 0.8), ((13824, 5120), 0.4),
                                     ((5120, 13824), 0.6)])
def test_llama13b_full_size_b1(shape, s):
    N, K = shape
    layer = workloads.pruned_layer("13b", N, K, s, "cfg4")
    x, t = workloads.decode_act("down" if K > N else "q", 1, K, 0.7, "cfg4")
    raw = workloads.silu_gate_up_act(1, K, "down", "cfg4") if K > N else \
        workloads.normal_act(1, K, "q", "cfg4")
    # threshold form on the unzeroed activations: same set except ties at t
    y, _ = run(layer.W, layer.mask, raw, float(np.float32(t[0])))
    ref = oracle.spmv(layer.W, layer.mask, raw, float(np.float32(t[0])))
    assert oracle.rel_err(y, ref) <= TOL


@pytest.mark.parametrize("shape", [(5120, 5120), (13824, 5120), (5120, 13824)])
@pytest.mark.parametrize("B", [4, 16])
def test_llama13b_full_size_batched(shape, B):
    # the Llama-13B shapes at the batch sizes of the decode sweep, half the entries zeroed
    N, K = shape
    layer = workloads.pruned_layer("13b", N, K, 0.5, "cfg4-batched")
    x, _ = workloads.decode_act("down" if K > N else "q", B, K, 0.5, "cfg4-batched")
    y, _ = run(layer.W, layer.mask, x)
    assert oracle.rel_err(y, oracle.spmv(layer.W, layer.mask, x)) <= TOL


def test_all_ones_mask_matches_cublas():
    # every weight kept: the decode equals the dense product cuBLAS computes (fp32
    # accumulation, no fp16 reduced-precision reductions)
    N, K, B = 1024, 2048, 16
    W = workloads.weight(N, K, "ones-cublas")
    x = workloads.normal_act(B, K, "ones-cublas")
    y, _ = run(W, np.ones((N, K), np.uint8), x)
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    ref = host(torch.matmul(dev(x), dev(W).t())).astype(np.float64)
    assert oracle.rel_err(y, ref) <= TOL
    assert oracle.rel_err(y, oracle.spmv(W, np.ones((N, K), np.uint8), x)) <= TOL


@pytest.mark.parametrize("N,K,B,a,t,use_bits", [
    (4096, 11008, 1, 0.5, 0.0, False), (4096, 11008, 1, 0.5, 0.3, False),
    (1000, 3000, 4, 0.3, 0.2, False), (300, 200, 16, 0.7, 0.1, False),
    (4096, 4096, 1, 0.0, 0.0, False), (513, 1000, 2, 0.5, 0.0, True),
    (11008, 4096, 8, 0.5, 0.25, True)])
def test_column_fetch_equals_whole_tiles(N, K, B, a, t, use_bits):
    # Column fetch (only the active columns' bytes are copied) and whole-tile copies share
    # the work split and the summation order, so they give the same bits; both match the
    # oracle.  spw_set_column_fetch(2) forces column fetch, 0 whole tiles.
    W = workloads.weight(N, K, "fetch")
    mask = workloads.random_mask(N, K, 0.5, "fetch")
    x = workloads.zero_random(workloads.normal_act(B, K, "fetch", B), a, "fetch")
    bits = None
    if use_bits:
        bits, _ = oracle.select_topk(x, K // 2)
    ys = []
    try:
        for mode in (0, 2):
            spw.spw_set_column_fetch(mode)
            y, _ = run(W, mask, x, t, bits)
            ys.append(y)
    finally:
        spw.spw_set_column_fetch(0)
    np.testing.assert_array_equal(ys[0], ys[1])
    ref = oracle.spmv(W, mask, x, t, bits)
    assert oracle.rel_err(ys[1], ref) <= TOL
