"""GPU parity of the tensor-core decode (spw_spmv_tc) against the fp64 oracle.

Bar: max|y - y_ref| / max|y_ref| <= 5e-3 over each call's whole output (fp16 inputs, fp32
accumulation in tensor memory, fp16 output), exact where the result is exact, split-K
arrival counters back at zero, run-to-run determinism.  Non-finite activations follow the
documented dense-product behaviour (0 * Inf = NaN reaches rows whose weight is dropped)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def run(W, mask, x, t=0.0, act_bits=None, ws_fill=None):
    lin = spw.SparseLinear(dev(W), dev(mask))
    B, K = x.shape
    ldx = -(-K // 8) * 8 if (B > 1 and K % 8) else None
    xd = dev(x) if ldx is None else padded_rows(x, ldx)
    ab = None if act_bits is None else dev(np.concatenate([act_bits, np.zeros(3, np.uint32)]))
    need = spw.spw_spmv_tc_workspace_bytes(lin.hdr, B)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    y = spw.spw_spmv_tc(lin.hdr, lin.buf, xd, t, ab, ws=ws)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    if need:
        # split-K counters (the workspace's first 4 * tiles bytes) are left at zero
        tiles = -(-lin.N // 128)
        assert int(ws[:4 * tiles].count_nonzero()) == 0
    return host(y).astype(np.float64), lin


@pytest.mark.parametrize("N,K", [(256, 512), (512, 256), (130, 70), (65, 4097), (1, 300),
                                 (300, 1), (200, 1000), (128, 4160)])
@pytest.mark.parametrize("B", [1, 3, 8, 16])
def test_parity_small(N, K, B):
    W = workloads.weight(N, K, "gtc")
    mask = workloads.random_mask(N, K, 0.5, "gtc")
    x = workloads.normal_act(B, K, "gtc", B)
    y, _ = run(W, mask, x)
    assert oracle.rel_err(y, oracle.spmv(W, mask, x, 0.0, None)) <= TOL, (N, K, B)


@pytest.mark.parametrize("B,t", [(4, 0.5), (16, 1.0), (8, 0.0)])
def test_threshold_and_column_set(B, t):
    N, K = 300, 900
    W = workloads.weight(N, K, "gtc-t")
    mask = workloads.random_mask(N, K, 0.5, "gtc-t")
    x, _ = workloads.zero_smallest(workloads.normal_act(B, K, "gtc-t"), 0.3)
    ab = oracle.select_topk(x, 500)[0]
    for a in (None, ab):
        y, _ = run(W, mask, x, t, a)
        assert oracle.rel_err(y, oracle.spmv(W, mask, x, t, a)) <= TOL, (B, t, a is None)


@pytest.mark.parametrize("name", ["gate", "down"])
def test_llama7b_full_size_b16(name):
    N, K = workloads.LLAMA7B_LAYERS[name]
    layer = workloads.pruned_layer(name, N, K, 0.5, "gtc-full")
    x, _ = workloads.decode_act(name, 16, K, 0.5, "gtc-full")
    y, _ = run(layer.W, layer.mask, x)
    assert oracle.rel_err(y, oracle.spmv(layer.W, layer.mask, x, 0.0, None)) <= TOL


def test_identity_exact_and_zero():
    K = 384
    x = workloads.normal_act(16, K, "gtc-id")
    y, _ = run(np.eye(K, dtype=np.float16), np.eye(K, dtype=np.uint8), x)
    np.testing.assert_array_equal(y, x.astype(np.float64))
    y, _ = run(workloads.weight(200, K, "gtc-z"), np.zeros((200, K), np.uint8), x)
    assert not y.any()


def test_agrees_with_cuda_core_decode_and_is_deterministic():
    N, K = 4096, 4096
    W = workloads.weight(N, K, "gtc-cc")
    mask = workloads.random_mask(N, K, 0.5, "gtc-cc")
    x = workloads.normal_act(8, K, "gtc-cc")
    a, lin = run(W, mask, x)
    b, _ = run(W, mask, x)
    np.testing.assert_array_equal(a, b)
    c = host(lin.spmv(dev(x))).astype(np.float64)
    ref = oracle.spmv(W, mask, x, 0.0, None)
    assert oracle.rel_err(a, ref) <= TOL and oracle.rel_err(c, ref) <= TOL


def test_nonfinite_activation_reaches_every_row():
    N, K = 200, 256
    W = workloads.weight(N, K, "gtc-nan")
    mask = workloads.random_mask(N, K, 0.5, "gtc-nan")
    x = workloads.normal_act(2, K, "gtc-nan")
    x[1, 17] = np.float16(np.inf)
    y, _ = run(W, mask, x)
    ref = oracle.spmv(W, mask, x, 0.0, None)
    # batch row 0 is finite and matches; row 1 is NaN or Inf everywhere (dense semantics)
    assert oracle.rel_err(y[:1], ref[:1]) <= TOL
    assert not np.isfinite(y[1]).any()
    # the oracle skips dropped weights: rows whose weight in column 17 is dropped stay finite
    assert np.isfinite(ref[1][mask[:, 17] == 0]).all()


def test_rejects_bad_arguments():
    N, K = 64, 64
    lin = spw.SparseLinear(dev(workloads.weight(N, K, "gtc-bad")),
                           dev(workloads.random_mask(N, K, 0.5, "gtc-bad")))
    x = torch.zeros((17, K), dtype=torch.float16, device="cuda")
    with pytest.raises(spw.SpwError):
        spw.spw_spmv_tc(lin.hdr, lin.buf, x)
    with pytest.raises(spw.SpwError):
        spw.spw_spmv_tc(lin.hdr, lin.buf, x[:2], threshold=-1.0)
