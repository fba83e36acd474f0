"""GPU parity of the prefill SpMM (tcgen05) against the fp64 oracle.

Bar: max|Y - Y_ref| / max|Y_ref| <= 5e-3 over each call's whole output (fp16 inputs, fp32
accumulation in tensor memory, fp16 output); exact where the result is exact.  Full-size
shapes are checked on seeded sampled rows (the oracle computes rows one by one)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def run(W, mask, X, ldx=None, ldy=None):
    lin = spw.SparseLinear(dev(W), dev(mask))
    M, K = X.shape
    if ldx is None and M > 1 and K % 8:
        ldx = -(-K // 8) * 8        # tensor copies need 16-byte row strides
    Xd = dev(X) if ldx is None else padded_rows(X, ldx)
    Y = None
    if ldy is not None:
        Y = torch.full((M, ldy), float("nan"), dtype=torch.float16, device="cuda")[:, :lin.N]
    out = lin.spmm(Xd, Y)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    return host(out).astype(np.float64), lin


@pytest.mark.parametrize("N,K,M", [(256, 512, 16), (512, 256, 16), (256, 512, 256),
                                   (300, 200, 37), (65, 130, 300), (1, 64, 1), (64, 1, 5),
                                   (513, 1000, 600), (128, 4160, 64)])
def test_parity_small(N, K, M):
    W = workloads.weight(N, K, "gspmm")
    mask = workloads.random_mask(N, K, 0.5, "gspmm")
    X = workloads.normal_act(M, K, "gspmm")
    Y, _ = run(W, mask, X)
    assert oracle.rel_err(Y, oracle.spmm(W, mask, X)) <= TOL, (N, K, M)


def test_tiny_config_layer():
    layer = workloads.pruned_layer("tiny", 256, 512, 0.5, "cfg1")
    X = workloads.normal_act(16, 512, "cfg1-prefill")
    Y, _ = run(layer.W, layer.mask, X)
    assert oracle.rel_err(Y, oracle.spmm(layer.W, layer.mask, X)) <= TOL


def test_identity_exact_and_zero():
    K = 384
    X = workloads.normal_act(300, K, "gspmm-id")
    Y, _ = run(np.eye(K, dtype=np.float16), np.eye(K, dtype=np.uint8), X)
    np.testing.assert_array_equal(Y, X.astype(np.float64))
    Y, _ = run(workloads.weight(200, K, "z"), np.zeros((200, K), np.uint8), X)
    assert not Y.any()


def test_dense_mask_matches_dense_product():
    N, K, M = 256, 640, 256
    W = workloads.weight(N, K, "gspmm-dense")
    X = workloads.normal_act(M, K, "gspmm-dense")
    Y, _ = run(W, np.ones((N, K), np.uint8), X)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    assert oracle.rel_err(Y, ref) <= TOL


def test_all_ones_mask_matches_cublas():
    N, K, M = 1024, 2048, 512
    W = workloads.weight(N, K, "gspmm-cublas")
    X = workloads.normal_act(M, K, "gspmm-cublas")
    Y, _ = run(W, np.ones((N, K), np.uint8), X)
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    ref = host(torch.matmul(dev(X), dev(W).t())).astype(np.float64)
    assert oracle.rel_err(Y, ref) <= TOL


def test_dropped_weights_never_read():
    N, K, M = 256, 512, 128
    W = workloads.weight(N, K, "gspmm-drop")
    mask = workloads.random_mask(N, K, 0.5, "gspmm-drop")
    W2 = W.copy()
    W2[mask == 0] = np.float16(np.nan)
    X = workloads.normal_act(M, K, "gspmm-drop")
    Y, _ = run(W2, mask, X)
    assert np.isfinite(Y).all()
    assert oracle.rel_err(Y, oracle.spmm(W, mask, X)) <= TOL


def test_spmm_equals_spmv_rows():
    N, K = 320, 1024
    W = workloads.weight(N, K, "gspmm-v")
    mask = workloads.random_mask(N, K, 0.5, "gspmm-v")
    X = workloads.normal_act(16, K, "gspmm-v")
    Y, lin = run(W, mask, X)
    y = host(lin.spmv(dev(X))).astype(np.float64)
    assert oracle.rel_err(Y, y) <= TOL


def test_strided_and_m_zero():
    N, K, M = 200, 264, 70
    W = workloads.weight(N, K, "gspmm-s")
    mask = workloads.random_mask(N, K, 0.5, "gspmm-s")
    X = workloads.normal_act(M, K, "gspmm-s")
    Y, lin = run(W, mask, X, ldx=272, ldy=208)
    assert oracle.rel_err(Y, oracle.spmm(W, mask, X)) <= TOL
    empty = torch.empty((0, K), dtype=torch.float16, device="cuda")
    assert lin.spmm(empty).shape == (0, N)


@pytest.mark.parametrize("name,s", [("q", 0.5), ("gate", 0.6), ("down", 0.7)])
def test_llama7b_prefill_m2048_sampled(name, s):
    N, K = workloads.LLAMA7B_LAYERS[name]
    M = 2048
    layer = workloads.pruned_layer(name, N, K, s, "cfg3")
    X = workloads.normal_act(M, K, "cfg3", name)
    Y, _ = run(layer.W, layer.mask, X)
    rows = np.sort(workloads.rng("cfg3-rows", name).choice(M, 128, replace=False)).astype(np.int32)
    ref = oracle.spmm(layer.W, layer.mask, X, rows)
    assert oracle.rel_err(Y[rows], ref) <= TOL
    assert np.isfinite(Y).all()


@pytest.mark.parametrize("N,K,M", [(5120, 5120, 2048), (5000, 5120, 2000), (5120, 13824, 2048)])
def test_hybrid_split_second_wave(N, K, M):
    # 160 output tiles on 148 SMs: the plan runs the first tiles whole and splits the
    # last ones along K so they fill the SMs as the whole tiles finish (Llama-13B
    # attention and down shapes at M = 2048, one ragged variant); rows of every token
    # tile are sampled, so whole and split tiles are both checked
    W = workloads.weight(N, K, "hyb")
    mask = workloads.random_mask(N, K, 0.5, "hyb")
    X = workloads.normal_act(M, K, "hyb")
    Y, ws = run(W, mask, X)
    rows = np.sort(np.concatenate([workloads.rng("hyb-rows", N, M).choice(M, 40, replace=False),
                                   [0, M - 1]])).astype(np.int32)
    ref = oracle.spmm(W, mask, X, rows)
    assert oracle.rel_err(Y[rows], ref) <= TOL
    assert np.isfinite(Y).all()


@pytest.mark.parametrize("N,K,M", [(256, 512, 256), (513, 1000, 600), (4096, 4096, 2048),
                                   (5120, 5120, 2048)])
def test_pair_mode_parity(N, K, M, monkeypatch):
    # SM-pair tiles (SPW_SPMM_PAIR=1): 256 weight rows per cluster of two CTAs, one
    # tcgen05 cta_group::2 MMA per k-slice; the ragged shape leaves the second CTA of the
    # last pair past N, and 5120 x 5120 at M = 2048 splits its second-wave tiles along K
    # (one counter and partial tile per 128-row half)
    monkeypatch.setenv("SPW_SPMM_PAIR", "1")
    W = workloads.weight(N, K, "pair")
    mask = workloads.random_mask(N, K, 0.5, "pair")
    X = workloads.normal_act(M, K, "pair")
    lin = spw.SparseLinear(dev(W), dev(mask))
    assert spw.spw_spmm_plan(lin.hdr, M)["cta_pair"] == 1
    Y, _ = run(W, mask, X)
    if M <= 600:
        assert oracle.rel_err(Y, oracle.spmm(W, mask, X)) <= TOL
    else:
        rows = np.sort(np.concatenate([workloads.rng("pair-rows", N, M).choice(M, 62, replace=False),
                                       [0, M - 1]])).astype(np.int32)
        assert oracle.rel_err(Y[rows], oracle.spmm(W, mask, X, rows)) <= TOL
    assert np.isfinite(Y).all()


def test_pair_mode_identity_exact(monkeypatch):
    monkeypatch.setenv("SPW_SPMM_PAIR", "1")
    K = 384
    X = workloads.normal_act(300, K, "pair-id")
    Y, _ = run(np.eye(K, dtype=np.float16), np.eye(K, dtype=np.uint8), X)
    np.testing.assert_array_equal(Y, X.astype(np.float64))
