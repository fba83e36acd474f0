"""GPU parity of prefill with per-token index sets and token grouping.

spw_group_tokens is index work: its permutation, tile signatures and grouped rows must
equal the oracle's bit for bit.  spw_spmm_tokens is a product: max|Y - Y_ref| /
max|Y_ref| <= 5e-3 against the fp64 oracle (Y_ref[m] = token m's own reduced product),
exact where the result is exact; full-size shapes on seeded sampled rows."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def dev_rows(X):
    """Device copy of X with 16-byte row strides (rows padded when K % 8 != 0)."""
    M, K = X.shape
    return dev(X) if M == 1 or K % 8 == 0 else padded_rows(X, -(-K // 8) * 8)


def grouped(X, t, T):
    Xg, perm, tsig = spw.spw_group_tokens(dev_rows(X), t, T)
    torch.cuda.synchronize()
    return host(Xg), host(perm), tsig.cpu().numpy().view(np.uint64)


def rule(X, t):
    xf = X.astype(np.float64)
    keep = ((xf != 0) & ~(np.abs(xf) < np.float64(np.float32(t)))) | np.isnan(xf)
    return np.where(keep, X, np.float16(0))


@pytest.mark.parametrize("M,K,T,t,domains", [
    (1, 64, 1, 0.0, 1), (37, 300, 8, 0.0, 3), (300, 4096, 128, 0.5, 4), (513, 4097, 256, 0.0, 5),
    (2048, 11008, 512, 0.4, 4), (100, 16384, 16, 1.0, 2), (64, 13824, 64, 0.0, 8)])
def test_grouping_matches_oracle_exactly(M, K, T, t, domains):
    X, _ = workloads.domain_tokens(M, K, domains, 0.5, "gtok")
    X[workloads.rng("gtok-z", M, K).random((M, K)) < 0.3] = 0
    Xg, perm, tsig = grouped(X, t, T)
    p_ref, s_ref = oracle.token_groups(X, t, T)
    np.testing.assert_array_equal(perm, p_ref)
    np.testing.assert_array_equal(tsig, s_ref)
    ldg = Xg.shape[1]
    np.testing.assert_array_equal(Xg[:, :K].view(np.uint16), rule(X, t)[p_ref].view(np.uint16))
    assert not Xg[:, K:ldg].view(np.uint16).any()


def test_grouping_special_values():
    # -0 and entries below t are dropped (written +0), NaN and |x| == t kept, Inf kept
    X = np.zeros((4, 70), np.float16)
    X[0, :4] = [-0.0, 0.25, 0.5, -0.5]
    X[1, 65] = np.inf
    X[2, 3] = np.nan
    X[3, 69] = 0.49951172
    Xg, perm, tsig = grouped(X, 0.5, 2)
    p_ref, s_ref = oracle.token_groups(X, 0.5, 2)
    np.testing.assert_array_equal(perm, p_ref)
    np.testing.assert_array_equal(tsig, s_ref)
    np.testing.assert_array_equal(Xg[:, :70].view(np.uint16), rule(X, 0.5)[p_ref].view(np.uint16))


def run_tokens(W, mask, X, t, ws=None):
    lin = spw.SparseLinear(dev(W), dev(mask))
    Y = lin.spmm_tokens(dev_rows(X), t, ws=ws)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    return host(Y).astype(np.float64), lin


@pytest.mark.parametrize("N,K,M,t,domains", [
    (256, 512, 16, 0.0, 2), (300, 700, 300, 0.5, 3), (513, 1000, 600, 0.3, 4),
    (128, 4160, 64, 0.0, 8), (1000, 4096, 1200, 0.6, 4), (65, 130, 7, 1.0, 1)])
def test_parity_small(N, K, M, t, domains):
    W = workloads.weight(N, K, "gtok-w")
    mask = workloads.random_mask(N, K, 0.5, "gtok-w")
    X, _ = workloads.domain_tokens(M, K, domains, 0.5, "gtok-x")
    Y, _ = run_tokens(W, mask, X, t)
    assert oracle.rel_err(Y, oracle.spmm_tokens(W, mask, X, t)) <= TOL, (N, K, M)


def test_split_parts_with_empty_lists():
    # few tokens and few used k-tiles: the plan splits K into more parts than a token
    # tile's list has k-tiles, so some parts run no k-step and contribute zeros
    N, K, M = 256, 4096, 48
    W = workloads.weight(N, K, "gtok-split")
    mask = workloads.random_mask(N, K, 0.5, "gtok-split")
    X = np.zeros((M, K), np.float16)
    X[:, 64 * 7:64 * 9] = workloads.normal_act(M, 128, "gtok-split")
    plan = spw.spw_spmm_tokens_plan(spw.SparseLinear(dev(W), dev(mask)).hdr, M)
    assert plan["k_parts"] > 2
    Y, lin = run_tokens(W, mask, X, 0.0)
    assert oracle.rel_err(Y, oracle.spmm_tokens(W, mask, X, 0.0)) <= TOL


def test_empty_tokens_give_exact_zeros():
    # tokens whose every entry the rule drops have an empty signature, sort first, and
    # their token tile visits no k-tile: their rows are exactly zero
    N, K, M = 384, 1024, 700
    W = workloads.weight(N, K, "gtok-e")
    mask = workloads.random_mask(N, K, 0.5, "gtok-e")
    X, _ = workloads.domain_tokens(M, K, 3, 0.5, "gtok-e")
    quiet = np.arange(0, M, 2)
    X[quiet] = np.clip(X[quiet], -0.25, 0.25)  # all below t = 0.3
    Y, _ = run_tokens(W, mask, X, 0.3)
    assert not Y[quiet].any()
    assert oracle.rel_err(Y, oracle.spmm_tokens(W, mask, X, 0.3)) <= TOL
    Y0, _ = run_tokens(W, mask, np.zeros((M, K), np.float16), 0.0)
    assert not Y0.any()


def test_threshold_zero_dense_tokens_equal_spw_spmm():
    # no zero entries: every token uses every k-tile, the order is the identity and the
    # product visits the same k-steps in the same order as spw_spmm -- bit-identical
    N, K, M = 512, 2048, 1024
    W = workloads.weight(N, K, "gtok-same")
    mask = workloads.random_mask(N, K, 0.5, "gtok-same")
    X = workloads.normal_act(M, K, "gtok-same")
    X[X == 0] = np.float16(1.0)
    Y, lin = run_tokens(W, mask, X, 0.0)
    Ys = host(lin.spmm(dev(X))).astype(np.float64)
    np.testing.assert_array_equal(Y, Ys)


def test_identity_exact_with_threshold():
    K = 384
    X, _ = workloads.domain_tokens(300, K, 3, 0.5, "gtok-id")
    Y, _ = run_tokens(np.eye(K, dtype=np.float16), np.eye(K, dtype=np.uint8), X, 0.5)
    np.testing.assert_array_equal(Y, rule(X, 0.5).astype(np.float64))


def test_counters_left_zero_and_deterministic():
    N, K, M = 1024, 4096, 96
    W = workloads.weight(N, K, "gtok-c")
    mask = workloads.random_mask(N, K, 0.5, "gtok-c")
    X, _ = workloads.domain_tokens(M, K, 4, 0.5, "gtok-c")
    lin = spw.SparseLinear(dev(W), dev(mask))
    need = spw.spw_spmm_tokens_workspace_bytes(lin.hdr, M)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    Y1, _ = run_tokens(W, mask, X, 0.2, ws)
    Y2 = host(lin.spmm_tokens(dev(X), 0.2, ws=ws)).astype(np.float64)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Y1, Y2)
    plan = spw.spw_spmm_tokens_plan(lin.hdr, M)
    assert plan["k_parts"] > 1  # split tiles: their arrival counters are back at zero
    n_counters = plan["token_tiles"] * plan["weight_tiles"] - plan["whole_tiles"]
    assert not ws[:4 * n_counters].any()


@pytest.mark.parametrize("name,t", [("down", 0.3), ("q", 0.5)])
def test_llama7b_prefill_sampled_rows(name, t):
    N, K = workloads.LLAMA7B_LAYERS[name]
    M = 2048
    layer = workloads.pruned_layer(name, N, K, 0.5, "gtok-7b")
    X, _ = workloads.domain_tokens(M, K, 4, 0.5, "gtok-7b", silu=(name == "down"))
    Y, lin = run_tokens(layer.W, layer.mask, X, t)
    rows = workloads.rng("gtok-7b-rows", name).choice(M, size=128, replace=False).astype(np.int32)
    Yr = oracle.spmm_tokens(layer.W, layer.mask, X, t, rows=rows)
    assert oracle.rel_err(Y[rows], Yr) <= TOL
