"""Pins of the oracle's products (CPU only).

y_b[n] = sum_k W[n,k] mask[n,k] x~_b[k] (reduced product over the reduction dimension,
"Reduced Matrix Multiplication" §4.2; equal to the masked dense product, "Accelerating
LLM GPU inference with moderately unstructured sparse weight matrices" §1), and
Y = X W_masked^T for prefill.  Pinned by exact rational brute force, numpy's float64
matmul, and closed forms.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads


def x_tilde(x16, t, act=None):
    """Numpy restatement of the per-entry rule, for comparison with the C oracle."""
    xf = x16.astype(np.float64)
    keep = (xf != 0) & ~(np.abs(xf) < np.float64(np.float32(t)))
    keep |= np.isnan(xf)
    if act is not None:
        K = x16.shape[1]
        inI = np.array([(int(act[k // 32]) >> (k % 32)) & 1 for k in range(K)], bool)
        keep &= inI[None, :]
    return np.where(keep, xf, 0.0)


@pytest.mark.parametrize("seed", range(25))
def test_spmv_exact_rational(seed):
    r = np.random.default_rng(seed)
    N, K, B = (int(v) for v in r.integers(1, 13, size=3))
    B = min(B, 4)
    W = (r.standard_normal((N, K)) * 2).astype(np.float16)
    mask = (r.random((N, K)) < 0.6).astype(np.uint8)
    x = r.standard_normal((B, K)).astype(np.float16)
    x[r.random((B, K)) < 0.3] = 0
    t = float(r.choice([0.0, 0.3, 1.0]))
    y = oracle.spmv(W, mask, x, t)
    xt = x_tilde(x, t)
    for b in range(B):
        for n in range(N):
            terms = [Fraction(float(W[n, k])) * Fraction(float(xt[b, k]))
                     for k in range(K) if mask[n, k]]
            exact = sum(terms, Fraction(0))
            bound = sum((abs(v) for v in terms), Fraction(0)) * Fraction(1, 2 ** 50)
            assert abs(Fraction(float(y[b, n])) - exact) <= bound


@pytest.mark.parametrize("N,K,B,t", [(256, 512, 1, 0.0), (512, 256, 4, 0.5),
                                     (100, 1000, 16, 1.0), (65, 130, 3, 0.0)])
def test_spmv_matches_numpy(N, K, B, t):
    W = workloads.weight(N, K, "np")
    mask = workloads.random_mask(N, K, 0.5, "np")
    x = workloads.normal_act(B, K, "np")
    y = oracle.spmv(W, mask, x, t)
    ref = x_tilde(x, t) @ (W.astype(np.float64) * mask).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_spmv_act_bits_restrict_columns():
    N, K = 70, 200
    W = workloads.weight(N, K, "act")
    mask = workloads.random_mask(N, K, 0.5, "act")
    x = workloads.normal_act(2, K, "act")
    bits, idx = oracle.select_topk(x, 50)
    y = oracle.spmv(W, mask, x, 0.0, bits)
    ref = x[:, idx].astype(np.float64) @ (W[:, idx].astype(np.float64) * mask[:, idx]).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_identity_is_exact():
    K = 96
    W = np.eye(K, dtype=np.float16)
    mask = np.eye(K, dtype=np.uint8)
    x = workloads.normal_act(3, K, "id")
    x[0, ::3] = 0
    y = oracle.spmv(W, mask, x, 0.3)
    np.testing.assert_array_equal(y, x_tilde(x, 0.3))


def test_diagonal_is_exact():
    K = 80
    d = workloads.weight(1, K, "diag", std=3.0)[0]
    W = np.diag(d).astype(np.float16)
    mask = np.eye(K, dtype=np.uint8)
    x = workloads.normal_act(2, K, "diag")
    y = oracle.spmv(W, mask, x)
    np.testing.assert_array_equal(y, d.astype(np.float64)[None, :] * x.astype(np.float64))


def test_zero_cases():
    N, K = 40, 70
    W = workloads.weight(N, K, "zero")
    x = workloads.normal_act(2, K, "zero")
    assert not oracle.spmv(W, np.zeros((N, K), np.uint8), x).any()
    assert not oracle.spmv(W, np.ones((N, K), np.uint8), np.zeros((2, K), np.float16)).any()
    assert not oracle.spmv(W, np.ones((N, K), np.uint8), x, 100.0).any()   # all dropped
    empty = np.zeros((1, (K + 31) // 32), np.uint32)[0]
    assert not oracle.spmv(W, np.ones((N, K), np.uint8), x, 0.0, empty).any()


def test_one_nonzero_per_row():
    N, K = 50, 90
    r = np.random.default_rng(3)
    cols = r.integers(0, K, N)
    W = workloads.weight(N, K, "one")
    mask = np.zeros((N, K), np.uint8)
    mask[np.arange(N), cols] = 1
    x = workloads.normal_act(1, K, "one")
    y = oracle.spmv(W, mask, x)
    np.testing.assert_array_equal(
        y[0], W[np.arange(N), cols].astype(np.float64) * x[0, cols].astype(np.float64))


def test_dropped_columns_contribute_nothing():
    N, K = 64, 256
    W = workloads.weight(N, K, "drop")
    mask = workloads.random_mask(N, K, 0.5, "drop")
    x, _ = workloads.zero_smallest(workloads.normal_act(2, K, "drop"), 0.5)
    y1 = oracle.spmv(W, mask, x, 0.0)
    W2 = W.copy()
    dead = np.all(x == 0, axis=0)
    W2[:, dead] = np.float16(1234.0)
    y2 = oracle.spmv(W2, mask, x, 0.0)
    np.testing.assert_array_equal(y1, y2)


def test_linearity():
    N, K = 64, 300
    W = workloads.weight(N, K, "lin")
    mask = workloads.random_mask(N, K, 0.5, "lin")
    x1 = workloads.normal_act(1, K, "lin1")
    x2 = workloads.normal_act(1, K, "lin2")
    xs = (x1.astype(np.float32) + x2.astype(np.float32)).astype(np.float16)
    # x1 + x2 rounded to fp16 is not exactly linear; compare against the rounded sum
    y = oracle.spmv(W, mask, xs)
    ref = (W.astype(np.float64) * mask) @ xs[0].astype(np.float64)
    np.testing.assert_allclose(y[0], ref, rtol=1e-12, atol=1e-14)
    ya, yb = oracle.spmv(W, mask, x1)[0], oracle.spmv(W, mask, x2)[0]
    assert oracle.rel_err(ya + yb, y[0]) < 5e-3


def test_spmm_matches_numpy_and_rows():
    N, K, M = 130, 200, 37
    W = workloads.weight(N, K, "mm")
    mask = workloads.random_mask(N, K, 0.4, "mm")
    X = workloads.normal_act(M, K, "mm")
    Y = oracle.spmm(W, mask, X)
    ref = X.astype(np.float64) @ (W.astype(np.float64) * mask).T
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-14)
    rows = np.array([36, 0, 5, 5], np.int32)
    np.testing.assert_array_equal(oracle.spmm(W, mask, X, rows), Y[rows])
    # each row equals the decode product of that row with no threshold
    np.testing.assert_array_equal(oracle.spmv(W, mask, X[5:6])[0], Y[5])


def test_spmm_transposed_operand_would_fail():
    # a non-square, non-symmetric case: swapping roles of N and K must not type-check
    N, K = 3, 5
    W = np.arange(1, N * K + 1, dtype=np.float16).reshape(N, K)
    mask = np.ones((N, K), np.uint8)
    X = np.zeros((1, K), np.float16)
    X[0, 4] = 1.0
    Y = oracle.spmm(W, mask, X)
    np.testing.assert_array_equal(Y[0], W[:, 4].astype(np.float64))


def test_rel_err_definition():
    assert oracle.rel_err(np.zeros(3), np.zeros(3)) == 0.0
    assert oracle.rel_err(np.array([0, 1e-30, 0]), np.zeros(3)) == float("inf")
    assert oracle.rel_err(np.array([1.0, 2.0]), np.array([1.0, 2.01])) == pytest.approx(0.01 / 2.01)
    assert oracle.rel_err(np.array([np.nan]), np.array([1.0])) == float("inf")
