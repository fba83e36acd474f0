"""Pins of the oracle's per-token prefill and token grouping (CPU only).

Per-token index sets ("Reduced Matrix Multiplication" §4.2 reduced product, §6.1 every
token of a batch keeps its own channels): Y[m,n] = sum_k x~[m,k] W[n,k] mask[n,k] with
the threshold rule applied to each entry of X.  Token grouping (§6.1: tokens with the
same or alike index sets share one dense product): tokens sorted by their k-tile
signature, ties by index; a token tile's signature is the OR of its tokens'.  Pinned by
exact rational brute force, the independently pinned single-token decode and plain
product, hand-derived orders and a vectorised restatement on small inputs.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads
from test_oracle_products import x_tilde


@pytest.mark.parametrize("seed", range(20))
def test_spmm_tokens_exact_rational(seed):
    r = np.random.default_rng(100 + seed)
    N, K, M = (int(v) for v in r.integers(1, 11, size=3))
    W = (r.standard_normal((N, K)) * 2).astype(np.float16)
    mask = (r.random((N, K)) < 0.6).astype(np.uint8)
    X = r.standard_normal((M, K)).astype(np.float16)
    X[r.random((M, K)) < 0.3] = 0
    t = float(r.choice([0.0, 0.3, 1.0]))
    Y = oracle.spmm_tokens(W, mask, X, t)
    xt = x_tilde(X, t)
    for m in range(M):
        for n in range(N):
            terms = [Fraction(float(W[n, k])) * Fraction(float(xt[m, k]))
                     for k in range(K) if mask[n, k]]
            exact = sum(terms, Fraction(0))
            bound = sum((abs(v) for v in terms), Fraction(0)) * Fraction(1, 2 ** 50)
            assert abs(Fraction(float(Y[m, n])) - exact) <= bound


@pytest.mark.parametrize("t", [0.0, 0.4, 1.2])
def test_each_row_is_that_tokens_decode(t):
    # row m is the single-token decode with the same rule (orc_spmv, pinned on its own)
    N, K, M = 70, 300, 9
    W = workloads.weight(N, K, "tok-rows")
    mask = workloads.random_mask(N, K, 0.5, "tok-rows")
    X = workloads.normal_act(M, K, "tok-rows")
    Y = oracle.spmm_tokens(W, mask, X, t)
    for m in range(M):
        np.testing.assert_array_equal(Y[m], oracle.spmv(W, mask, X[m:m + 1], t)[0])


def test_threshold_zero_is_the_plain_product():
    N, K, M = 65, 130, 7
    W = workloads.weight(N, K, "tok-t0")
    mask = workloads.random_mask(N, K, 0.5, "tok-t0")
    X = workloads.normal_act(M, K, "tok-t0")
    X[:, ::3] = 0
    np.testing.assert_array_equal(oracle.spmm_tokens(W, mask, X, 0.0), oracle.spmm(W, mask, X))


def test_rule_boundary_and_rows():
    # one kept weight per row: |x| == t is kept (exact product), |x| < t and zeros dropped
    K = 8
    W = np.zeros((K, K), np.float16)
    mask = np.eye(K, dtype=np.uint8)
    np.fill_diagonal(W, 3.0)
    X = np.array([[0.5, 0.25, -0.5, 0.0, 0.49951172, -0.75, 2.0, -0.0]], np.float16)
    Y = oracle.spmm_tokens(W, mask, X, 0.5)
    np.testing.assert_array_equal(Y[0], [1.5, 0.0, -1.5, 0.0, 0.0, -2.25, 6.0, 0.0])
    X2 = np.vstack([X, -X, 2 * X])
    Y2 = oracle.spmm_tokens(W, mask, X2, 0.5, rows=np.array([2, 0]))
    np.testing.assert_array_equal(Y2[1], Y[0])
    np.testing.assert_array_equal(Y2[0], oracle.spmm_tokens(W, mask, 2 * X, 0.5)[0])


def test_groups_reverse_order_closed_form():
    # token m keeps one entry, in k-tile M-1-m: signature 2^(M-1-m), so the order is reversed
    M, T = 12, 4
    K = 64 * M
    X = np.zeros((M, K), np.float16)
    for m in range(M):
        X[m, 64 * (M - 1 - m) + 5] = 1.0
    perm, tile_sig = oracle.token_groups(X, 0.0, T)
    np.testing.assert_array_equal(perm, np.arange(M)[::-1])
    # positions 4j..4j+3 hold tokens with k-tiles 4j..4j+3
    np.testing.assert_array_equal(tile_sig[:, 0], [0xF << (4 * j) for j in range(3)])


def test_groups_equal_signatures_keep_index_order():
    M, K = 10, 200
    X = workloads.normal_act(M, K, "tok-eq")  # no zeros: every token uses all 4 k-tiles
    perm, tile_sig = oracle.token_groups(X, 0.0, 3)
    np.testing.assert_array_equal(perm, np.arange(M))
    np.testing.assert_array_equal(tile_sig[:, 0], [0xF] * 4)


def test_groups_word_zero_decides_first_and_threshold_counts():
    # K = 5000: 79 k-tiles in two words.  Token 0: k-tile 64 only (word 1); token 1:
    # k-tile 0 only (word 0); token 2: only entries below t (empty signature); token 3:
    # k-tiles 0 and 64.  Word 0 is compared first: 2 < 0 < 1 < 3.
    K = 5000
    X = np.zeros((4, K), np.float16)
    X[0, 64 * 64 + 1] = 2.0
    X[1, 7] = -2.0
    X[2, 10] = 0.25
    X[2, 4500] = -0.125
    X[3, 3] = 1.0
    X[3, 64 * 64] = 1.0
    perm, tile_sig = oracle.token_groups(X, 0.5, 2)
    np.testing.assert_array_equal(perm, [2, 0, 1, 3])
    np.testing.assert_array_equal(tile_sig, np.array([[0, 1], [1, 1]], np.uint64))


def groups_vectorised(X, t, T):
    """Restatement of the grouping with numpy reshapes and Python's sort."""
    M, K = X.shape
    nk = -(-K // 64)
    keep = x_tilde(X, t) != 0
    keep |= np.isnan(X.astype(np.float64))
    pad = np.zeros((M, nk * 64), bool)
    pad[:, :K] = keep
    act = pad.reshape(M, nk, 64).any(axis=2)
    words = (nk + 63) // 64
    sig = np.zeros((M, words), np.uint64)
    for kt in range(nk):
        sig[act[:, kt], kt // 64] |= np.uint64(1) << np.uint64(kt % 64)
    order = sorted(range(M), key=lambda m: (tuple(int(v) for v in sig[m]), m))
    tiles = -(-M // T)
    tsig = np.zeros((tiles, words), np.uint64)
    for r, m in enumerate(order):
        tsig[r // T] |= sig[m]
    return np.array(order, np.uint32), tsig


@pytest.mark.parametrize("seed", range(12))
def test_groups_match_vectorised_restatement(seed):
    r = np.random.default_rng(seed)
    M = int(r.integers(1, 40))
    K = int(r.choice([1, 63, 64, 65, 300, 4096, 4097, 9000]))
    T = int(r.choice([1, 3, 8, 16]))
    # a few "domains", each with its own active k-tiles, so equal signatures occur
    nk = -(-K // 64)
    dom = r.random((3, nk)) < 0.5
    X = r.standard_normal((M, K)).astype(np.float16)
    for m in range(M):
        cols = np.repeat(dom[r.integers(0, 3)], 64)[:K]
        X[m, ~cols] = 0
    X[r.random((M, K)) < 0.2] = 0
    t = float(r.choice([0.0, 0.7]))
    perm, tile_sig = oracle.token_groups(X, t, T)
    p2, s2 = groups_vectorised(X, t, T)
    np.testing.assert_array_equal(perm, p2)
    np.testing.assert_array_equal(tile_sig, s2)
