"""Pins of the oracle's 2:4 + residual split (CPU only).

"Accelerating LLM GPU inference with moderately unstructured sparse weight matrices"
(abstract, §1): a 2:4 structured part for the sparse tensor cores plus a residual that
keeps the SpMM exact.  Reading: in each group of four columns of a row, the first two
kept weights form the 2:4 part, the others the residual.  Pinned by hand-derived masks,
set identities, the per-group count formula and the pinned product.
"""
import numpy as np
import pytest

import oracle
import workloads


def test_hand_example():
    mask = np.array([[1, 1, 1, 1, 0, 0, 1, 0, 1, 0],
                     [0, 1, 0, 1, 0, 1, 0, 1, 1, 1],
                     [1, 0, 1, 1, 1, 1, 1, 0, 0, 1]], np.uint8)
    s, r = oracle.split24(mask)
    np.testing.assert_array_equal(s, [[1, 1, 0, 0, 0, 0, 1, 0, 1, 0],
                                      [0, 1, 0, 1, 0, 1, 0, 1, 1, 1],
                                      [1, 0, 1, 0, 1, 1, 0, 0, 0, 1]])
    np.testing.assert_array_equal(r, [[0, 0, 1, 1, 0, 0, 0, 0, 0, 0],
                                      [0, 0, 0, 0, 0, 0, 0, 0, 0, 0],
                                      [0, 0, 0, 1, 0, 0, 1, 0, 0, 0]])


@pytest.mark.parametrize("N,K,density", [(7, 4, 0.5), (33, 130, 0.5), (64, 257, 0.7), (5, 1, 0.9),
                                         (16, 64, 1.0), (16, 64, 0.0)])
def test_partition_and_counts(N, K, density):
    mask = workloads.random_mask(N, K, density, "split24")
    s, r = oracle.split24(mask)
    assert not (s & r).any()
    np.testing.assert_array_equal((s | r).astype(bool), mask.astype(bool))
    Kp = -(-K // 4) * 4
    pad = lambda a: np.pad(a.astype(int), ((0, 0), (0, Kp - K))).reshape(N, -1, 4).sum(axis=2)
    cnt, cs, cr = pad(mask), pad(s), pad(r)
    np.testing.assert_array_equal(cs, np.minimum(cnt, 2))
    np.testing.assert_array_equal(cr, np.maximum(cnt - 2, 0))


def test_structured_mask_has_empty_residual():
    N, K = 40, 96
    r = np.random.default_rng(3)
    mask = np.zeros((N, K), np.uint8)
    for n in range(N):
        for g in range(0, K, 4):
            mask[n, g + r.choice(4, size=int(r.integers(0, 3)), replace=False)] = 1
    s, res = oracle.split24(mask)
    np.testing.assert_array_equal(s, mask)
    assert not res.any()


def test_parts_sum_to_the_product():
    N, K, M = 70, 200, 5
    W = workloads.weight(N, K, "split24-prod")
    mask = workloads.random_mask(N, K, 0.5, "split24-prod")
    X = workloads.normal_act(M, K, "split24-prod")
    s, r = oracle.split24(mask)
    np.testing.assert_allclose(oracle.spmm(W, s, X) + oracle.spmm(W, r, X),
                               oracle.spmm(W, mask, X), rtol=0, atol=1e-12)
