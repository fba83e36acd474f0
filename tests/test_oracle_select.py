"""Pins of the oracle's column selection (CPU only).

Threshold rule (reading of "Reduced Matrix Multiplication" §4.1-§4.2 with the
configuration's "entries |v| < t zeroed"): an entry takes part iff v != 0 and not
|v| < t; a column is active iff some batch row's entry takes part.  Checked by brute
force in exact rational arithmetic and on special values.

Top-k (same article, §5.1): score = sum over the batch of |x|, highest first, ties by
lower index, listed ascending.  Checked against Python's sorted() on exact Fractions.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads


def bits_to_set(bits, K):
    return {k for k in range(K) if (int(bits[k // 32]) >> (k % 32)) & 1}


def brute_threshold(x16, t):
    B, K = x16.shape
    tq = Fraction(float(np.float32(t)))
    out = set()
    for k in range(K):
        for b in range(B):
            v = float(x16[b, k])
            if np.isnan(v) or np.isinf(v):   # not zero and never below a finite t
                out.add(k)
                continue
            if v != 0 and not (abs(Fraction(v)) < tq):
                out.add(k)
    return out


SPECIALS = np.array([0.0, -0.0, 1.0, -1.0, 0.5, -0.5, 2.0 ** -24, -(2.0 ** -24), 65504.0,
                     np.inf, -np.inf, np.nan, 0.25, 0.2498, 1e-3], dtype=np.float16)


@pytest.mark.parametrize("seed", range(40))
def test_threshold_brute_force(seed):
    r = np.random.default_rng(seed)
    B, K = int(r.integers(1, 5)), int(r.integers(1, 70))
    x = r.choice(SPECIALS, size=(B, K)) if seed % 2 else \
        r.standard_normal((B, K)).astype(np.float16)
    t = float(r.choice([0.0, 0.25, 0.5, 1.0, 2.0 ** -24, 1e-3, 100.0]))
    bits, count = oracle.select_threshold(x, t)
    want = brute_threshold(x, t)
    assert bits_to_set(bits, K) == want
    assert count == len(want)
    # bits beyond K stay clear
    for k in range(K, 32 * bits.size):
        assert not (int(bits[k // 32]) >> (k % 32)) & 1


def test_threshold_special_cases():
    x = np.array([[0.0, -0.0, 0.25, np.float16(0.25) - np.float16(2 ** -12), np.nan,
                   -0.25, np.inf, 2.0 ** -24]], dtype=np.float16)
    bits, count = oracle.select_threshold(x, 0.25)
    # zeros dropped, |x| == t kept, just below t dropped, NaN kept, -t kept, inf kept,
    # smallest subnormal dropped
    assert bits_to_set(bits, x.shape[1]) == {2, 4, 5, 6}
    assert count == 4
    bits, count = oracle.select_threshold(x, 0.0)
    assert bits_to_set(bits, x.shape[1]) == {2, 3, 4, 5, 6, 7}   # t = 0: every nonzero


def test_threshold_union_over_batch():
    x = np.zeros((3, 40), np.float16)
    x[0, 1] = 1.0
    x[1, 33] = -2.0
    x[2, 39] = 0.1   # below t
    bits, count = oracle.select_threshold(x, 0.5)
    assert bits_to_set(bits, 40) == {1, 33} and count == 2


def test_threshold_rejects_bad_t():
    x = np.ones((1, 8), np.float16)
    for t in (-1.0, float("nan"), float("inf")):
        with pytest.raises(oracle.OracleError):
            oracle.select_threshold(x, t)


def brute_topk(x16, k):
    B, K = x16.shape
    scores = []
    for c in range(K):
        col = [float(v) for v in x16[:, c]]
        if any(not np.isfinite(v) for v in col):
            s = (1, Fraction(0))        # non-finite scores above every finite one
        else:
            s = (0, sum((abs(Fraction(v)) for v in col), Fraction(0)))
        scores.append((s, c))
    ranked = sorted(scores, key=lambda sc: (-sc[0][0], -sc[0][1], sc[1]))
    return sorted(c for _, c in ranked[:k])


@pytest.mark.parametrize("seed", range(30))
def test_topk_brute_force(seed):
    r = np.random.default_rng(100 + seed)
    B, K = int(r.integers(1, 5)), int(r.integers(1, 90))
    if seed % 3 == 0:   # many ties
        x = r.choice(np.array([0, 1, -1, 2, 0.5], np.float16), size=(B, K))
    elif seed % 3 == 1:
        x = r.choice(SPECIALS, size=(B, K))
    else:
        x = r.standard_normal((B, K)).astype(np.float16)
    k = int(r.integers(0, K + 1))
    bits, idx = oracle.select_topk(x, k)
    want = brute_topk(x, k)
    assert list(idx) == want
    assert bits_to_set(bits, K) == set(want)


def test_topk_properties_at_config_size():
    x = workloads.silu_gate_up_act(1, 11008, "topk")
    for keep in (2752, 5504, 8256):
        bits, idx = oracle.select_topk(x, keep)
        assert idx.size == keep and np.all(np.diff(idx.astype(np.int64)) > 0)
        score = np.abs(x.astype(np.float64)).sum(axis=0)
        chosen = np.zeros(11008, bool)
        chosen[idx] = True
        assert score[chosen].min() >= score[~chosen].max()


def test_topk_ties_prefer_lower_index():
    x = np.ones((2, 10), np.float16)
    _, idx = oracle.select_topk(x, 3)
    assert list(idx) == [0, 1, 2]
    x[0, 7] = 2
    _, idx = oracle.select_topk(x, 3)
    assert list(idx) == [0, 1, 7]


def test_topk_rejects_bad_k():
    x = np.ones((1, 8), np.float16)
    for k in (-1, 9):
        with pytest.raises(oracle.OracleError):
            oracle.select_topk(x, k)
