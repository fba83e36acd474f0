"""Brute force over tiny shapes, and linearity of the decode in its activations.

Every product call is checked against the fp64 oracle on many seeded random shapes with
N and K drawn from 1..70: one or two tiles in each direction, ragged in both, with
densities from empty to full, random batches, token counts and thresholds.  The bar is
the products' own: max|y - y_ref| / max|y_ref| <= 5e-3 over the whole output, and an
exactly zero output where the reference is zero.

Linearity: for activations x1 and x2 with disjoint supports, the threshold rule keeps
in x1 + x2 exactly what it keeps in x1 and in x2, so y(x1 + x2) = y(x1) + y(x2) up to
rounding, for the decode and the prefill alike."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]

DENSITIES = (0.0, 0.1, 0.5, 0.9, 1.0)


def rows16(X):
    """Device copy of X with 16-byte row strides (rows padded when K % 8 != 0)."""
    M, K = X.shape
    return dev(X) if M == 1 or K % 8 == 0 else padded_rows(X, -(-K // 8) * 8)


def case(tag, i, max_rows):
    r = workloads.rng("tiny-sweep", tag, i)
    N, K = int(r.integers(1, 71)), int(r.integers(1, 71))
    rows = int(r.integers(1, max_rows + 1))
    density = float(r.choice(DENSITIES))
    t = float(r.choice([0.0, 0.0, 0.5, 1.5]))
    W = workloads.weight(N, K, "tiny-sweep", tag, i)
    mask = workloads.random_mask(N, K, density, "tiny-sweep", tag, i)
    x = workloads.normal_act(rows, K, "tiny-sweep", tag, i)
    x = workloads.zero_random(x, float(r.choice([0.0, 0.5, 1.0])), "tiny-sweep", tag, i)
    return W, mask, x, t


def check(y, ref, what):
    y = host(y).astype(np.float64)
    assert oracle.rel_err(y, ref) <= TOL, what
    if not ref.any():
        assert not y.any(), what


def ok():
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK


def test_decode_tiny_shapes_brute_force():
    for i in range(1000):
        W, mask, x, t = case("spmv", i, 16)
        lin = spw.SparseLinear(dev(W), dev(mask))
        y = lin.spmv(rows16(x), t)
        ok()
        check(y, oracle.spmv(W, mask, x, t), ("spmv", i, W.shape, x.shape[0], t))


def test_prefill_tiny_shapes_brute_force():
    for i in range(300):
        W, mask, X, _ = case("spmm", i, 300)
        lin = spw.SparseLinear(dev(W), dev(mask))
        Y = lin.spmm(rows16(X))
        ok()
        check(Y, oracle.spmm(W, mask, X), ("spmm", i, W.shape, X.shape[0]))


def test_token_prefill_tiny_shapes_brute_force():
    for i in range(200):
        W, mask, X, t = case("tokens", i, 300)
        lin = spw.SparseLinear(dev(W), dev(mask))
        Y = lin.spmm_tokens(rows16(X), t)
        ok()
        check(Y, oracle.spmm_tokens(W, mask, X, t), ("tokens", i, W.shape, X.shape[0], t))


def test_2of4_prefill_tiny_shapes_brute_force():
    for i in range(200):
        W, mask, X, _ = case("spmm24", i, 300)
        lin = spw.SparseLinear24(dev(W), dev(mask))
        Y = lin.spmm(rows16(X))
        ok()
        check(Y, oracle.spmm(W, mask, X), ("spmm24", i, W.shape, X.shape[0]))


def disjoint_split(x, *seed):
    """x1 + x2 == x exactly, with no position nonzero in both."""
    m = workloads.rng(*seed).random(x.shape) < 0.5
    zero = np.float16(0)
    return np.where(m, x, zero), np.where(m, zero, x)


@pytest.mark.parametrize("t", [0.0, 0.5])
@pytest.mark.parametrize("B", [1, 4, 16])
def test_decode_linear_in_disjoint_activations(B, t):
    N, K = 1000, 3000
    W = workloads.weight(N, K, "lin")
    mask = workloads.random_mask(N, K, 0.5, "lin")
    x = workloads.normal_act(B, K, "lin", B)
    x1, x2 = disjoint_split(x, "lin-split", B)
    lin = spw.SparseLinear(dev(W), dev(mask))
    ys = []
    for v in (x, x1, x2):
        ys.append(host(lin.spmv(rows16(v), t)).astype(np.float64))
        ok()
    assert oracle.rel_err(ys[1] + ys[2], ys[0]) <= 2 * TOL
    assert oracle.rel_err(ys[0], oracle.spmv(W, mask, x, t)) <= TOL


def test_prefill_linear_in_disjoint_activations():
    N, K, M = 640, 1500, 300
    W = workloads.weight(N, K, "lin-mm")
    mask = workloads.random_mask(N, K, 0.5, "lin-mm")
    X = workloads.normal_act(M, K, "lin-mm")
    X1, X2 = disjoint_split(X, "lin-mm-split")
    lin = spw.SparseLinear(dev(W), dev(mask))
    Ys = []
    for v in (X, X1, X2):
        Ys.append(host(lin.spmm(rows16(v))).astype(np.float64))
        ok()
    assert oracle.rel_err(Ys[1] + Ys[2], Ys[0]) <= 2 * TOL
    assert oracle.rel_err(Ys[0], oracle.spmm(W, mask, X)) <= TOL
