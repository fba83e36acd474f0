"""GPU parity of the column selection against the oracle: bit-exact bitmaps, counts and
ascending index lists."""
import numpy as np
import pytest

import oracle
import workloads
from gpu_util import dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]

SPECIALS = np.array([0.0, -0.0, 1.0, -1.0, 0.5, 2.0 ** -24, 65504.0, np.inf, -np.inf, np.nan,
                     0.25, 0.2498], dtype=np.float16)


def words(K):
    return (K + 31) // 32


@pytest.mark.parametrize("B,K,t", [(1, 512, 0.0), (1, 4096, 0.5), (4, 11008, 0.3),
                                   (16, 4096, 1.0), (3, 1000, 0.25), (2, 33, 0.1),
                                   (1, 1, 0.0), (16, 13824, 0.7)])
def test_threshold_matches_oracle(B, K, t):
    x = workloads.silu_gate_up_act(B, K, "gsel", t)
    x, _ = workloads.zero_smallest(x, 0.3)
    bits, count = spw.spw_select_threshold(dev(x), t)
    ref_bits, ref_count = oracle.select_threshold(x, t)
    np.testing.assert_array_equal(host(bits)[:words(K)], ref_bits)
    assert int(host(count)[0]) == ref_count


def test_threshold_special_values_and_stride():
    r = np.random.default_rng(5)
    x = r.choice(SPECIALS, size=(5, 300))
    xd = padded_rows(x, 304)
    for t in (0.0, 0.25, 1.0):
        bits, count = spw.spw_select_threshold(xd, t)
        ref_bits, ref_count = oracle.select_threshold(x, t)
        np.testing.assert_array_equal(host(bits)[:words(300)], ref_bits)
        assert int(host(count)[0]) == ref_count


@pytest.mark.parametrize("B,K,k", [(1, 11008, 2752), (1, 11008, 5504), (1, 11008, 8256),
                                   (4, 4096, 1000), (16, 5120, 1), (2, 70, 70), (1, 70, 0),
                                   (3, 24576, 12000)])
def test_topk_matches_oracle(B, K, k):
    x = workloads.silu_gate_up_act(B, K, "gtopk", k)
    bits, idx = spw.spw_select_topk(dev(x), k)
    ref_bits, ref_idx = oracle.select_topk(x, k)
    np.testing.assert_array_equal(host(bits)[:words(K)], ref_bits)
    np.testing.assert_array_equal(host(idx), ref_idx)


def test_topk_ties_and_specials():
    r = np.random.default_rng(9)
    for trial in range(6):
        B, K = int(r.integers(1, 5)), int(r.integers(1, 400))
        x = r.choice(SPECIALS if trial % 2 else np.array([0, 1, -1, 2], np.float16), size=(B, K))
        k = int(r.integers(0, K + 1))
        bits, idx = spw.spw_select_topk(dev(x), k)
        ref_bits, ref_idx = oracle.select_topk(x, k)
        np.testing.assert_array_equal(host(bits)[:words(K)], ref_bits)
        np.testing.assert_array_equal(host(idx), ref_idx)


@pytest.mark.parametrize("K", [1, 33, 1000, 11008, 24576])
def test_topk_one_row_ties_and_specials(K):
    # one row: few distinct magnitudes (many ties, both signs), and Inf / NaN, which tie
    # above every finite value; every k from none to all
    r = np.random.default_rng(K)
    vals = np.array([0, -0.0, 0.5, -0.5, 1, -1, 2, 65504, -65504, 6e-8, np.inf, -np.inf, np.nan],
                    np.float16)
    x = r.choice(vals, size=(1, K), p=[.2, .1, .15, .15, .1, .1, .1, .02, .02, .02, .01, .01, .02])
    for k in sorted({0, 1, K // 3, K // 2, K - 1, K} - {-1}):
        if k < 0:
            continue
        bits, idx = spw.spw_select_topk(dev(x), k)
        ref_bits, ref_idx = oracle.select_topk(x, k)
        np.testing.assert_array_equal(host(bits)[:words(K)], ref_bits)
        np.testing.assert_array_equal(host(idx)[:k], ref_idx)


def test_topk_too_large_k_is_unsupported():
    x = dev(np.ones((1, 30000), np.float16))
    with pytest.raises(spw.SpwError) as e:
        spw.spw_select_topk(x, 5)
    assert e.value.status == spw.SPW_ERR_UNSUPPORTED
