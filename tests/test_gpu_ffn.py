"""GPU parity of the fused FFN activation (spw_spmv_ffn) against the fp64 oracle.

h = fp16(SiLU(g) * u) with g, u the fp16 gate and up decode outputs, and the column-set
words of h under the threshold rule ("Reduced Matrix Multiplication" §4.2).  Bars:
- h within the products' tolerance of the oracle's h (g and u are fp32 sums on the GPU,
  exact sums in the oracle, each rounded once to fp16, so they can differ by one unit in
  the last place);
- the column-set words equal, bit for bit, the threshold rule applied to the returned h
  (the rule itself is the pinned one), and equal the oracle's words except for columns
  whose |h| lies within rounding of the threshold;
- pair and split-K counters back at zero, run-to-run determinism."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def bits_to_bool(words, n):
    w = np.asarray(words).view(np.uint32)
    return np.array([(w[k // 32] >> (k % 32)) & 1 for k in range(n)], dtype=bool)


def run(Wg, mg, Wu, mu, x, t, ws=None):
    lg = spw.SparseLinear(dev(Wg), dev(mg))
    lu = spw.SparseLinear(dev(Wu), dev(mu))
    B, K = x.shape
    ldx = -(-K // 8) * 8 if (B > 1 and K % 8) else None
    xd = dev(x) if ldx is None else padded_rows(x, ldx)
    need = spw.spw_spmv_ffn_workspace_bytes(lg.hdr, lu.hdr, B)
    if ws is None:
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    h, bits = spw.spw_spmv_ffn(lg.hdr, lg.buf, lu.hdr, lu.buf, xd, t, ws=ws)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    return host(h), host(bits), ws, (lg, lu)


def check(h, bits, Wg, mg, Wu, mu, x, t):
    N = Wg.shape[0]
    h_ref, bits_ref = oracle.ffn(Wg, mg, Wu, mu, x, t)
    assert oracle.rel_err(h.astype(np.float64), h_ref.astype(np.float64)) <= TOL
    # the words are the threshold rule on the returned h, exactly
    own, _ = oracle.select_threshold(h, t)
    np.testing.assert_array_equal(bits.view(np.uint32), own)
    # and the oracle's words, except where h sits at the threshold within rounding
    diff = bits_to_bool(bits, N) != bits_to_bool(bits_ref, N)
    if diff.any():
        near = np.abs(np.abs(h_ref.astype(np.float64)) - t) <= 2.0 ** -9 * max(t, 1e-3)
        assert near[:, diff].any(axis=0).all(), np.nonzero(diff)
    return h_ref


@pytest.mark.parametrize("N,K", [(256, 512), (130, 70), (64, 4097), (300, 1), (1, 300), (200, 1000)])
@pytest.mark.parametrize("B", [1, 3, 8, 16])
def test_parity_small(N, K, B):
    Wg, Wu = workloads.weight(N, K, "ffn-g"), workloads.weight(N, K, "ffn-u")
    mg, mu = workloads.random_mask(N, K, 0.5, "ffn-g"), workloads.random_mask(N, K, 0.4, "ffn-u")
    x = workloads.normal_act(B, K, "ffn-x", B)
    for t in (0.0, 0.01):
        h, bits, ws, (lg, _) = run(Wg, mg, Wu, mu, x, t)
        check(h, bits, Wg, mg, Wu, mu, x, t)
        # split-K and pair counters (the start of each workspace section) are zero again
        assert int(ws[:4 * lg.hdr.n_strips].count_nonzero()) == 0


@pytest.mark.parametrize("B", [1, 16])
def test_llama7b_gate_up_full_size(B):
    N, K = workloads.LLAMA7B_LAYERS["gate"]
    g = workloads.pruned_layer("gate", N, K, 0.5, "ffn-full")
    u = workloads.pruned_layer("up", N, K, 0.5, "ffn-full")
    x = workloads.normal_act(B, K, "ffn-full-x", B)
    # a threshold near the median |h| of the oracle's result keeps about half the columns
    h0, _ = oracle.ffn(g.W, g.mask, u.W, u.mask, x[:1], 0.0)
    t = float(np.median(np.abs(h0.astype(np.float64))))
    h, bits, _, _ = run(g.W, g.mask, u.W, u.mask, x, t)
    check(h, bits, g.W, g.mask, u.W, u.mask, x, t)
    kept = bits_to_bool(bits, N).mean()
    assert 0.3 < kept <= 1.0


def test_feeds_the_down_projection():
    # h and its column set drive the down projection; the oracle runs the same chain on
    # its own h and column set
    N, K = 512, 384
    Wg, Wu = workloads.weight(N, K, "ffn-c-g"), workloads.weight(N, K, "ffn-c-u")
    mg, mu = workloads.random_mask(N, K, 0.5, "ffn-c-g"), workloads.random_mask(N, K, 0.5, "ffn-c-u")
    Wd, md = workloads.weight(K, N, "ffn-c-d"), workloads.random_mask(K, N, 0.5, "ffn-c-d")
    x = workloads.normal_act(4, K, "ffn-c-x")
    t = 0.02
    h, bits, _, _ = run(Wg, mg, Wu, mu, x, t)
    h_ref, bits_ref = oracle.ffn(Wg, mg, Wu, mu, x, t)
    down = spw.SparseLinear(dev(Wd), dev(md))
    y = host(down.spmv(dev(h), threshold=t, act_bits=dev(bits.view(np.uint32)))).astype(np.float64)
    y_ref = oracle.spmv(Wd, md, h_ref, t, bits_ref)
    assert oracle.rel_err(y, y_ref) <= TOL


def test_deterministic_and_workspace_reuse():
    N, K = 1024, 2048
    Wg, Wu = workloads.weight(N, K, "ffn-d-g"), workloads.weight(N, K, "ffn-d-u")
    mg, mu = workloads.random_mask(N, K, 0.5, "ffn-d-g"), workloads.random_mask(N, K, 0.5, "ffn-d-u")
    x = workloads.normal_act(8, K, "ffn-d-x")
    h1, b1, ws, _ = run(Wg, mg, Wu, mu, x, 0.05)
    h2, b2, _, _ = run(Wg, mg, Wu, mu, x, 0.05, ws=ws)
    np.testing.assert_array_equal(h1.view(np.uint16), h2.view(np.uint16))
    np.testing.assert_array_equal(b1, b2)


def test_nonfinite_input_reaches_h_and_is_kept():
    N, K = 128, 256
    Wg, Wu = workloads.weight(N, K, "ffn-n-g"), workloads.weight(N, K, "ffn-n-u")
    mg = np.ones((N, K), np.uint8)
    mu = np.ones((N, K), np.uint8)
    x = workloads.normal_act(2, K, "ffn-n-x")
    x[1, 5] = np.float16(np.nan)
    h, bits, _, _ = run(Wg, mg, Wu, mu, x, 0.1)
    assert np.isnan(h[1].astype(np.float64)).all()      # every row of g and u sees the NaN
    assert bits_to_bool(bits, N).all()                  # NaN is kept by the threshold rule
    h_ref, _ = oracle.ffn(Wg, mg, Wu, mu, x[:1], 0.1)
    assert oracle.rel_err(h[:1].astype(np.float64), h_ref.astype(np.float64)) <= TOL


def test_rejects_bad_arguments():
    K = 128
    g = spw.SparseLinear(dev(workloads.weight(64, K, "ffn-bad")), dev(workloads.random_mask(64, K, 0.5, "ffn-bad")))
    u = spw.SparseLinear(dev(workloads.weight(96, K, "ffn-bad")), dev(workloads.random_mask(96, K, 0.5, "ffn-bad")))
    x = torch.zeros((1, K), dtype=torch.float16, device="cuda")
    with pytest.raises(spw.SpwError):  # gate and up shapes differ
        spw.spw_spmv_ffn(g.hdr, g.buf, u.hdr, u.buf, x)
    with pytest.raises(spw.SpwError):  # negative threshold
        spw.spw_spmv_ffn(g.hdr, g.buf, g.hdr, g.buf, x, threshold=-1.0)
    with pytest.raises(spw.SpwError):  # batch above 16
        spw.spw_spmv_ffn(g.hdr, g.buf, g.hdr, g.buf, torch.zeros((17, K), dtype=torch.float16, device="cuda"))
    assert spw.spw_spmv_ffn_workspace_bytes(g.hdr, u.hdr, 1) == 0
