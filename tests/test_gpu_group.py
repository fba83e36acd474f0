"""GPU parity of spw_spmv_group (several layers decoded in one launch) against the oracle
and against separate spw_spmv calls."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def make(shapes, tag):
    out = []
    for i, (N, K) in enumerate(shapes):
        W = workloads.weight(N, K, tag, i)
        mask = workloads.random_mask(N, K, 0.5, tag, i)
        out.append((W, mask, spw.SparseLinear(dev(W), dev(mask))))
    return out


@pytest.mark.parametrize("B", [1, 4])
def test_group_matches_oracle(B):
    shapes = [(4096, 4096), (4096, 4096), (1000, 4096), (11008, 4096)]
    L = make(shapes, "group")
    xs = [workloads.zero_random(workloads.normal_act(B, K, "group", i), 0.3, "group", i)
          for i, (N, K) in enumerate(shapes)]
    ys = spw.spw_spmv_group([l.hdr for _, _, l in L], [l.buf for _, _, l in L],
                            [dev(x) for x in xs], 0.1)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    for (W, mask, _), x, y in zip(L, xs, ys):
        assert oracle.rel_err(host(y).astype(np.float64), oracle.spmv(W, mask, x, 0.1)) <= TOL


def test_group_ragged_column_sets_and_counters():
    shapes = [(130, 70), (65, 200), (300, 129)]
    L = make(shapes, "group-r")
    B = 3
    xs = [workloads.normal_act(B, K, "group-r", i) for i, (N, K) in enumerate(shapes)]
    ab = [oracle.select_topk(xs[0], 30)[0], None, oracle.select_topk(xs[2], 100)[0]]
    abd = [None if a is None else dev(np.concatenate([a, np.zeros(3, np.uint32)])) for a in ab]
    xds = [padded_rows(x, -(-x.shape[1] // 8) * 8) for x in xs]
    hdrs = [l.hdr for _, _, l in L]
    ws = torch.zeros(spw.spw_spmv_group_workspace_bytes(hdrs, B), dtype=torch.uint8, device="cuda")
    for rep in range(2):
        ys = spw.spw_spmv_group(hdrs, [l.buf for _, _, l in L], xds, 0.0, abd, ws=ws)
        torch.cuda.synchronize()
        assert spw.spw_last_device_status() == spw.SPW_OK
        for (W, mask, _), x, a, y in zip(L, xs, ab, ys):
            assert oracle.rel_err(host(y).astype(np.float64), oracle.spmv(W, mask, x, 0.0, a)) <= TOL
    # the first layer's counters sit at the start of the workspace and must be zero again
    assert int(ws[:4 * (-(-shapes[0][0] // 64))].count_nonzero()) == 0


def test_group_of_one_is_spmv_bit_for_bit():
    (W, mask, lin), = make([(4096, 11008)], "group-1")
    x = workloads.silu_gate_up_act(2, 11008, "group-1")
    a = host(lin.spmv(dev(x), 0.2))
    (b,) = spw.spw_spmv_group([lin.hdr], [lin.buf], [dev(x)], 0.2)
    np.testing.assert_array_equal(host(b), a)


def test_group_rejects_bad_sizes():
    (W, mask, lin), = make([(64, 64)], "group-bad")
    x = dev(workloads.normal_act(1, 64, "group-bad"))
    with pytest.raises(spw.SpwError):
        spw.spw_spmv_group([lin.hdr] * 9, [lin.buf] * 9, [x] * 9)


def test_prepared_group_matches_group_call():
    # DecodeGroup only caches the argument arrays: same launch, same bits, and it keeps
    # working when the input and output tensors change between calls
    shapes = [(300, 512), (128, 512), (700, 512)]
    lins = [spw.SparseLinear(dev(workloads.weight(N, K, f"prep{i}")),
                             dev(workloads.random_mask(N, K, 0.5, f"prep{i}")))
            for i, (N, K) in enumerate(shapes)]
    hdrs, bufs = [l.hdr for l in lins], [l.buf for l in lins]
    g = spw.DecodeGroup(hdrs, bufs, 3)
    for seed in ("a", "b"):
        x = dev(workloads.normal_act(3, 512, "prep-x", seed))
        ys = [torch.empty((3, N), dtype=torch.float16, device="cuda") for N, _ in shapes]
        g([x] * 3, ys, threshold=0.1)
        ref = spw.spw_spmv_group(hdrs, bufs, [x] * 3, 0.1)
        torch.cuda.synchronize()
        for y, r in zip(ys, ref):
            np.testing.assert_array_equal(host(y).view(np.uint16), host(r).view(np.uint16))
    assert spw.spw_last_device_status() == spw.SPW_OK


def test_bindings_check_tensor_sizes():
    # the library cannot see tensor sizes, so the bindings compare them with the header
    # before any launch: short inputs, outputs, weight buffers or column sets are refused
    (W, mask, lin), = make([(200, 304)], "sizes")
    x = dev(workloads.normal_act(2, 304, "sizes"))
    with pytest.raises(ValueError):
        spw.spw_spmv(lin.hdr, lin.buf, x[:, :296].contiguous())
    with pytest.raises(ValueError):
        spw.spw_spmv(lin.hdr, lin.buf, x, y=torch.empty((2, 199), dtype=torch.float16, device="cuda"))
    with pytest.raises(ValueError):
        spw.spw_spmv(lin.hdr, lin.buf[:-16], x)
    with pytest.raises(ValueError):
        spw.spw_spmv(lin.hdr, lin.buf, x, act_bits=torch.zeros(9, dtype=torch.int32, device="cuda"))
    with pytest.raises(ValueError):
        spw.spw_spmm(lin.hdr, lin.buf, x, torch.empty((1, 200), dtype=torch.float16, device="cuda"))
    g = spw.DecodeGroup([lin.hdr], [lin.buf], 2)
    with pytest.raises(ValueError):
        g([x], [torch.empty((1, 200), dtype=torch.float16, device="cuda")])
    ok = g([x], [torch.empty((2, 200), dtype=torch.float16, device="cuda")])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(ok[0]), host(lin.spmv(x)))
