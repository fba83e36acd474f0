"""GPU tests of the bounded-wait timeout path of the product kernels.

Every pipeline wait in the decode, prefill and tensor-core decode kernels gives up after a
limit (about one second by default); the kernel then reports SPW_ERR_TIMEOUT through the
device status word, drains the copies and tensor-core operations it has in flight (those
drain waits keep the default limit), frees its tensor memory and returns, so the context
stays usable.  spw_set_wait_limit_cycles shortens the limit: 100 cycles is far less than
a weight copy needs, so the first wait of the next call gives up.  Each test checks the
reported status, then restores the default limit, zeroes the workspace (its counters are
undefined after a timeout) and checks that the next call matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]

TINY = 100  # SM cycles: shorter than any copy from memory


@pytest.fixture
def layer():
    N, K = 1024, 2048
    W = workloads.weight(N, K, "timeout")
    mask = workloads.random_mask(N, K, 0.5, "timeout")
    lin = spw.SparseLinear(dev(W), dev(mask))
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    return W, mask, lin


def run_with_tiny_limit(call):
    prev = spw.spw_set_wait_limit_cycles(TINY)
    try:
        call()
        torch.cuda.synchronize()
        status = spw.spw_last_device_status()
    finally:
        spw.spw_set_wait_limit_cycles(0)
    assert prev == 2_000_000_000
    assert spw.spw_set_wait_limit_cycles(0) == 2_000_000_000  # restored
    return status


def test_decode_timeout_then_recovers():
    # Several tiles per warp, so that the producer has to wait for a freed stage (a wait
    # of microseconds): a layer with at most a tile per warp may finish without waiting.
    N, K = 4096, 11008
    W = workloads.weight(N, K, "timeout-down")
    mask = workloads.random_mask(N, K, 0.5, "timeout-down")
    lin = spw.SparseLinear(dev(W), dev(mask))
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    x = workloads.normal_act(1, K, "timeout-x")
    xd = dev(x)
    ws = torch.zeros(max(16, spw.spw_spmv_workspace_bytes(lin.hdr, 1)), dtype=torch.uint8,
                     device="cuda")
    status = run_with_tiny_limit(lambda: spw.spw_spmv(lin.hdr, lin.buf, xd, ws=ws))
    assert status == spw.SPW_ERR_TIMEOUT
    ws.zero_()
    y = host(spw.spw_spmv(lin.hdr, lin.buf, xd, ws=ws)).astype(np.float64)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    assert oracle.rel_err(y, oracle.spmv(W, mask, x)) <= TOL


def test_prefill_timeout_then_recovers(layer):
    W, mask, lin = layer
    X = workloads.normal_act(64, W.shape[1], "timeout-X")
    Xd = dev(X)
    status = run_with_tiny_limit(lambda: lin.spmm(Xd))
    assert status == spw.SPW_ERR_TIMEOUT
    Y = host(lin.spmm(Xd)).astype(np.float64)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    assert oracle.rel_err(Y, oracle.spmm(W, mask, X)) <= TOL


def test_tensor_core_decode_timeout_then_recovers(layer):
    W, mask, lin = layer
    x = workloads.normal_act(16, W.shape[1], "timeout-tc")
    xd = dev(x)
    need = spw.spw_spmv_tc_workspace_bytes(lin.hdr, 16)
    ws = torch.zeros(max(16, need), dtype=torch.uint8, device="cuda")
    status = run_with_tiny_limit(lambda: spw.spw_spmv_tc(lin.hdr, lin.buf, xd, ws=ws))
    assert status == spw.SPW_ERR_TIMEOUT
    ws.zero_()
    y = host(spw.spw_spmv_tc(lin.hdr, lin.buf, xd, ws=ws)).astype(np.float64)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    assert oracle.rel_err(y, oracle.spmv(W, mask, x)) <= TOL

