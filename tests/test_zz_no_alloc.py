"""GPU test of spw_spmv_noalloc, the decode entry point that allocates nothing.

Some callers cannot call cudaMalloc (a framework that owns all device memory, or a path
that may not take an allocation's implicit synchronisation).  spw_spmv_noalloc serves
them with the library's fixed scratch array instead of a caller workspace.  This test
calls it through the C-ABI twice in a row and checks each result against spw_spmv (the
entry point with a caller workspace) within the tolerance the parity tests use.  The
file sorts last so that a run stopping at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("B,a", [(1, 0.0), (4, 0.5)])
def test_noalloc_matches_spmv_twice(B, a):
    N, K = 4096, 11008
    layer = workloads.pruned_layer("down", N, K, 0.5, "noalloc")
    lin = spw.SparseLinear(dev(layer.W), dev(layer.mask))
    assert spw.spw_spmv_workspace_bytes(lin.hdr, B) <= \
        spw.lib().spw_spmv_noalloc_max_scratch_bytes()
    for call in range(2):
        x, _ = workloads.decode_act("down", B, K, a, "noalloc", call)
        xd = dev(x)
        want = host(lin.spmv(xd)).astype(np.float64)
        y = torch.full((B, N), float("nan"), dtype=torch.float16, device="cuda")
        h = lin.hdr
        torch.cuda.synchronize()
        torch_before = torch.cuda.memory_allocated()
        free_before, _ = torch.cuda.mem_get_info()  # cudaMemGetInfo
        rc = spw.lib().spw_spmv_noalloc(
            ctypes.byref(h), ctypes.c_void_p(lin.buf.data_ptr()), ctypes.c_void_p(xd.data_ptr()),
            B, xd.stride(0), 0.0, None, ctypes.c_void_p(y.data_ptr()), N,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == spw.SPW_OK, spw.status_string(rc)
        torch.cuda.synchronize()
        # The call itself allocates nothing: neither through torch's allocator nor on the
        # device (the first call's one-time work -- the array's address lookup and loading
        # the kernels -- is done by then, so the second call is the one to check).
        assert torch.cuda.memory_allocated() == torch_before
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free_before
        assert spw.spw_last_device_status() == spw.SPW_OK
        got = host(y).astype(np.float64)
        assert oracle.rel_err(got, want) <= TOL
        assert oracle.rel_err(got, oracle.spmv(layer.W, layer.mask, x)) <= TOL


def test_noalloc_bad_argument_launches_nothing():
    # An argument spw_spmv would reject (here a misaligned output pointer) is rejected
    # before the counter clear is queued: the stream sees no work from the call.
    N, K = 256, 512
    layer = workloads.pruned_layer("tiny", N, K, 0.5, "noalloc-bad")
    lin = spw.SparseLinear(dev(layer.W), dev(layer.mask))
    x = dev(workloads.normal_act(1, K, "noalloc-bad"))
    y = torch.zeros((1, N + 8), dtype=torch.float16, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    h = lin.hdr
    rc = spw.lib().spw_spmv_noalloc(
        ctypes.byref(h), ctypes.c_void_p(lin.buf.data_ptr()), ctypes.c_void_p(x.data_ptr()),
        1, K, 0.0, None, ctypes.c_void_p(y.data_ptr() + 2), N, ctypes.c_void_p(s.cuda_stream))
    assert rc == spw.SPW_ERR_ALIGNMENT
    rc = spw.lib().spw_spmv_noalloc(
        ctypes.byref(h), ctypes.c_void_p(lin.buf.data_ptr()), ctypes.c_void_p(x.data_ptr()),
        1, K, -1.0, None, ctypes.c_void_p(y.data_ptr()), N, ctypes.c_void_p(s.cuda_stream))
    assert rc == spw.SPW_ERR_INVALID_ARG
    assert s.query()  # nothing was queued
    assert int(torch.count_nonzero(y)) == 0


def test_noalloc_rejects_oversized_requests():
    # A header for a 65536 x 4096 weight: its batch-16 workspace exceeds the fixed
    # scratch, so the call must be refused on the host before anything is launched or
    # read (the zero buffers below, sized as the header says, are never touched).
    N, K = 65536, 4096
    h = spw.spw_format()
    h.magic, h.version, h.N, h.K, h.TN, h.TK = 0x31424354, 1, N, K, 64, 64
    h.n_strips, h.n_ktiles = N // 64, K // 64
    T = h.n_strips * h.n_ktiles
    h.off_bitmaps = 256
    h.off_tileptr = -(-(256 + 8 * 64 * T) // 256) * 256
    h.off_values = -(-(h.off_tileptr + 4 * (T + 1)) // 256) * 256
    h.bytes_total = h.off_values + 16 * T
    h.nnz, h.max_tile_units = 8 * T, 1
    limit = spw.lib().spw_spmv_noalloc_max_scratch_bytes()
    assert spw.spw_spmv_workspace_bytes(h, 16) > limit
    buf = torch.zeros(h.bytes_total, dtype=torch.uint8, device="cuda")
    x = torch.zeros((16, K), dtype=torch.float16, device="cuda")
    y = torch.zeros((16, N), dtype=torch.float16, device="cuda")
    with pytest.raises(spw.SpwError) as e:
        spw.spw_spmv_noalloc(h, buf, x, y=y)
    assert e.value.status == spw.SPW_ERR_UNSUPPORTED
