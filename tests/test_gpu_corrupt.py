"""Per-tile buffer checks in the product kernels.

A buffer whose header is valid but whose sections disagree -- a tile whose bitmaps claim
more kept weights than any tile may hold, a tile whose bitmaps claim a few more kept
weights than its own values hold, or tile pointers outside the values section --
must come back as SPW_ERR_FORMAT from spw_last_device_status, with every access kept
inside the buffer and the stages, and the next call on a consistent buffer (same
workspace) must be correct again: the split-K counters are left at zero."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]

N, K = 256, 512


def layer():
    W = workloads.weight(N, K, "corrupt")
    mask = workloads.random_mask(N, K, 0.5, "corrupt")
    return W, mask, spw.SparseLinear(dev(W), dev(mask))


def corrupted(lin, what):
    h = lin.hdr
    buf = lin.buf.clone()
    if what == "bitmaps":
        # tile 0: all 64 x 64 bits set, far more kept weights than max_tile_units allows
        buf[h.off_bitmaps:h.off_bitmaps + 512] = 0xFF
    elif what == "overclaim":
        # tile 0: 16 more bits set than its values hold -- still far fewer than a stage
        # holds, so only the count against the tile's own size can catch it
        words = buf[h.off_bitmaps:h.off_bitmaps + 512].view(torch.int64)
        bits = words.cpu().numpy().view(np.uint64)
        added = 0
        for w in range(64):
            for r in range(64):
                if added < 16 and not (int(bits[w]) >> r) & 1:
                    bits[w] = np.uint64(int(bits[w]) | (1 << r))
                    added += 1
        buf[h.off_bitmaps:h.off_bitmaps + 512] = torch.from_numpy(bits.view(np.uint8).copy()).cuda()
    else:
        # tile 0's end (= tile 1's start) far past the values section
        T = h.n_strips * h.n_ktiles
        tp = buf[h.off_tileptr:h.off_tileptr + 4 * (T + 1)].view(torch.int32)
        tp[1] = 0x7FFFFFFF
    return buf


def status():
    torch.cuda.synchronize()
    return spw.spw_last_device_status()


@pytest.fixture
def fetch_mode(request):
    prev = spw.spw_set_column_fetch(request.param)
    yield request.param
    spw.spw_set_column_fetch(prev)


@pytest.mark.parametrize("fetch_mode", [0, 2], ids=["whole-tiles", "column-fetch"], indirect=True)
@pytest.mark.parametrize("what", ["bitmaps", "overclaim", "tileptr"])
@pytest.mark.parametrize("B", [1, 8])
def test_decode_reports_format_and_recovers(what, B, fetch_mode):
    W, mask, lin = layer()
    assert status() == spw.SPW_OK
    x = workloads.normal_act(B, K, "corrupt", B)
    ws = lin.workspace(B)
    spw.spw_spmv(lin.hdr, corrupted(lin, what), dev(x), ws=ws)
    assert status() == spw.SPW_ERR_FORMAT
    y = spw.spw_spmv(lin.hdr, lin.buf, dev(x), ws=ws)
    assert status() == spw.SPW_OK
    assert oracle.rel_err(host(y).astype(np.float64), oracle.spmv(W, mask, x, 0.0, None)) <= TOL


@pytest.mark.parametrize("what", ["bitmaps", "overclaim", "tileptr"])
def test_tensor_core_decode_reports_format_and_recovers(what):
    W, mask, lin = layer()
    assert status() == spw.SPW_OK
    x = workloads.normal_act(16, K, "corrupt-tc")
    need = spw.spw_spmv_tc_workspace_bytes(lin.hdr, 16)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    spw.spw_spmv_tc(lin.hdr, corrupted(lin, what), dev(x), ws=ws)
    assert status() == spw.SPW_ERR_FORMAT
    y = spw.spw_spmv_tc(lin.hdr, lin.buf, dev(x), ws=ws)
    assert status() == spw.SPW_OK
    assert oracle.rel_err(host(y).astype(np.float64), oracle.spmv(W, mask, x, 0.0, None)) <= TOL


@pytest.mark.parametrize("what", ["bitmaps", "overclaim", "tileptr"])
def test_prefill_reports_format_and_recovers(what):
    W, mask, lin = layer()
    assert status() == spw.SPW_OK
    X = workloads.normal_act(200, K, "corrupt-mm")
    spw.spw_spmm(lin.hdr, corrupted(lin, what), dev(X))
    assert status() == spw.SPW_ERR_FORMAT
    Y = spw.spw_spmm(lin.hdr, lin.buf, dev(X))
    assert status() == spw.SPW_OK
    assert oracle.rel_err(host(Y).astype(np.float64), oracle.spmm(W, mask, X)) <= TOL
