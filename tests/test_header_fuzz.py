"""Host-side robustness of header validation and launch planning (CPU, no device).

Every call validates its header and arguments on the host and answers with a status
code; nothing may abort, trap or hang.  Random and extreme headers (huge N and K,
inconsistent offsets, sizes that overflow 32 bits) go through check_header and, when
accepted, through the prefill plan's arithmetic (spw_spmm_plan with an explicit SM
count runs entirely on the host).  Accepted plans must satisfy the invariants the
kernel's indexing relies on."""
import ctypes

from hypothesis import given, settings
from hypothesis import strategies as st

import spmm_tiled_column_b200 as spw


def geometric_header(N, K, units):
    h = spw.spw_format()
    h.magic, h.version, h.N, h.K, h.TN, h.TK = 0x31424354, 1, N, K, 64, 64
    h.n_strips, h.n_ktiles = -(-N // 64), -(-K // 64)
    T = h.n_strips * h.n_ktiles
    h.off_bitmaps = 256
    h.off_tileptr = -(-(256 + 8 * 64 * T) // 256) * 256
    h.off_values = -(-(h.off_tileptr + 4 * (T + 1)) // 256) * 256
    h.bytes_total = h.off_values + 16 * units * T
    h.nnz, h.max_tile_units = min(N * K, 8 * units * T), units
    return h


u32 = st.integers(0, 2**32 - 1)
u64 = st.integers(0, 2**64 - 1)


@settings(max_examples=300, deadline=None)
@given(magic=st.sampled_from([0x31424354, 0, 0x31424353]), version=st.sampled_from([1, 0, 2]),
       N=u32, K=u32, TN=st.sampled_from([64, 32, 0]), TK=st.sampled_from([64, 128]),
       n_strips=u32, n_ktiles=u32, nnz=u64, total=u64, ob=u64, ot=u64, ov=u64, units=u32,
       M=st.integers(-5, 1 << 20), sms=st.integers(1, 1024))
def test_arbitrary_headers_get_a_status(magic, version, N, K, TN, TK, n_strips, n_ktiles, nnz,
                                        total, ob, ot, ov, units, M, sms):
    h = spw.spw_format()
    (h.magic, h.version, h.N, h.K, h.TN, h.TK, h.n_strips, h.n_ktiles, h.nnz, h.bytes_total,
     h.off_bitmaps, h.off_tileptr, h.off_values, h.max_tile_units) = (
        magic, version, N, K, TN, TK, n_strips, n_ktiles, nnz, total, ob, ot, ov, units)
    info = spw.spw_spmm_plan_info()
    rc = spw.lib().spw_spmm_plan(ctypes.byref(h), M, sms, ctypes.byref(info))
    assert rc in (spw.SPW_OK, spw.SPW_ERR_INVALID_ARG, spw.SPW_ERR_FORMAT, spw.SPW_ERR_UNSUPPORTED)
    assert spw.lib().spw_spmv_workspace_bytes(ctypes.byref(h), 1) >= 0


@settings(max_examples=200, deadline=None)
@given(N=st.integers(1, 1 << 20), K=st.integers(1, 1 << 16), units=st.integers(1, 512),
       M=st.integers(1, 1 << 16), sms=st.integers(1, 1024))
def test_valid_headers_plan_consistently(N, K, units, M, sms):
    h = geometric_header(N, K, units)
    info = spw.spw_spmm_plan_info()
    rc = spw.lib().spw_spmm_plan(ctypes.byref(h), M, sms, ctypes.byref(info))
    assert rc in (spw.SPW_OK, spw.SPW_ERR_UNSUPPORTED)
    if rc != spw.SPW_OK:
        return
    tiles = info.token_tiles * info.weight_tiles
    pair = info.cta_pair
    assert pair in (0, 1) and info.reserved == 0
    assert info.weight_tiles == -(-N // (256 if pair else 128))
    assert info.token_tile % 16 == 0 and info.token_tile * info.token_tiles >= M
    assert 1 <= info.k_parts and 0 <= info.whole_tiles <= tiles
    assert info.ctas == (info.whole_tiles + (tiles - info.whole_tiles) * info.k_parts) * (2 if pair else 1)
    if info.k_parts > 1:
        assert info.k_parts <= max(1, h.n_ktiles)
