"""Pins of the oracle's TCB v1 encoder / decoder (CPU only).

The encoder is the definition of the layout, so it is pinned by (1) hand-derived buffers
in tests/golden/tcb_v1_examples.txt, (2) an independent vectorised reader
(tests/tcb_reader.py) and (3) invariants: bitmap popcount equals the mask's nnz, the
tile pointers follow from the bitmaps, every padding byte is zero, and decoding returns
W * mask bit for bit (dropped positions 0x0000, kept -0.0 stays 0x8000).
"""
import numpy as np
import pytest

import oracle
import workloads
from tcb_reader import (bit_matrix, dense_from_buffer, header, padding_is_zero,
                        parse_golden, golden_inputs, sections)

GOLDEN = parse_golden()


def masked_bits(W, mask):
    W = np.asarray(W)
    if W.dtype == np.float16:
        W = W.view(np.uint16)
    return np.where(mask != 0, W, np.uint16(0)).astype(np.uint16)


@pytest.mark.parametrize("case", GOLDEN, ids=[c["name"] for c in GOLDEN])
def test_golden_encode(case):
    W, mask = golden_inputs(case)
    buf = oracle.tcb_encode(W, mask)
    h = header(buf)
    for k, v in case["header"].items():
        assert h[k] == v, (k, h[k], v)
    assert buf.size == case["header"]["bytes_total"]
    assert not np.any(buf[76:256]), "header tail must be zero"
    _, bm, tp, vals = sections(buf)
    expect_bm = np.zeros_like(bm)
    for (s, k), w in case["bitmap"].items():
        expect_bm[s, k] = w
    np.testing.assert_array_equal(bm, expect_bm)
    np.testing.assert_array_equal(tp, np.array(case["tileptr"], dtype=np.uint32))
    np.testing.assert_array_equal(vals, case["values"])
    assert padding_is_zero(buf)
    assert oracle.tcb_query(mask) == (case["header"]["bytes_total"], case["header"]["nnz"])


@pytest.mark.parametrize("case", GOLDEN, ids=[c["name"] for c in GOLDEN])
def test_golden_decode(case):
    W, mask = golden_inputs(case)
    buf = oracle.tcb_encode(W, mask)
    dense = oracle.tcb_decode(buf)
    if "dense" in case:
        np.testing.assert_array_equal(dense, case["dense"])
    np.testing.assert_array_equal(dense, masked_bits(W, mask))


def adversarial_masks():
    out = []
    for N, K in [(64, 64), (65, 130), (1, 1), (1, 200), (200, 1), (130, 129)]:
        out.append((f"zero_{N}x{K}", np.zeros((N, K), np.uint8)))
        out.append((f"ones_{N}x{K}", np.ones((N, K), np.uint8)))
        cb = ((np.arange(N)[:, None] + np.arange(K)[None, :]) % 2).astype(np.uint8)
        out.append((f"checker_{N}x{K}", cb))
    # single bits at the word-boundary rows of a strip and the last row/column
    for r in (0, 31, 32, 63):
        m = np.zeros((128, 128), np.uint8)
        m[r, 5] = 1
        m[64 + r, 127] = 1
        out.append((f"bit_row{r}", m))
    m = np.zeros((128, 192), np.uint8)
    m[:64, 64:128] = 1      # one full tile, empty neighbours
    out.append(("one_full_tile", m))
    m = np.zeros((100, 70), np.uint8)
    m[99, 69] = 1           # last row of a ragged strip, last column of a ragged tile
    out.append(("last_corner", m))
    return out


@pytest.mark.parametrize("name,mask", adversarial_masks(), ids=lambda v: v if isinstance(v, str) else "")
def test_adversarial_roundtrip(name, mask):
    N, K = mask.shape
    W = workloads.weight(N, K, "adv", name)
    buf = oracle.tcb_encode(W, mask)
    h = header(buf)
    assert h["nnz"] == int(mask.sum())
    np.testing.assert_array_equal(oracle.tcb_decode(buf), masked_bits(W, mask))
    np.testing.assert_array_equal(dense_from_buffer(buf), masked_bits(W, mask))
    assert padding_is_zero(buf)


@pytest.mark.parametrize("N,K,density", [(64, 64, 0.5), (257, 511, 0.5), (130, 70, 0.3),
                                         (96, 320, 0.6), (7, 1000, 0.2), (300, 65, 0.8)])
def test_random_masks(N, K, density):
    W = workloads.weight(N, K, "rand", density)
    mask = workloads.random_mask(N, K, density, "rand")
    buf = oracle.tcb_encode(W, mask)
    h, bm, tp, vals = sections(buf)
    # header geometry
    assert (h["N"], h["K"], h["TN"], h["TK"]) == (N, K, 64, 64)
    assert h["n_strips"] == -(-N // 64) and h["n_ktiles"] == -(-K // 64)
    for key in ("off_bitmaps", "off_tileptr", "off_values"):
        assert h[key] % 256 == 0
    # bitmaps are the mask
    bits, full = bit_matrix(bm, N, K)
    np.testing.assert_array_equal(bits, mask.astype(bool))
    assert not full[N:, :].any() and not full[:, K:].any()
    # popcount == nnz
    assert h["nnz"] == int(mask.sum()) == int(full.sum())
    # tile pointers follow from the bitmaps
    S, T = h["n_strips"], h["n_ktiles"]
    counts = full.reshape(S, 64, T, 64).sum(axis=(1, 3)).reshape(-1)
    expect_tp = np.concatenate([[0], np.cumsum((counts + 7) // 8)])
    np.testing.assert_array_equal(tp, expect_tp.astype(np.uint32))
    assert h["max_tile_units"] == int(((counts + 7) // 8).max())
    assert h["bytes_total"] == h["off_values"] + 16 * int(tp[-1]) == buf.size
    # values: independent reader and the oracle decoder both give W * mask
    np.testing.assert_array_equal(dense_from_buffer(buf), masked_bits(W, mask))
    np.testing.assert_array_equal(oracle.tcb_decode(buf), masked_bits(W, mask))
    assert padding_is_zero(buf)


def test_magnitude_mask_layer_roundtrip():
    layer = workloads.pruned_layer("q", 256, 512, 0.5, "tiny")
    buf = oracle.tcb_encode(layer.W, layer.mask)
    assert header(buf)["nnz"] == 256 * 256
    np.testing.assert_array_equal(oracle.tcb_decode(buf), masked_bits(layer.W, layer.mask))


def test_kept_signed_zero_and_specials_preserved():
    W = np.array([[0x8000, 0x0000, 0x7C00, 0xFC00, 0x7E00, 0x0001]], dtype=np.uint16)
    mask = np.ones_like(W, dtype=np.uint8)
    buf = oracle.tcb_encode(W, mask)
    np.testing.assert_array_equal(oracle.tcb_decode(buf), W)
    _, _, _, vals = sections(buf)
    np.testing.assert_array_equal(vals[:6], W[0])


def test_decode_rejects_corruption():
    W = workloads.weight(70, 70, "corrupt")
    mask = workloads.random_mask(70, 70, 0.5, "corrupt")
    buf = oracle.tcb_encode(W, mask)
    bad = buf.copy()
    bad[0] ^= 1
    with pytest.raises(oracle.OracleError):
        oracle.tcb_decode(bad)
    bad = buf.copy()
    bad[4] = 2  # version
    with pytest.raises(oracle.OracleError):
        oracle.tcb_decode(bad)
    with pytest.raises(oracle.OracleError):
        oracle.tcb_decode(buf[:-16])  # truncated values section
    bad = buf.copy()
    h = header(buf)
    # set a bitmap bit for row 70+ (beyond N) in strip 1
    off = h["off_bitmaps"] + 8 * (1 * h["n_ktiles"] * 64 + 3)
    bad[off + 7] |= 0x80
    with pytest.raises(oracle.OracleError):
        oracle.tcb_decode(bad)


def test_encode_rejects_bad_args():
    W = np.zeros((4, 4), np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.tcb_encode(np.zeros((0, 4), np.uint16), np.zeros((0, 4), np.uint8))
    assert oracle.tcb_query(np.ones((4, 4), np.uint8))[1] == 16
    with pytest.raises(oracle.OracleError):
        oracle.tcb_query(np.ones((4, 0), np.uint8))
