"""GPU parity of compress / decompress / query / read against the oracle encoder.

Bar: the device TCB buffer equals the oracle's byte for byte (memcmp of the whole
buffer), and decompress returns W * mask bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import dev, host, needs_gpu, padded_rows
from tcb_reader import golden_inputs, parse_golden
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def masked(W, mask):
    return np.where(mask != 0, np.asarray(W).view(np.uint16), 0).astype(np.uint16)


def check_roundtrip(W, mask, ldw=None, ldm=None):
    N, K = mask.shape
    Wd = dev(W) if ldw is None else padded_rows(np.asarray(W).view(np.float16), ldw)
    if ldm is None:
        md = dev(mask)
    else:
        mb = np.zeros((N, ldm), np.uint8)
        mb[:, :K] = mask
        md = dev(mb)[:, :K]
    ref = oracle.tcb_encode(W, mask)
    nbytes, nnz = spw.spw_format_query(md)
    assert (nbytes, nnz) == (ref.size, int(mask.astype(bool).sum()))
    buf, hdr = spw.spw_compress(Wd, md)
    got = host(buf)
    assert got.size == ref.size
    assert np.array_equal(got, ref), f"first differing byte {np.argmax(got != ref)}"
    assert hdr.bytes_total == ref.size and hdr.nnz == nnz
    dense = host(spw.spw_decompress(hdr, buf)).view(np.uint16)
    np.testing.assert_array_equal(dense, masked(W, mask))
    return buf, hdr


@pytest.mark.parametrize("case", parse_golden(), ids=lambda c: c["name"])
def test_golden_cases(case):
    W, mask = golden_inputs(case)
    check_roundtrip(W.view(np.float16), mask)


@pytest.mark.parametrize("N,K,density", [(64, 64, 0.5), (256, 512, 0.5), (512, 256, 0.5),
                                         (130, 70, 0.3), (65, 130, 0.6), (1, 1, 1.0),
                                         (1, 200, 0.5), (200, 1, 0.5), (333, 1000, 0.45),
                                         (129, 4097, 0.2)])
def test_random_masks(N, K, density):
    W = workloads.weight(N, K, "gfmt", density)
    mask = workloads.random_mask(N, K, density, "gfmt")
    check_roundtrip(W, mask)


def test_adversarial_masks():
    for N, K in [(64, 64), (65, 130), (130, 129)]:
        W = workloads.weight(N, K, "adv")
        for mask in (np.zeros((N, K), np.uint8), np.ones((N, K), np.uint8),
                     ((np.arange(N)[:, None] + np.arange(K)[None, :]) % 2).astype(np.uint8)):
            check_roundtrip(W, mask)
    for r in (0, 31, 32, 63):
        m = np.zeros((128, 128), np.uint8)
        m[r, 5] = 1
        m[64 + r, 127] = 1
        check_roundtrip(workloads.weight(128, 128, "bit", r), m)


def test_strided_inputs_and_special_values():
    N, K = 70, 100
    W = workloads.weight(N, K, "strided")
    Wb = W.view(np.uint16).copy()
    Wb[0, :6] = [0x8000, 0x0000, 0x7C00, 0xFC00, 0x7E00, 0x0001]  # -0, +0, inf, -inf, nan, subnormal
    mask = workloads.random_mask(N, K, 0.5, "strided")
    mask[0, :6] = 1
    mask[mask != 0] = 7  # any nonzero byte means kept
    check_roundtrip(Wb.view(np.float16), mask, ldw=104, ldm=112)


def test_llama_shape_magnitude_mask():
    layer = workloads.pruned_layer("gate", 11008, 4096, 0.5, "gfmt")
    check_roundtrip(layer.W, layer.mask)


def test_format_read_and_errors():
    W = workloads.weight(100, 200, "read")
    mask = workloads.random_mask(100, 200, 0.5, "read")
    buf, hdr = spw.spw_compress(dev(W), dev(mask))
    h2 = spw.spw_format_read(buf)
    assert h2.as_dict() == hdr.as_dict()
    with pytest.raises(spw.SpwError) as e:
        spw.spw_format_read(buf[:-16])
    assert e.value.status == spw.SPW_ERR_FORMAT
    small = torch.empty(hdr.bytes_total - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(spw.SpwError) as e:
        spw.spw_compress(dev(W), dev(mask), buf=small)
    assert e.value.status == spw.SPW_ERR_BUFFER_TOO_SMALL
    corrupt = buf.clone()
    corrupt[0] = 0
    with pytest.raises(spw.SpwError) as e:
        spw.spw_format_read(corrupt)
    assert e.value.status == spw.SPW_ERR_FORMAT
