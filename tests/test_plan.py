"""Host-side launch plan of the prefill / tensor-core decode kernel (CPU, no launch).

spw_spmm_plan reports, for a format, M and an SM count, the token tile, how the output
tiles are split along K and the workspace.  The kernel indexes its CTAs and partial
tiles from exactly these numbers, so the invariants below are the ones its indexing
relies on."""
import os

import pytest
import torch

import spmm_tiled_column_b200 as spw


@pytest.fixture(params=[0, 1], ids=["one-cta-tiles", "pair-tiles"])
def pair_env(request, monkeypatch):
    """Plans with the default one-CTA tiles and with SM-pair tiles (SPW_SPMM_PAIR=1, read
    by the library at plan time)."""
    if request.param:
        monkeypatch.setenv("SPW_SPMM_PAIR", "1")
    else:
        monkeypatch.delenv("SPW_SPMM_PAIR", raising=False)
    return request.param


def header(N, K, units=300):
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


def test_llama7b_prefill_runs_whole_tiles(monkeypatch):
    monkeypatch.delenv("SPW_SPMM_PAIR", raising=False)
    p = spw.spw_spmm_plan(header(4096, 4096), 2048, 148)
    assert p["cta_pair"] == 0
    assert (p["token_tile"], p["token_tiles"], p["weight_tiles"]) == (512, 4, 32)
    assert (p["k_parts"], p["whole_tiles"], p["ctas"], p["workspace_bytes"]) == (1, 128, 128, 0)


def test_llama7b_prefill_pair_tiles(monkeypatch):
    monkeypatch.setenv("SPW_SPMM_PAIR", "1")
    # 256-row tiles on SM pairs: 16 weight tiles x 4 token tiles = 64 pair tiles, one wave
    # on the 74 SM pairs of 148 SMs
    p = spw.spw_spmm_plan(header(4096, 4096), 2048, 148)
    assert p["cta_pair"] == 1
    assert (p["token_tile"], p["token_tiles"], p["weight_tiles"]) == (512, 4, 16)
    assert (p["k_parts"], p["whole_tiles"], p["ctas"], p["workspace_bytes"]) == (1, 64, 128, 0)


def test_second_wave_tiles_are_split(monkeypatch):
    monkeypatch.delenv("SPW_SPMM_PAIR", raising=False)
    # 160 output tiles on 148 SMs: 148 run whole, the 12 left over in K parts
    p = spw.spw_spmm_plan(header(5120, 5120), 2048, 148)
    assert p["whole_tiles"] == 148 and p["k_parts"] > 1
    assert p["ctas"] == 148 + 12 * p["k_parts"]
    assert p["workspace_bytes"] == 256 + 12 * p["k_parts"] * 512 * 128 * 4


def test_second_wave_pair_tiles_are_split(monkeypatch):
    monkeypatch.setenv("SPW_SPMM_PAIR", "1")
    # 80 pair tiles on 74 SM pairs: 74 run whole, the 6 left over in K parts; each of a
    # split tile's two 128-row halves has its own counter and partial tiles
    p = spw.spw_spmm_plan(header(5120, 5120), 2048, 148)
    assert p["cta_pair"] == 1 and p["weight_tiles"] == 20
    assert p["whole_tiles"] == 74 and p["k_parts"] > 1
    assert p["ctas"] == 2 * (74 + 6 * p["k_parts"])
    assert p["workspace_bytes"] == 256 + 12 * p["k_parts"] * 512 * 128 * 4


def test_one_cta_tiles_below_256_tokens(monkeypatch):
    monkeypatch.setenv("SPW_SPMM_PAIR", "1")
    p = spw.spw_spmm_plan(header(4096, 4096), 255, 148)
    assert p["cta_pair"] == 0 and p["weight_tiles"] == 32


def test_small_token_counts_split_every_tile():
    # decode-sized batches: few output tiles, so K is split across all of them
    p = spw.spw_spmm_plan(header(4096, 4096), 16, 148)
    assert p["whole_tiles"] == 0 and p["k_parts"] > 1
    assert p["ctas"] == 32 * p["k_parts"] <= 2 * 148


@pytest.mark.parametrize("sms", [8, 132, 148])
@pytest.mark.parametrize("N,K", [(128, 64), (1000, 512), (4096, 4096), (5120, 5120), (11008, 4096),
                                 (5120, 13824), (300, 100)])
@pytest.mark.parametrize("M", [1, 16, 100, 512, 2048, 5000])
def test_plan_invariants(N, K, M, sms, pair_env):
    h = header(N, K)
    p = spw.spw_spmm_plan(h, M, sms)
    pair = p["cta_pair"]
    assert pair == (1 if (pair_env and M >= 256 and N > 128) else 0)
    mt, tiles = p["token_tile"], p["token_tiles"] * p["weight_tiles"]
    assert p["weight_tiles"] == -(-N // (256 if pair else 128))
    assert mt % 16 == 0 and 16 <= mt <= 512 and mt * p["token_tiles"] >= M
    if pair:
        assert mt >= 128  # each CTA loads mt / 2 tokens per MMA half: whole 8-row atoms
    assert 1 <= p["k_parts"] <= max(1, h.n_ktiles)
    assert 0 <= p["whole_tiles"] <= tiles
    assert p["ctas"] == (p["whole_tiles"] + (tiles - p["whole_tiles"]) * p["k_parts"]) * (2 if pair else 1)
    split = (tiles - p["whole_tiles"]) * (2 if pair else 1)  # 128-row halves with partials
    if p["k_parts"] == 1:
        assert split == 0 and p["workspace_bytes"] == 0
    else:
        assert split > 0
        assert p["workspace_bytes"] == -(-4 * split // 256) * 256 + 4 * split * p["k_parts"] * mt * 128
    slots = sms // 2 if pair else sms
    if 0 < p["whole_tiles"] < tiles:  # the hybrid only for more than one and fewer than two waves
        assert slots < tiles < 2 * slots


def test_plan_errors():
    h = header(256, 256)
    with pytest.raises(spw.SpwError) as e:
        spw.spw_spmm_plan(h, 0, 148)
    assert e.value.status == spw.SPW_ERR_INVALID_ARG
    bad = header(256, 256)
    bad.magic = 0
    with pytest.raises(spw.SpwError) as e:
        spw.spw_spmm_plan(bad, 64, 148)
    assert e.value.status == spw.SPW_ERR_FORMAT
    if not torch.cuda.is_available():  # no device to ask for its SM count
        with pytest.raises(spw.SpwError) as e:
            spw.spw_spmm_plan(h, 64, 0)
        assert e.value.status == spw.SPW_ERR_CUDA


@pytest.mark.parametrize("sms", [8, 148])
@pytest.mark.parametrize("N,K", [(128, 64), (1000, 512), (4096, 4096), (4096, 11008), (300, 100)])
@pytest.mark.parametrize("M", [1, 16, 100, 512, 2048, 5000])
def test_2of4_and_token_plans(N, K, M, sms, monkeypatch):
    monkeypatch.setenv("SPW_SPMM_PAIR", "1")  # neither product uses SM-pair tiles
    h = header(N, K)
    p24 = spw.spw_spmm24_plan(h, M, sms)
    assert p24["cta_pair"] == 0 and p24["weight_tiles"] == -(-N // 128)
    # tensor memory holds the accumulators and the metadata columns: <= 256 tokens
    mt = p24["token_tile"]
    assert mt % 16 == 0 and 16 <= mt <= 256 and mt * p24["token_tiles"] >= M
    tiles = p24["token_tiles"] * p24["weight_tiles"]
    assert p24["ctas"] == p24["whole_tiles"] + (tiles - p24["whole_tiles"]) * p24["k_parts"]
    pt = spw.spw_spmm_tokens_plan(h, M, sms)
    assert pt["cta_pair"] == 0 and pt["token_tile"] <= 512
    # the grouped input, permutation, tile signatures and grouping scratch follow the
    # product's own workspace
    words = ((K + 63) // 64 + 63) // 64
    assert pt["workspace_bytes"] >= 2 * M * (-(-K // 8) * 8) + 4 * M + 8 * words * pt["token_tiles"]


def test_token_plan_limits():
    with pytest.raises(spw.SpwError) as e:
        spw.spw_spmm_tokens_plan(header(256, 16448), 64, 148)
    assert e.value.status == spw.SPW_ERR_UNSUPPORTED
    with pytest.raises(spw.SpwError) as e:
        spw.spw_spmm_tokens_plan(header(256, 256), 16385, 148)
    assert e.value.status == spw.SPW_ERR_UNSUPPORTED
