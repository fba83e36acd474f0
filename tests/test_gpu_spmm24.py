"""GPU parity of the 2:4 + residual prefill (tcgen05.mma.sp) against the fp64 oracle.

spw_split24 is index and byte work: its residual mask must equal the oracle split bit for
bit, and its 2:4 buffer, read back through the layout include/spw.h documents, must
hold exactly the oracle's 2:4 part.  spw_spmm24 is a product: max|Y - Y_ref| /
max|Y_ref| <= 5e-3 against the oracle's masked product (S + R = W masked), exact where
the result is exact; full-size shapes on seeded sampled rows."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import TOL, dev, host, needs_gpu, padded_rows
import spmm_tiled_column_b200 as spw

pytestmark = [pytest.mark.gpu, needs_gpu]


def structured_mask(N, K, *seed):
    """At most two kept weights in every group of four columns (a 2:4 mask)."""
    return workloads.structured24_mask(N, K, *seed)


def read_s24(buf: np.ndarray, N: int, K: int) -> np.ndarray:
    """Dense N x K fp16 bits of the 2:4 part, decoded from the documented layout."""
    nk, ns = -(-K // 64), -(-N // 64)
    T = nk * ns
    S = np.zeros((ns * 64, nk * 64), np.uint16)
    vals = buf[:T * 4096].view(np.uint16).reshape(T, 64, 32)
    meta = buf[T * 4096:T * 5120].view(np.uint32).reshape(T, 64, 4).transpose(0, 2, 1)
    assert not meta[:, 2:].any()
    pad = buf[T * 5120:T * 5120 + 1024].view(np.uint32).reshape(64, 4)
    assert (pad[:, :2] == 0x44444444).all() and not pad[:, 2:].any()
    for t in range(T):
        s, kt = divmod(t, nk)
        for r in range(64):
            sw = (r >> 1) & 3
            row = np.concatenate([vals[t, r, 8 * (c ^ sw):8 * (c ^ sw) + 8] for c in range(4)])
            for j in range(2):
                for k1 in range(2):
                    L = 16 * (r >> 4) + 8 * k1 + (r & 7)
                    half = (int(meta[t, j, L]) >> (16 * ((r >> 3) & 1))) & 0xFFFF
                    for g in range(4):
                        nib = (half >> (4 * g)) & 0xF
                        i0, i1 = nib & 3, nib >> 2
                        assert i0 < i1
                        G = 8 * j + 4 * k1 + g
                        S[64 * s + r, 64 * kt + 4 * G + i0] = row[2 * G]
                        S[64 * s + r, 64 * kt + 4 * G + i1] = row[2 * G + 1]
    return S[:N, :K]


@pytest.mark.parametrize("N,K,density", [(64, 64, 0.5), (130, 200, 0.6), (300, 1000, 0.5), (64, 64, 1.0)])
def test_split_matches_oracle_exactly(N, K, density):
    W = workloads.weight(N, K, "s24-split")
    W[0, :4] = [-0.0, 1.0, -2.0, 0.5]
    mask = workloads.random_mask(N, K, density, "s24-split")
    s24, mask_r = spw.spw_split24(dev(W), dev(mask))
    torch.cuda.synchronize()
    ms, mr = oracle.split24(mask)
    np.testing.assert_array_equal(host(mask_r), mr)
    S = read_s24(host(s24), N, K)
    np.testing.assert_array_equal(S, np.where(ms != 0, W.view(np.uint16), np.uint16(0)))


def run24(W, mask, X):
    lin = spw.SparseLinear24(dev(W), dev(mask))
    M, K = X.shape
    Xd = dev(X) if M == 1 or K % 8 == 0 else padded_rows(X, -(-K // 8) * 8)
    Y = lin.spmm(Xd)
    torch.cuda.synchronize()
    assert spw.spw_last_device_status() == spw.SPW_OK
    return host(Y).astype(np.float64), lin


@pytest.mark.parametrize("N,K,M,kind", [
    (128, 64, 64, "structured"), (128, 64, 64, "random"), (256, 512, 16, "random"),
    (300, 200, 37, "random"), (513, 1000, 600, "random"), (65, 130, 300, "structured"),
    (1000, 4096, 256, "structured"), (128, 4160, 64, "dense")])
def test_parity_small(N, K, M, kind):
    W = workloads.weight(N, K, "s24")
    if kind == "structured":
        mask = structured_mask(N, K, "s24")
    elif kind == "dense":
        mask = np.ones((N, K), np.uint8)
    else:
        mask = workloads.random_mask(N, K, 0.5, "s24")
    X = workloads.normal_act(M, K, "s24")
    Y, _ = run24(W, mask, X)
    assert oracle.rel_err(Y, oracle.spmm(W, mask, X)) <= TOL, (N, K, M, kind)


def test_identity_exact_and_structured_residual_empty():
    K = 384
    X = workloads.normal_act(300, K, "s24-id")
    Y, lin = run24(np.eye(K, dtype=np.float16), np.eye(K, dtype=np.uint8), X)
    np.testing.assert_array_equal(Y, X.astype(np.float64))
    assert lin.hdr_r.nnz == 0
    W = workloads.weight(200, K, "s24-z")
    Y, _ = run24(W, np.zeros((200, K), np.uint8), X)
    assert not Y.any()


def test_all_ones_mask_matches_cublas():
    # every group keeps four: two on the sparse tensor cores, two in the residual
    N, K, M = 512, 1024, 512
    W = workloads.weight(N, K, "s24-ones")
    X = workloads.normal_act(M, K, "s24-ones")
    Y, _ = run24(W, np.ones((N, K), np.uint8), X)
    Wd, Xd = dev(W), dev(X)
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    ref = host(torch.matmul(Xd, Wd.t())).astype(np.float64)
    assert oracle.rel_err(Y, ref) <= TOL
    assert oracle.rel_err(Y, oracle.spmm(W, np.ones((N, K), np.uint8), X)) <= TOL


@pytest.mark.parametrize("name,kind", [("q", "random"), ("q", "structured")])
def test_llama7b_prefill_sampled_rows(name, kind):
    N, K = workloads.LLAMA7B_LAYERS[name]
    M = 2048
    layer = workloads.pruned_layer(name, N, K, 0.5, "s24-7b")
    mask = layer.mask if kind == "random" else structured_mask(N, K, "s24-7b")
    X = workloads.normal_act(M, K, "s24-7b")
    Y, _ = run24(layer.W, mask, X)
    rows = workloads.rng("s24-7b-rows", name, kind).choice(M, size=128, replace=False).astype(np.int32)
    assert oracle.rel_err(Y[rows], oracle.spmm(layer.W, mask, X, rows=rows)) <= TOL
