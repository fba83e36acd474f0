"""Seeded synthetic inputs for the sparse-weight SpMV / SpMM workloads.

This module builds inputs only: weights, pruning masks and activations with the shapes,
value distributions and sparsity structure of the pages' workloads (Llama-7B / 13B
linear-layer shapes, fp16 weights from N(0, 0.02), moderate unstructured sparsity,
activations with zeroed entries).  It holds none of the method's arithmetic (no format
encoding, no column selection, no products); both the oracle-side tests and the CUDA-side
tests and benchmark draw their inputs from here.

Everything is numpy on the host.  Values are drawn in float64 from a PCG64 generator
and rounded to fp16 by numpy (IEEE round-to-nearest-even).  Seeds are derived from a
description string with SHA-256, so that every (config, shape, sparsity, batch) has its
own stream that does not depend on Python's hash randomisation.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass

import numpy as np

# Llama-7B and Llama-13B linear-layer shapes as (N, K) = (out_features, in_features).
LLAMA7B_LAYERS = {
    "q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096), "o": (4096, 4096),
    "gate": (11008, 4096), "up": (11008, 4096), "down": (4096, 11008),
}
LLAMA13B_SHAPES = {"attn": (5120, 5120), "gate_up": (13824, 5120), "down": (5120, 13824)}


def seed_of(*parts) -> int:
    """Stable 64-bit seed from a description, e.g. seed_of('cfg2', 4096, 4096, 0.5, 1)."""
    h = hashlib.sha256("|".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:8], "little")


def rng(*parts) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed_of(*parts)))


def weight(N: int, K: int, *seed_parts, std: float = 0.02) -> np.ndarray:
    """fp16 N x K weight drawn from N(0, std^2)."""
    return (rng("weight", N, K, *seed_parts).standard_normal((N, K)) * std).astype(np.float16)


def magnitude_mask(W: np.ndarray, sparsity: float) -> np.ndarray:
    """Per-row magnitude pruning mask (uint8, 1 = kept).

    In every row the K - floor(sparsity * K) entries of largest |w| are kept; ties go to
    the lower column index.  |w| is compared on the fp16 values: the key of an entry is
    its fp16 magnitude bits (monotone in |w|) followed by the reversed column index, so
    keys are unique and the kept set is exactly {key >= the keep-th largest key}.
    """
    W = np.ascontiguousarray(W, dtype=np.float16)
    N, K = W.shape
    drop = int(np.floor(sparsity * K + 1e-9))
    keep = K - drop
    mask = np.zeros((N, K), dtype=np.uint8)
    if keep == 0:
        return mask
    mag = (W.view(np.uint16) & np.uint16(0x7FFF)).astype(np.int64)
    rev = (K - 1 - np.arange(K, dtype=np.int64))[None, :]
    for r0 in range(0, N, 1024):   # row blocks bound the temporary memory
        key = (mag[r0:r0 + 1024] << 20) | rev
        kth = np.partition(key, K - keep, axis=1)[:, K - keep]
        mask[r0:r0 + 1024] = key >= kth[:, None]
    return mask


def random_mask(N: int, K: int, density: float, *seed_parts) -> np.ndarray:
    """Independent Bernoulli(density) mask, uint8."""
    return (rng("mask", N, K, density, *seed_parts).random((N, K)) < density).astype(np.uint8)


def normal_act(B: int, K: int, *seed_parts) -> np.ndarray:
    """fp16 B x K activations from N(0, 1)."""
    return rng("act", B, K, *seed_parts).standard_normal((B, K)).astype(np.float16)


def silu_gate_up_act(B: int, K: int, *seed_parts) -> np.ndarray:
    """fp16 down-projection input SiLU(g) * u with g, u ~ N(0, 1), computed in fp64."""
    r = rng("silu", B, K, *seed_parts)
    g = r.standard_normal((B, K))
    u = r.standard_normal((B, K))
    return (g / (1.0 + np.exp(-g)) * u).astype(np.float16)


def zero_smallest(x: np.ndarray, frac: float) -> tuple[np.ndarray, np.ndarray]:
    """Zero exactly floor(frac * K) entries of smallest |x| in every row (ties: lower index).

    Returns (zeroed copy, per-row threshold t = smallest surviving |x|, or inf when every
    entry of the row was zeroed).
    """
    x = np.array(x, dtype=np.float16, copy=True)
    B, K = x.shape
    nz = int(np.floor(frac * K + 1e-9))
    t = np.full(B, np.inf)
    if nz == 0:
        t[:] = np.min(np.abs(x.astype(np.float64)), axis=1)
        return x, t
    mag = np.abs(x.astype(np.float64))
    order = np.argsort(mag, axis=1, kind="stable")
    for b in range(B):
        x[b, order[b, :nz]] = 0
        if nz < K:
            t[b] = mag[b, order[b, nz]]
    return x, t


def zero_random(x: np.ndarray, frac: float, *seed_parts) -> np.ndarray:
    """Zero exactly floor(frac * K) entries per row at seeded random positions."""
    x = np.array(x, dtype=np.float16, copy=True)
    B, K = x.shape
    nz = int(np.floor(frac * K + 1e-9))
    r = rng("zero_random", B, K, frac, *seed_parts)
    for b in range(B):
        x[b, r.permutation(K)[:nz]] = 0
    return x


@dataclass
class Layer:
    """One pruned linear layer: fp16 weight, its mask, and a description."""
    name: str
    W: np.ndarray
    mask: np.ndarray
    sparsity: float

    @property
    def shape(self):
        return self.W.shape


def pruned_layer(name: str, N: int, K: int, sparsity: float, *seed_parts) -> Layer:
    """N(0, 0.02) fp16 weight with a per-row magnitude mask at the given sparsity."""
    W = weight(N, K, name, sparsity, *seed_parts)
    return Layer(name, W, magnitude_mask(W, sparsity), sparsity)


def decode_act(layer_name: str, B: int, K: int, act_sparsity: float, *seed_parts):
    """Decode-step activations for a Llama linear: SiLU(g) * u for the down projection,
    N(0, 1) otherwise, with the smallest floor(a * K) entries of every row zeroed."""
    if layer_name == "down":
        x = silu_gate_up_act(B, K, layer_name, *seed_parts)
    else:
        x = normal_act(B, K, layer_name, *seed_parts)
    zx, t = zero_smallest(x, act_sparsity)
    return zx, t


def domain_tokens(M: int, K: int, n_domains: int, block_density: float, *seed_parts,
                  silu: bool = False) -> tuple[np.ndarray, np.ndarray]:
    """Prefill tokens drawn from n_domains "domains" whose channel use differs.

    Each domain keeps a seeded random subset of the 64-column channel blocks (each block
    with probability block_density, at least one block); every token belongs to one
    domain (drawn uniformly, tokens interleaved in random order), takes N(0, 1) values --
    SiLU(g) * u with g, u ~ N(0, 1) when silu is set -- and is zero in every block its
    domain does not use.  Returns (fp16 M x K tokens, domain id per token)."""
    r = rng("domains", M, K, n_domains, block_density, *seed_parts)
    nk = -(-K // 64)
    blocks = r.random((n_domains, nk)) < block_density
    for d in range(n_domains):
        if not blocks[d].any():
            blocks[d, r.integers(nk)] = True
    dom = r.integers(0, n_domains, size=M)
    if silu:
        g = r.standard_normal((M, K))
        u = r.standard_normal((M, K))
        x = g / (1.0 + np.exp(-g)) * u
    else:
        x = r.standard_normal((M, K))
    cols = np.repeat(blocks, 64, axis=1)[:, :K]
    x[~cols[dom]] = 0.0
    return x.astype(np.float16), dom


def structured24_mask(N: int, K: int, *seed_parts, extra: float = 0.0,
                      count: int | None = None, dense_channels: float = 0.0) -> np.ndarray:
    """A 2:4-structured mask: in every group of four columns of a row, 0, 1 or 2 kept
    positions (uniform count; exactly `count` when given; seeded random positions).
    Then, outside the 2:4 pattern: each dropped position is kept with probability
    `extra`, and a seeded `dense_channels` fraction of the input channels (columns) is
    kept whole -- outlier features left unpruned -- so that the residual of a 2:4 +
    residual split sits in those columns."""
    r = rng("mask24", N, K, extra, count, dense_channels, *seed_parts)
    G = -(-K // 4)
    cnt = (r.integers(0, 3, size=(N, G, 1)) if count is None
           else np.full((N, G, 1), int(count)))
    rank = np.argsort(np.argsort(r.random((N, G, 4)), axis=2), axis=2)
    keep = (rank < cnt).reshape(N, 4 * G)[:, :K]
    if extra > 0:
        keep |= r.random((N, K)) < extra
    if dense_channels > 0:
        keep[:, r.permutation(K)[:max(1, int(round(dense_channels * K)))]] = True
    return keep.astype(np.uint8)
