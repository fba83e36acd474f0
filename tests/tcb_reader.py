"""Test helpers: an independent numpy reader of TCB v1 buffers and the golden parser.

The reader re-derives the dense masked weight from a buffer with vectorised numpy (a
different route from the oracle's loops), following the TCB v1 definition:
64-row strips, 64-column tiles, u64 column bitmaps, values column-major per tile in
set-bit order, tiles padded to 16 bytes, sections 256-byte aligned.
"""
from __future__ import annotations

import os

import numpy as np

HEADER_FIELDS = [  # (name, offset, numpy dtype)
    ("magic", 0, np.uint32), ("version", 4, np.uint32), ("N", 8, np.uint32),
    ("K", 12, np.uint32), ("TN", 16, np.uint32), ("TK", 20, np.uint32),
    ("n_strips", 24, np.uint32), ("n_ktiles", 28, np.uint32), ("nnz", 32, np.uint64),
    ("bytes_total", 40, np.uint64), ("off_bitmaps", 48, np.uint64),
    ("off_tileptr", 56, np.uint64), ("off_values", 64, np.uint64),
    ("max_tile_units", 72, np.uint32),
]


def header(buf: np.ndarray) -> dict:
    buf = np.asarray(buf, dtype=np.uint8)
    return {name: int(buf[off:off + np.dtype(dt).itemsize].view(dt)[0])
            for name, off, dt in HEADER_FIELDS}


def sections(buf: np.ndarray):
    h = header(buf)
    S, T = h["n_strips"], h["n_ktiles"]
    bm = buf[h["off_bitmaps"]:h["off_bitmaps"] + 8 * S * T * 64].view(np.uint64).reshape(S, T * 64)
    tp = buf[h["off_tileptr"]:h["off_tileptr"] + 4 * (S * T + 1)].view(np.uint32)
    vals = buf[h["off_values"]:h["bytes_total"]].view(np.uint16)
    return h, bm, tp, vals


def bit_matrix(bm: np.ndarray, N: int, K: int) -> np.ndarray:
    """Expand u64 column bitmaps [S, T*64] into a bool matrix [N, K]."""
    S = bm.shape[0]
    bits = ((bm[:, None, :] >> np.arange(64, dtype=np.uint64)[None, :, None]) & np.uint64(1))
    full = bits.astype(bool).reshape(S * 64, -1)  # row 64 s + r, column k
    return full[:N, :K], full


def dense_from_buffer(buf: np.ndarray) -> np.ndarray:
    """Dense masked weight (uint16 bits) read back from a TCB v1 buffer."""
    h, bm, tp, vals = sections(buf)
    N, K, S, T = h["N"], h["K"], h["n_strips"], h["n_ktiles"]
    _, full = bit_matrix(bm, N, K)
    out = np.zeros((S * 64, T * 64), dtype=np.uint16)
    for s in range(S):
        for kt in range(T):
            t = s * T + kt
            tile = full[64 * s:64 * s + 64, 64 * kt:64 * kt + 64]
            # column-major order of set bits: transpose, then row-major nonzero
            cols, rows = np.nonzero(tile.T)
            n = cols.size
            seg = vals[8 * tp[t]:8 * tp[t] + n]
            out[64 * s + rows, 64 * kt + cols] = seg
    return out[:N, :K]


def padding_is_zero(buf: np.ndarray) -> bool:
    """Every byte outside the defined fields and the stored values is zero."""
    h, bm, tp, vals = sections(buf)
    S, T = h["n_strips"], h["n_ktiles"]
    used = np.zeros(h["bytes_total"], dtype=bool)
    used[:76] = True
    used[h["off_bitmaps"]:h["off_bitmaps"] + 8 * S * T * 64] = True
    used[h["off_tileptr"]:h["off_tileptr"] + 4 * (S * T + 1)] = True
    counts = np.array([int(sum(bin(int(w)).count("1") for w in bm[s, 64 * kt:64 * kt + 64]))
                       for s in range(S) for kt in range(T)], dtype=np.int64)
    for t in range(S * T):
        start = h["off_values"] + 16 * int(tp[t])
        used[start:start + 2 * int(counts[t])] = True
    return not np.any(np.asarray(buf[:h["bytes_total"]])[~used])


def parse_golden(path: str | None = None) -> list[dict]:
    path = path or os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                "tcb_v1_examples.txt")
    cases, cur = [], None
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest, "bitmap": {}}
        elif key == "end":
            cases.append(cur)
            cur = None
        elif key in ("N", "K"):
            cur[key] = int(rest)
        elif key in ("W", "dense"):
            cur[key] = np.array([[int(v, 16) for v in row.split()] for row in rest.split("/")],
                                dtype=np.uint16)
        elif key == "mask":
            cur[key] = np.array([[int(v) for v in row.split()] for row in rest.split("/")],
                                dtype=np.uint8)
        elif key == "kept":
            cur[key] = [(int(a), int(b), int(c, 16)) for a, b, c in
                        (g.split() for g in rest.split("/"))]
        elif key == "header":
            cur[key] = {k: int(v, 16) if k == "magic" else int(v)
                        for k, v in (kv.split("=") for kv in rest.split())}
        elif key == "bitmap":
            s, k, w = rest.split()
            cur["bitmap"][(int(s), int(k))] = int(w, 16)
        elif key == "tileptr":
            cur[key] = [int(v) for v in rest.split()]
        elif key == "values":
            cur[key] = np.array([int(v, 16) for v in rest.replace("/", " ").split()],
                                dtype=np.uint16)
        else:
            raise ValueError(f"unknown golden key {key!r}")
    return cases


def golden_inputs(case: dict, seed: int = 7):
    """(W bits, mask) for a golden case; sparse cases get random bits where dropped."""
    N, K = case["N"], case["K"]
    if "W" in case:
        return case["W"].copy(), case["mask"].copy()
    r = np.random.default_rng(seed)
    W = r.integers(0, 0x7C00, size=(N, K), dtype=np.uint16)  # finite junk, must be ignored
    mask = np.zeros((N, K), dtype=np.uint8)
    for n, k, bits in case["kept"]:
        W[n, k] = bits
        mask[n, k] = 1
    return W, mask
