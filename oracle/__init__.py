"""Oracle for the sparse-weight SpMV / SpMM path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this package.  The product (``spmm_tiled_column_b200``) never
imports it and has no CPU fallback.

The arithmetic lives in ``oracle.c`` (plain single-threaded C, fp64).  This module only
compiles it with gcc into ``liboracle.so`` and marshals numpy arrays in and out.  Each C
function's header comment names the page passage it follows; the pins that tie it to
facts outside itself are in ``tests/test_oracle_*.py``.

Parity status: every function here is pinned (no "parity unpinned" entries).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK = 0
ERR_ARG = 1
ERR_BUFFER_TOO_SMALL = 3
ERR_FORMAT = 4


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (skipped when the library is newer).

    ORACLE_LIB_OVERRIDE names another build of oracle.c to load instead; only
    tests/test_oracle_mutations.py sets it, in child processes that check that the pins
    reject copies of the oracle with a planted mistake.
    """
    override = os.environ.get("ORACLE_LIB_OVERRIDE")
    if override:
        return override
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                    "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i, u64, f = ctypes.c_int, ctypes.c_uint64, ctypes.c_float
        lib.orc_half_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_half_to_double.restype = ctypes.c_double
        lib.orc_tcb_query.argtypes = [P, i, i, i, P, P]
        lib.orc_tcb_encode.argtypes = [P, i, P, i, i, i, P, u64]
        lib.orc_tcb_decode.argtypes = [P, u64, P, i]
        lib.orc_select_threshold.argtypes = [P, i, i, i, f, P, P]
        lib.orc_select_topk.argtypes = [P, i, i, i, i, P, P]
        lib.orc_spmv.argtypes = [P, i, P, i, i, i, P, i, i, f, P, P]
        lib.orc_spmm.argtypes = [P, i, P, i, i, i, P, i, i, P, i, P]
        lib.orc_double_to_half.argtypes = [ctypes.c_double]
        lib.orc_double_to_half.restype = ctypes.c_uint16
        lib.orc_round_to_half.argtypes = [P, ctypes.c_int64, P]
        lib.orc_silu_mul.argtypes = [P, P, i, i, i, P]
        lib.orc_spmm_tokens.argtypes = [P, i, P, i, i, i, P, i, i, f, P, i, P]
        lib.orc_token_groups.argtypes = [P, i, i, i, f, i, P, P]
        lib.orc_split24.argtypes = [P, i, i, i, P, P]
        for name in ("orc_tcb_query", "orc_tcb_encode", "orc_tcb_decode",
                     "orc_select_threshold", "orc_select_topk", "orc_spmv", "orc_spmm",
                     "orc_round_to_half", "orc_silu_mul", "orc_spmm_tokens",
                     "orc_token_groups", "orc_split24"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _half_bits(a: np.ndarray) -> np.ndarray:
    """fp16 array (or its uint16 bit view) -> C-contiguous uint16 bits."""
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16 or uint16 bits, got {a.dtype}")
    return np.ascontiguousarray(a)


def _check(rc: int, what: str):
    if rc != OK:
        raise OracleError(f"{what} returned status {rc}")


def half_to_double(bits: int) -> float:
    return _load().orc_half_to_double(int(bits))


def tcb_query(mask: np.ndarray) -> tuple[int, int]:
    """(bytes_total, nnz) of the TCB v1 buffer for an N x K mask."""
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    N, K = mask.shape
    nbytes, nnz = ctypes.c_uint64(), ctypes.c_uint64()
    _check(_load().orc_tcb_query(_ptr(mask), N, K, K, ctypes.byref(nbytes),
                                 ctypes.byref(nnz)), "orc_tcb_query")
    return nbytes.value, nnz.value


def tcb_encode(W: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Reference TCB v1 buffer (uint8 array of exactly bytes_total bytes)."""
    Wb = _half_bits(W)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    N, K = Wb.shape
    assert mask.shape == (N, K)
    nbytes, _ = tcb_query(mask)
    buf = np.zeros(nbytes, dtype=np.uint8)
    _check(_load().orc_tcb_encode(_ptr(Wb), K, _ptr(mask), K, N, K, _ptr(buf), nbytes),
           "orc_tcb_encode")
    return buf


def tcb_decode(buf: np.ndarray) -> np.ndarray:
    """Dense masked weight (fp16 bits, uint16 N x K) from a TCB v1 buffer."""
    buf = np.ascontiguousarray(buf, dtype=np.uint8)
    if buf.size < 16:
        raise OracleError("buffer shorter than a header")
    N = int(buf[8:12].view(np.uint32)[0])
    K = int(buf[12:16].view(np.uint32)[0])
    out = np.zeros((max(N, 1), max(K, 1)), dtype=np.uint16)
    _check(_load().orc_tcb_decode(_ptr(buf), buf.size, _ptr(out), out.shape[1]),
           "orc_tcb_decode")
    return out


def select_threshold(x: np.ndarray, t: float) -> tuple[np.ndarray, int]:
    """(act_bits uint32[ceil(K/32)], count) for the threshold rule over a B x K batch."""
    xb = _half_bits(np.atleast_2d(x))
    B, K = xb.shape
    bits = np.zeros((K + 31) // 32, dtype=np.uint32)
    count = ctypes.c_uint32()
    _check(_load().orc_select_threshold(_ptr(xb), B, K, K, ctypes.c_float(t), _ptr(bits),
                                        ctypes.byref(count)), "orc_select_threshold")
    return bits, count.value


def select_topk(x: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """(act_bits, ascending index list) of the top-k columns by summed |x|."""
    xb = _half_bits(np.atleast_2d(x))
    B, K = xb.shape
    bits = np.zeros((K + 31) // 32, dtype=np.uint32)
    idx = np.zeros(max(k, 1), dtype=np.uint32)
    _check(_load().orc_select_topk(_ptr(xb), B, K, K, int(k), _ptr(bits), _ptr(idx)),
           "orc_select_topk")
    return bits, idx[:k]


def spmv(W: np.ndarray, mask: np.ndarray, x: np.ndarray, t: float = 0.0,
         act_bits: np.ndarray | None = None) -> np.ndarray:
    """fp64 B x N decode result y_b = W_masked . x~_b."""
    Wb = _half_bits(W)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    xb = _half_bits(np.atleast_2d(x))
    N, K = Wb.shape
    B = xb.shape[0]
    assert xb.shape[1] == K and mask.shape == (N, K)
    if act_bits is not None:
        act_bits = np.ascontiguousarray(act_bits, dtype=np.uint32)
        assert act_bits.size >= (K + 31) // 32
    y = np.zeros((B, N), dtype=np.float64)
    _check(_load().orc_spmv(_ptr(Wb), K, _ptr(mask), K, N, K, _ptr(xb), B, K,
                            ctypes.c_float(t), _ptr(act_bits), _ptr(y)), "orc_spmv")
    return y


def spmm(W: np.ndarray, mask: np.ndarray, X: np.ndarray,
         rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 prefill result Y = X . W_masked^T (only the listed rows of X if given)."""
    Wb = _half_bits(W)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    Xb = _half_bits(np.atleast_2d(X))
    N, K = Wb.shape
    M = Xb.shape[0]
    assert Xb.shape[1] == K and mask.shape == (N, K)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        n_rows = rows.size
    else:
        n_rows = M
    Y = np.zeros((n_rows, N), dtype=np.float64)
    _check(_load().orc_spmm(_ptr(Wb), K, _ptr(mask), K, N, K, _ptr(Xb), M, K, _ptr(rows),
                            n_rows, _ptr(Y)), "orc_spmm")
    return Y


def spmm_tokens(W: np.ndarray, mask: np.ndarray, X: np.ndarray, t: float,
                rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 prefill result with a per-token index set: Y = X~ . W_masked^T, where x~[m,k]
    keeps X[m,k] only when the threshold rule keeps it (only the listed rows if given)."""
    Wb = _half_bits(W)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    Xb = _half_bits(np.atleast_2d(X))
    N, K = Wb.shape
    M = Xb.shape[0]
    assert Xb.shape[1] == K and mask.shape == (N, K)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        n_rows = rows.size
    else:
        n_rows = M
    Y = np.zeros((n_rows, N), dtype=np.float64)
    _check(_load().orc_spmm_tokens(_ptr(Wb), K, _ptr(mask), K, N, K, _ptr(Xb), M, K,
                                   ctypes.c_float(t), _ptr(rows), n_rows, _ptr(Y)),
           "orc_spmm_tokens")
    return Y


def token_groups(X: np.ndarray, t: float, token_tile: int) -> tuple[np.ndarray, np.ndarray]:
    """Token grouping: (perm uint32[M], tile_sig uint64[ceil(M/T), words]).

    perm lists the tokens sorted by k-tile signature (ties by index); tile_sig[j] is the
    OR of the signatures of positions j*T .. (j+1)*T-1."""
    Xb = _half_bits(np.atleast_2d(X))
    M, K = Xb.shape
    words = (-(-K // 64) + 63) // 64
    tiles = -(-M // token_tile)
    perm = np.zeros(M, dtype=np.uint32)
    tile_sig = np.zeros((tiles, words), dtype=np.uint64)
    _check(_load().orc_token_groups(_ptr(Xb), M, K, K, ctypes.c_float(t), int(token_tile),
                                    _ptr(perm), _ptr(tile_sig)), "orc_token_groups")
    return perm, tile_sig


def split24(mask: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """2:4 + residual split of a mask: (mask_s, mask_r), uint8 N x K each; in every
    group of four columns of a row the first two kept weights go to mask_s, the rest to
    mask_r."""
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    N, K = mask.shape
    ms = np.zeros((N, K), np.uint8)
    mr = np.zeros((N, K), np.uint8)
    _check(_load().orc_split24(_ptr(mask), K, N, K, _ptr(ms), _ptr(mr)), "orc_split24")
    return ms, mr


def round_to_half(v: np.ndarray) -> np.ndarray:
    """fp64 values -> binary16 (float16 array), round to nearest, ties to even."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.zeros(v.shape, dtype=np.uint16)
    _check(_load().orc_round_to_half(_ptr(v), v.size, _ptr(out)), "orc_round_to_half")
    return out.view(np.float16)


def silu_mul(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """h = fp16(SiLU(g) * u) element-wise for fp16 B x N arrays (float16 result)."""
    gb = _half_bits(np.atleast_2d(g))
    ub = _half_bits(np.atleast_2d(u))
    assert gb.shape == ub.shape
    B, N = gb.shape
    h = np.zeros((B, N), dtype=np.uint16)
    _check(_load().orc_silu_mul(_ptr(gb), _ptr(ub), B, N, N, _ptr(h)), "orc_silu_mul")
    return h.view(np.float16)


def ffn(Wg: np.ndarray, mask_g: np.ndarray, Wu: np.ndarray, mask_u: np.ndarray,
        x: np.ndarray, t: float = 0.0) -> tuple[np.ndarray, np.ndarray]:
    """Fused FFN activation of a decode batch: (h float16 B x N, act_bits of h).

    g and u are the gate and up products rounded once to fp16 (what the two decode calls
    return), h = fp16(SiLU(g) * u), and the column set is the threshold rule on h."""
    g = round_to_half(spmv(Wg, mask_g, x, 0.0, None))
    u = round_to_half(spmv(Wu, mask_u, x, 0.0, None))
    h = silu_mul(g, u)
    bits, _ = select_threshold(h, t)
    return h, bits


def rel_err(y, y_ref) -> float:
    """max|y - y_ref| / max|y_ref| over the whole output of one call.

    When max|y_ref| is 0 the result is 0.0 if y is exactly zero everywhere, else inf.
    NaN anywhere in y where y_ref is finite counts as inf.
    """
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    if y.shape != y_ref.shape:
        raise ValueError(f"shape mismatch {y.shape} vs {y_ref.shape}")
    if y.size == 0:
        return 0.0
    if np.isnan(y).any() and not np.isnan(y_ref).any():
        return float("inf")
    scale = np.max(np.abs(y_ref))
    diff = np.max(np.abs(y - y_ref))
    if scale == 0:
        return 0.0 if diff == 0 else float("inf")
    return float(diff / scale)
