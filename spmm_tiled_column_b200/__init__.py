"""spmm_tiled_column_b200 -- Python binding of libspw.so, the sparse-weight SpMV/SpMM library.

Argument marshalling only: every function below checks tensor dtypes/devices, allocates
outputs with torch when the caller did not pass them, and calls the C function of the
same name in libspw.so (see include/spw.h) on torch's current CUDA stream.  All compute
runs in the library's CUDA kernels; there is no CPU path.  If libspw.so is missing or
cannot be loaded, the first call raises.

Tensors: fp16 weights / activations as torch.float16 (or int16/uint16 bit views), the
mask as torch.uint8 (nonzero = kept), TCB buffers as torch.uint8, bitmaps as torch.int32.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspw.so")

SPW_OK = 0
SPW_ERR_INVALID_ARG = 1
SPW_ERR_ALIGNMENT = 2
SPW_ERR_BUFFER_TOO_SMALL = 3
SPW_ERR_FORMAT = 4
SPW_ERR_UNSUPPORTED = 5
SPW_ERR_CUDA = 6
SPW_ERR_TIMEOUT = 7

# C function name -> (argtypes, restype)
_P = ctypes.c_void_p
_I = ctypes.c_int
_U64 = ctypes.c_uint64
_F = ctypes.c_float


class spw_format(ctypes.Structure):
    """Host copy of the TCB v1 header (same layout as the C struct)."""
    _fields_ = [("magic", ctypes.c_uint32), ("version", ctypes.c_uint32),
                ("N", ctypes.c_uint32), ("K", ctypes.c_uint32),
                ("TN", ctypes.c_uint32), ("TK", ctypes.c_uint32),
                ("n_strips", ctypes.c_uint32), ("n_ktiles", ctypes.c_uint32),
                ("nnz", ctypes.c_uint64), ("bytes_total", ctypes.c_uint64),
                ("off_bitmaps", ctypes.c_uint64), ("off_tileptr", ctypes.c_uint64),
                ("off_values", ctypes.c_uint64), ("max_tile_units", ctypes.c_uint32),
                ("reserved", ctypes.c_uint32)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


_FP = ctypes.POINTER(spw_format)


class spw_spmm_plan_info(ctypes.Structure):
    _fields_ = [("token_tile", ctypes.c_int32), ("token_tiles", ctypes.c_int32),
                ("weight_tiles", ctypes.c_int32), ("k_parts", ctypes.c_int32),
                ("whole_tiles", ctypes.c_int32), ("ctas", ctypes.c_int32),
                ("cta_pair", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_uint64)]
SIGNATURES = {
    "spw_status_string": ([_I], ctypes.c_char_p),
    "spw_version": ([], _I),
    "spw_set_launch_overlap": ([_I], _I),
    "spw_set_wait_limit_cycles": ([_U64], _U64),
    "spw_set_column_fetch": ([_I], _I),
    "spw_format_query": ([_P, _I, _I, _I, _P, _P, _P], _I),
    "spw_compress": ([_P, _I, _P, _I, _I, _I, _P, _U64, _FP, _P], _I),
    "spw_format_read": ([_P, _U64, _FP, _P], _I),
    "spw_decompress": ([_FP, _P, _P, _I, _P], _I),
    "spw_select_threshold": ([_P, _I, _I, _I, _F, _P, _P, _P], _I),
    "spw_select_topk": ([_P, _I, _I, _I, _I, _P, _P, _P], _I),
    "spw_spmv_workspace_bytes": ([_FP, _I], _U64),
    "spw_spmv": ([_FP, _P, _P, _I, _I, _F, _P, _P, _I, _P, _U64, _P], _I),
    "spw_spmm_workspace_bytes": ([_FP, _I], _U64),
    "spw_spmm": ([_FP, _P, _P, _I, _I, _P, _I, _P, _U64, _P], _I),
    "spw_spmv_tc_workspace_bytes": ([_FP, _I], _U64),
    "spw_spmv_tc": ([_FP, _P, _P, _I, _I, _F, _P, _P, _I, _P, _U64, _P], _I),
    "spw_spmv_auto_path": ([_I], _I),
    "spw_spmv_auto_workspace_bytes": ([_FP, _I], _U64),
    "spw_spmv_auto": ([_FP, _P, _P, _I, _I, _F, _P, _P, _I, _P, _U64, _P], _I),
    "spw_last_device_status": ([_P, _P], _I),
    "spw_spmv_group_workspace_bytes": ([_I, _FP, _I], _U64),
    "spw_spmv_group": ([_I, _FP, _P, _P, _P, _P, _P, _P, _I, _F, _P, _U64, _P], _I),
    "spw_spmv_noalloc_max_scratch_bytes": ([], _U64),
    "spw_spmv_noalloc": ([_FP, _P, _P, _I, _I, _F, _P, _P, _I, _P], _I),
    "spw_spmv_ffn_workspace_bytes": ([_FP, _FP, _I], _U64),
    "spw_spmm_plan": ([_FP, _I, _I, ctypes.POINTER(spw_spmm_plan_info)], _I),
    "spw_spmv_ffn": ([_FP, _P, _FP, _P, _P, _I, _I, _F, _P, _I, _P, _P, _U64, _P], _I),
    "spw_group_tokens_workspace_bytes": ([_I, _I], _U64),
    "spw_group_tokens": ([_P, _I, _I, _I, _F, _I, _P, _I, _P, _P, _P, _U64, _P], _I),
    "spw_spmm_tokens_workspace_bytes": ([_FP, _I], _U64),
    "spw_spmm_tokens_plan": ([_FP, _I, _I, ctypes.POINTER(spw_spmm_plan_info)], _I),
    "spw_spmm_tokens": ([_FP, _P, _P, _I, _I, _F, _P, _I, _P, _U64, _P], _I),
    "spw_s24_bytes": ([_I, _I], _U64),
    "spw_split24": ([_P, _I, _P, _I, _I, _I, _P, _U64, _P, _I, _P], _I),
    "spw_spmm24_workspace_bytes": ([_FP, _I], _U64),
    "spw_spmm24_plan": ([_FP, _I, _I, ctypes.POINTER(spw_spmm_plan_info)], _I),
    "spw_spmm24": ([_FP, _P, _P, _U64, _P, _I, _I, _P, _I, _P, _U64, _P], _I),
}


class SpwError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libspw.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing; build it with "
                               "`python -m spmm_tiled_column_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().spw_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != SPW_OK:
        raise SpwError(fn, status)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _half(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype in (torch.int16, torch.uint16):
        t = t.view(torch.float16)
    if t.dtype != torch.float16:
        raise TypeError(f"{name} must be float16 (or a 16-bit bit view), got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t


def _rows(t: torch.Tensor, name: str) -> tuple[torch.Tensor, int]:
    """2-D row-major view and its leading dimension (elements)."""
    if t.dim() == 1:
        t = t.unsqueeze(0)
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    return t, max(t.stride(0), t.shape[1])


def _need(t: torch.Tensor, rows: int, cols: int, name: str):
    """A 2-D view must hold at least rows x cols elements: the library reads or writes
    that much through its pointer and cannot see the tensor's size."""
    if t.shape[0] < rows or t.shape[1] < cols:
        raise ValueError(f"{name} is {tuple(t.shape)}; the call needs at least {rows} x {cols}")


def _need_buf(buf: torch.Tensor, h, name: str = "buf"):
    if not buf.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if buf.numel() * buf.element_size() < h.bytes_total:
        raise ValueError(f"{name} holds {buf.numel() * buf.element_size()} bytes; the format "
                         f"header says {h.bytes_total}")


def _nbytes(t: torch.Tensor | None, name: str = "ws") -> int:
    """Bytes of a raw buffer handed to the library with its size (0 for None); the
    library writes through its pointer on the device, so it must be a CUDA tensor."""
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t.numel() * t.element_size()


def _need_words(a: torch.Tensor | None, n: int, name: str = "act_bits"):
    """A column-set or output bit array of ceil(n / 32) 32-bit words, on the GPU."""
    if a is not None and _nbytes(a, name) < 4 * ((n + 31) // 32):
        raise ValueError(f"{name} needs at least {(n + 31) // 32} 32-bit words")


def _need_u32(a: torch.Tensor, n: int, name: str):
    """An output array of n 32-bit entries, on the GPU."""
    if _nbytes(a, name) < 4 * n:
        raise ValueError(f"{name} needs at least {n} 32-bit entries")


def _mask_like(mask: torch.Tensor, N: int, K: int) -> tuple[torch.Tensor, int]:
    """An N x K uint8 CUDA mask with unit column stride, and its leading dimension."""
    m, ld = _rows(mask, "mask")
    if m.dtype != torch.uint8 or not m.is_cuda:
        raise TypeError("mask must be a CUDA uint8 tensor")
    if tuple(m.shape) != (N, K):
        raise ValueError(f"mask is {tuple(m.shape)}; the weight is {N} x {K}")
    return m, ld


def _hdr(h) -> spw_format:
    if isinstance(h, spw_format):
        return h
    f = spw_format()
    for k, v in dict(h).items():
        setattr(f, k, int(v))
    return f


def spw_set_launch_overlap(enable: bool) -> bool:
    """Enable/disable programmatic launch overlap of consecutive spw_spmv calls (see
    include/spw.h for the one condition it needs); returns the previous setting."""
    return bool(lib().spw_set_launch_overlap(1 if enable else 0))


def spw_set_column_fetch(mode: int) -> int:
    """Decode column fetch: 0 whole tiles (default), 1 when a call carries a column set or a
    threshold above zero, 2 always; returns the previous mode (see include/spw.h)."""
    prev = int(lib().spw_set_column_fetch(int(mode)))
    if prev < 0:
        raise ValueError("column fetch mode must be 0, 1 or 2")
    return prev


def spw_set_wait_limit_cycles(cycles: int) -> int:
    """Set the limit of the kernels' bounded pipeline waits in SM cycles (0: the default,
    about one second); returns the previous limit.  A test hook for the timeout path (see
    include/spw.h)."""
    return int(lib().spw_set_wait_limit_cycles(int(cycles)))


# ------------------------------------------------------------------ format

def spw_format_query(mask: torch.Tensor, stream=None) -> tuple[int, int]:
    """(bytes_total, nnz) of the TCB v1 buffer for an N x K uint8 mask."""
    mask, ld = _rows(mask, "mask")
    if mask.dtype != torch.uint8 or not mask.is_cuda:
        raise TypeError("mask must be a CUDA uint8 tensor")
    nbytes, nnz = ctypes.c_uint64(), ctypes.c_uint64()
    _check("spw_format_query", lib().spw_format_query(
        _ptr(mask), mask.shape[0], mask.shape[1], ld, ctypes.byref(nbytes), ctypes.byref(nnz),
        _stream(stream)))
    return nbytes.value, nnz.value


def spw_compress(W: torch.Tensor, mask: torch.Tensor, buf: torch.Tensor | None = None,
                 stream=None) -> tuple[torch.Tensor, spw_format]:
    """Compress W * mask into a TCB v1 buffer; returns (uint8 device buffer, header)."""
    W, ldw = _rows(_half(W, "W"), "W")
    N, K = W.shape
    mask, ldm = _mask_like(mask, N, K)
    if buf is None:
        nbytes, _ = spw_format_query(mask, stream)
        buf = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    hdr = spw_format()
    _check("spw_compress", lib().spw_compress(
        _ptr(W), ldw, _ptr(mask), ldm, N, K, _ptr(buf), _nbytes(buf, "buf"), ctypes.byref(hdr),
        _stream(stream)))
    return buf, hdr


def spw_format_read(buf: torch.Tensor, stream=None) -> spw_format:
    hdr = spw_format()
    _check("spw_format_read", lib().spw_format_read(_ptr(buf), _nbytes(buf, "buf"), ctypes.byref(hdr),
                                                    _stream(stream)))
    return hdr


def spw_decompress(hdr, buf: torch.Tensor, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """Dense masked weight (fp16, N x K) from a TCB v1 buffer."""
    h = _hdr(hdr)
    if out is None:
        out = torch.empty((h.N, h.K), dtype=torch.float16, device=buf.device)
    out2, ld = _rows(_half(out, "out"), "out")
    _need_buf(buf, h)
    _need(out2, h.N, h.K, "out")
    _check("spw_decompress", lib().spw_decompress(ctypes.byref(h), _ptr(buf), _ptr(out2), ld,
                                                  _stream(stream)))
    return out


# ------------------------------------------------------------------ selection

def _act_words(K: int) -> int:
    return (K + 31) // 32


def spw_select_threshold(x: torch.Tensor, t: float, act_bits: torch.Tensor | None = None,
                         count: torch.Tensor | None = None, stream=None):
    """(act_bits int32[ceil(K/32)], count int32[1]) for the threshold rule."""
    x, ldx = _rows(_half(x, "x"), "x")
    B, K = x.shape
    if act_bits is None:
        act_bits = torch.empty(_act_words(K) + 3, dtype=torch.int32, device=x.device)
    if count is None:
        count = torch.empty(1, dtype=torch.int32, device=x.device)
    _need_words(act_bits, K)
    _need_u32(count, 1, "count")
    _check("spw_select_threshold", lib().spw_select_threshold(
        _ptr(x), B, K, ldx, float(t), _ptr(act_bits), _ptr(count), _stream(stream)))
    return act_bits, count


def spw_select_topk(x: torch.Tensor, k: int, act_bits: torch.Tensor | None = None,
                    idx: torch.Tensor | None = None, stream=None):
    """(act_bits int32[ceil(K/32)], ascending idx int32[k]) of the top-k columns."""
    x, ldx = _rows(_half(x, "x"), "x")
    B, K = x.shape
    if act_bits is None:
        act_bits = torch.empty(_act_words(K) + 3, dtype=torch.int32, device=x.device)
    if idx is None:
        idx = torch.empty(max(int(k), 1), dtype=torch.int32, device=x.device)
    _need_words(act_bits, K)
    _need_u32(idx, int(k), "idx")
    _check("spw_select_topk", lib().spw_select_topk(
        _ptr(x), B, K, ldx, int(k), _ptr(act_bits), _ptr(idx), _stream(stream)))
    return act_bits, idx[:k]


# ------------------------------------------------------------------ products

def spw_spmv_workspace_bytes(hdr, B: int) -> int:
    h = _hdr(hdr)
    return int(lib().spw_spmv_workspace_bytes(ctypes.byref(h), int(B)))


def spw_spmv(hdr, buf: torch.Tensor, x: torch.Tensor, threshold: float = 0.0,
             act_bits: torch.Tensor | None = None, y: torch.Tensor | None = None,
             ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode y (B x N fp16) = W_masked . x~ with column skipping.

    ws: a zero-initialised uint8 workspace of spw_spmv_workspace_bytes(hdr, B) bytes
    (allocated here with torch.zeros when not given)."""
    h = _hdr(hdr)
    x2, ldx = _rows(_half(x, "x"), "x")
    B = x2.shape[0]
    if y is None:
        y = torch.empty((B, h.N), dtype=torch.float16, device=x.device)
    y2, ldy = _rows(_half(y, "y"), "y")
    _need_buf(buf, h)
    _need(x2, B, h.K, "x")
    _need(y2, B, h.N, "y")
    _need_words(act_bits, h.K)
    if ws is None:
        ws = torch.zeros(max(spw_spmv_workspace_bytes(h, B), 16), dtype=torch.uint8,
                         device=x.device)
    _check("spw_spmv", lib().spw_spmv(
        ctypes.byref(h), _ptr(buf), _ptr(x2), B, ldx, float(threshold), _ptr(act_bits),
        _ptr(y2), ldy, _ptr(ws), _nbytes(ws), _stream(stream)))
    return y


def _hdr_array(hdrs) -> ctypes.Array:
    arr = (spw_format * len(hdrs))()
    for i, h in enumerate(hdrs):
        arr[i] = _hdr(h)
    return arr


def spw_spmv_group_workspace_bytes(hdrs, B: int) -> int:
    return int(lib().spw_spmv_group_workspace_bytes(len(hdrs), _hdr_array(hdrs), int(B)))


def spw_spmv_group(hdrs, bufs, xs, threshold: float = 0.0, act_bits=None, ys=None, ws=None,
                   stream=None):
    """Decode several layers in one launch; returns the list of outputs (B x N_l each)."""
    n = len(hdrs)
    harr = _hdr_array(hdrs)
    x2 = [_rows(_half(x, "x"), "x") for x in xs]
    B = x2[0][0].shape[0]
    if ys is None:
        ys = [torch.empty((B, int(h.N)), dtype=torch.float16, device=xs[0].device) for h in harr]
    y2 = [_rows(_half(y, "y"), "y") for y in ys]
    if len(bufs) != n or len(x2) != n or len(y2) != n or (act_bits is not None and len(act_bits) != n):
        raise ValueError(f"expected {n} buffers, inputs and outputs (and column sets)")
    for i, h in enumerate(harr):
        _need_buf(bufs[i], h, f"bufs[{i}]")
        _need(x2[i][0], B, h.K, f"xs[{i}]")
        _need(y2[i][0], B, h.N, f"ys[{i}]")
        _need_words(None if act_bits is None else act_bits[i], h.K, f"act_bits[{i}]")
    if ws is None:
        ws = torch.zeros(max(spw_spmv_group_workspace_bytes(hdrs, B), 16), dtype=torch.uint8,
                         device=xs[0].device)
    P = ctypes.c_void_p * n
    I = ctypes.c_int * n
    ab = None if act_bits is None else P(*[None if a is None else a.data_ptr() for a in act_bits])
    _check("spw_spmv_group", lib().spw_spmv_group(
        n, harr, P(*[b.data_ptr() for b in bufs]), P(*[t.data_ptr() for t, _ in x2]),
        I(*[ld for _, ld in x2]), ab, P(*[t.data_ptr() for t, _ in y2]), I(*[ld for _, ld in y2]),
        B, float(threshold), _ptr(ws), _nbytes(ws), _stream(stream)))
    return ys


def spw_spmv_noalloc(hdr, buf: torch.Tensor, x: torch.Tensor, threshold: float = 0.0,
                     act_bits: torch.Tensor | None = None, y: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Decode like spw_spmv, with the library's own fixed scratch instead of a workspace.

    For callers that cannot allocate device memory; see include/spw.h for the size
    limit and for why overlapping calls race."""
    h = _hdr(hdr)
    x2, ldx = _rows(_half(x, "x"), "x")
    B = x2.shape[0]
    if y is None:
        y = torch.empty((B, h.N), dtype=torch.float16, device=x.device)
    y2, ldy = _rows(_half(y, "y"), "y")
    _need_buf(buf, h)
    _need(x2, x2.shape[0], h.K, "x")
    _need(y2, x2.shape[0], h.N, "y")
    _need_words(act_bits, h.K)
    _check("spw_spmv_noalloc", lib().spw_spmv_noalloc(
        ctypes.byref(h), _ptr(buf), _ptr(x2), B, ldx, float(threshold), _ptr(act_bits),
        _ptr(y2), ldy, _stream(stream)))
    return y


def spw_spmm_workspace_bytes(hdr, M: int) -> int:
    h = _hdr(hdr)
    return int(lib().spw_spmm_workspace_bytes(ctypes.byref(h), int(M)))


def spw_spmm(hdr, buf: torch.Tensor, X: torch.Tensor, Y: torch.Tensor | None = None,
             ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Prefill Y (M x N fp16) = X . W_masked^T on tcgen05 tensor cores."""
    h = _hdr(hdr)
    X2, ldx = _rows(_half(X, "X"), "X")
    M = X2.shape[0]
    if Y is None:
        Y = torch.empty((M, h.N), dtype=torch.float16, device=X.device)
    Y2, ldy = _rows(_half(Y, "Y"), "Y")
    _need_buf(buf, h)
    _need(X2, M, h.K, "X")
    _need(Y2, M, h.N, "Y")
    need = spw_spmm_workspace_bytes(h, M)
    if ws is None and need:
        ws = torch.zeros(need, dtype=torch.uint8, device=X.device)
    _check("spw_spmm", lib().spw_spmm(
        ctypes.byref(h), _ptr(buf), _ptr(X2), M, ldx, _ptr(Y2), ldy, _ptr(ws),
        _nbytes(ws), _stream(stream)))
    return Y


def spw_spmm_plan(hdr, M: int, sm_count: int = 0) -> dict:
    """The launch plan of spw_spmm for M tokens on sm_count SMs (0: the current device)."""
    info = spw_spmm_plan_info()
    _check("spw_spmm_plan", lib().spw_spmm_plan(ctypes.byref(_hdr(hdr)), int(M), int(sm_count),
                                                ctypes.byref(info)))
    return {name: getattr(info, name) for name, _ in info._fields_}


def spw_group_tokens_workspace_bytes(M: int, K: int) -> int:
    return int(lib().spw_group_tokens_workspace_bytes(int(M), int(K)))


def spw_group_tokens(X: torch.Tensor, t: float, token_tile: int, ws: torch.Tensor | None = None,
                     stream=None) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Token grouping of X (M x K fp16): (Xg M x ceil8(K) fp16, perm int32[M], tile_sig
    int64[ceil(M / token_tile), words]); see spw_group_tokens in include/spw.h."""
    X2, ldx = _rows(_half(X, "X"), "X")
    M, K = X2.shape[0], X2.shape[1]
    words = ((K + 63) // 64 + 63) // 64
    ldg = (K + 7) // 8 * 8
    Xg = torch.empty((M, ldg), dtype=torch.float16, device=X.device)
    perm = torch.empty(M, dtype=torch.int32, device=X.device)
    tsig = torch.empty((-(-M // int(token_tile)), words), dtype=torch.int64, device=X.device)
    need = spw_group_tokens_workspace_bytes(M, K)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    _check("spw_group_tokens", lib().spw_group_tokens(
        _ptr(X2), M, K, ldx, ctypes.c_float(t), int(token_tile), _ptr(Xg), ldg, _ptr(perm),
        _ptr(tsig), _ptr(ws), _nbytes(ws), _stream(stream)))
    return Xg, perm, tsig


def spw_spmm_tokens_workspace_bytes(hdr, M: int) -> int:
    return int(lib().spw_spmm_tokens_workspace_bytes(ctypes.byref(_hdr(hdr)), int(M)))


def spw_spmm_tokens_plan(hdr, M: int, sm_count: int = 0) -> dict:
    """The launch plan of spw_spmm_tokens (its token tile is the grouping's T)."""
    info = spw_spmm_plan_info()
    _check("spw_spmm_tokens_plan", lib().spw_spmm_tokens_plan(
        ctypes.byref(_hdr(hdr)), int(M), int(sm_count), ctypes.byref(info)))
    return {name: getattr(info, name) for name, _ in info._fields_}


def spw_spmm_tokens(hdr, buf: torch.Tensor, X: torch.Tensor, threshold: float,
                    Y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """Prefill with per-token index sets: Y = X~ . W_masked^T, tokens grouped by the
    k-tiles they use (see spw_spmm_tokens in include/spw.h).  ws: a uint8 workspace of
    spw_spmm_tokens_workspace_bytes(hdr, M) bytes whose first (split-K counter) bytes are
    zero; allocated zeroed here when omitted."""
    h = _hdr(hdr)
    X2, ldx = _rows(_half(X, "X"), "X")
    M = X2.shape[0]
    if Y is None:
        Y = torch.empty((M, h.N), dtype=torch.float16, device=X.device)
    Y2, ldy = _rows(_half(Y, "Y"), "Y")
    _need_buf(buf, h)
    _need(X2, M, h.K, "X")
    _need(Y2, M, h.N, "Y")
    if ws is None:
        ws = torch.zeros(max(spw_spmm_tokens_workspace_bytes(h, M), 16), dtype=torch.uint8,
                         device=X.device)
    _check("spw_spmm_tokens", lib().spw_spmm_tokens(
        ctypes.byref(h), _ptr(buf), _ptr(X2), M, ldx, ctypes.c_float(threshold), _ptr(Y2), ldy,
        _ptr(ws), _nbytes(ws), _stream(stream)))
    return Y


def spw_spmv_tc_workspace_bytes(hdr, B: int) -> int:
    h = _hdr(hdr)
    return int(lib().spw_spmv_tc_workspace_bytes(ctypes.byref(h), int(B)))


def spw_spmv_tc(hdr, buf: torch.Tensor, x: torch.Tensor, threshold: float = 0.0,
                act_bits: torch.Tensor | None = None, y: torch.Tensor | None = None,
                ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode y (B x N fp16) on tensor cores; arguments as spw_spmv.  ws: a zero-initialised
    uint8 workspace of spw_spmv_tc_workspace_bytes(hdr, B) bytes (allocated here when
    needed and not given)."""
    h = _hdr(hdr)
    x2, ldx = _rows(_half(x, "x"), "x")
    B = x2.shape[0]
    if y is None:
        y = torch.empty((B, h.N), dtype=torch.float16, device=x.device)
    y2, ldy = _rows(_half(y, "y"), "y")
    _need_buf(buf, h)
    _need(x2, B, h.K, "x")
    _need(y2, B, h.N, "y")
    _need_words(act_bits, h.K)
    need = spw_spmv_tc_workspace_bytes(h, B)
    if ws is None and need:
        ws = torch.zeros(need, dtype=torch.uint8, device=x.device)
    _check("spw_spmv_tc", lib().spw_spmv_tc(
        ctypes.byref(h), _ptr(buf), _ptr(x2), B, ldx, float(threshold), _ptr(act_bits),
        _ptr(y2), ldy, _ptr(ws), _nbytes(ws), _stream(stream)))
    return y


def spw_spmv_auto_path(B: int) -> int:
    """0 when spw_spmv_auto takes the CUDA-core decode for batch B, 1 for the tensor-core
    decode, -1 for B outside 1..16."""
    return int(lib().spw_spmv_auto_path(int(B)))


def spw_spmv_auto_workspace_bytes(hdr, B: int) -> int:
    h = _hdr(hdr)
    return int(lib().spw_spmv_auto_workspace_bytes(ctypes.byref(h), int(B)))


def spw_spmv_auto(hdr, buf: torch.Tensor, x: torch.Tensor, threshold: float = 0.0,
                  act_bits: torch.Tensor | None = None, y: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode y (B x N fp16) on the path chosen by batch size; arguments as spw_spmv.  ws:
    a zero-initialised uint8 workspace of spw_spmv_auto_workspace_bytes(hdr, B) bytes
    (allocated here when needed and not given)."""
    h = _hdr(hdr)
    x2, ldx = _rows(_half(x, "x"), "x")
    B = x2.shape[0]
    if y is None:
        y = torch.empty((B, h.N), dtype=torch.float16, device=x.device)
    y2, ldy = _rows(_half(y, "y"), "y")
    _need_buf(buf, h)
    _need(x2, B, h.K, "x")
    _need(y2, B, h.N, "y")
    _need_words(act_bits, h.K)
    need = spw_spmv_auto_workspace_bytes(h, B)
    if ws is None and need:
        ws = torch.zeros(need, dtype=torch.uint8, device=x.device)
    _check("spw_spmv_auto", lib().spw_spmv_auto(
        ctypes.byref(h), _ptr(buf), _ptr(x2), B, ldx, float(threshold), _ptr(act_bits),
        _ptr(y2), ldy, _ptr(ws), _nbytes(ws), _stream(stream)))
    return y


def spw_spmv_ffn_workspace_bytes(hdr_gate, hdr_up, B: int) -> int:
    return int(lib().spw_spmv_ffn_workspace_bytes(ctypes.byref(_hdr(hdr_gate)),
                                                  ctypes.byref(_hdr(hdr_up)), B))


def spw_spmv_ffn(hdr_gate, buf_gate: torch.Tensor, hdr_up, buf_up: torch.Tensor, x: torch.Tensor,
                 threshold: float = 0.0, h: torch.Tensor | None = None,
                 act_bits: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                 stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Fused FFN activation: h (B x N fp16) = SiLU(W_gate x) * (W_up x) and the column-set
    words of h under the threshold rule, in one launch.  ws: a zero-initialised uint8
    workspace of spw_spmv_ffn_workspace_bytes(hdr_gate, hdr_up, B) bytes (allocated here
    when not given).  Returns (h, act_bits)."""
    hg, hu = _hdr(hdr_gate), _hdr(hdr_up)
    x2, ldx = _rows(_half(x, "x"), "x")
    B = x2.shape[0]
    if h is None:
        h = torch.empty((B, hg.N), dtype=torch.float16, device=x.device)
    h2, ldh = _rows(_half(h, "h"), "h")
    _need_buf(buf_gate, hg, "buf_gate")
    _need_buf(buf_up, hu, "buf_up")
    _need(x2, B, hg.K, "x")
    _need(h2, B, hg.N, "h")
    if act_bits is None:
        act_bits = torch.empty(((hg.N + 31) // 32,), dtype=torch.int32, device=x.device)
    _need_words(act_bits, hg.N)
    if ws is None:
        need = spw_spmv_ffn_workspace_bytes(hg, hu, B)
        ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=x.device)
    _check("spw_spmv_ffn", lib().spw_spmv_ffn(
        ctypes.byref(hg), _ptr(buf_gate), ctypes.byref(hu), _ptr(buf_up), _ptr(x2), B, ldx,
        float(threshold), _ptr(h2), ldh, _ptr(act_bits), _ptr(ws), _nbytes(ws), _stream(stream)))
    return h, act_bits


def spw_last_device_status(stream=None) -> int:
    code = ctypes.c_int()
    _check("spw_last_device_status", lib().spw_last_device_status(_stream(stream),
                                                                  ctypes.byref(code)))
    return code.value


class DecodeGroup:
    """A prepared spw_spmv_group call for a fixed set of layers and batch size.

    The header array, weight pointers and workspace are built once; each call only
    refreshes the input and output pointers and leading dimensions, so the per-call host
    cost is one library call (serving loops that decode the same layers every step)."""

    def __init__(self, hdrs, bufs, B: int, ws: torch.Tensor | None = None):
        self.n = len(hdrs)
        if self.n != len(bufs):
            raise ValueError("one weight buffer per header")
        self.B = int(B)
        self._harr = _hdr_array(hdrs)
        for i, h in enumerate(self._harr):
            _need_buf(bufs[i], h, f"bufs[{i}]")
        self._K = [int(h.K) for h in self._harr]
        self._N = [int(h.N) for h in self._harr]
        self._bufs = list(bufs)  # keeps the weights alive
        P = ctypes.c_void_p * self.n
        I = ctypes.c_int * self.n
        self._pbufs = P(*[b.data_ptr() for b in bufs])
        self._px, self._py, self._pab = P(), P(), P()
        self._ldx, self._ldy = I(), I()
        if ws is None:
            need = spw_spmv_group_workspace_bytes(self._harr, self.B)
            ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=bufs[0].device)
        self.ws = ws

    def __call__(self, xs, ys, threshold: float = 0.0, act_bits=None, stream=None):
        """Decode into ys (one B x N_l fp16 tensor per layer) from xs (B x K_l each)."""
        if len(xs) != self.n or len(ys) != self.n:
            raise ValueError(f"expected {self.n} inputs and outputs")
        for i in range(self.n):
            x, y = xs[i], ys[i]
            if x.dtype != torch.float16 or y.dtype != torch.float16:
                raise TypeError("inputs and outputs must be float16")
            if not (x.is_cuda and y.is_cuda):
                raise ValueError("inputs and outputs must be CUDA tensors")
            xr = x.shape[0] if x.dim() == 2 else 1
            yr = y.shape[0] if y.dim() == 2 else 1
            if xr < self.B or x.shape[-1] < self._K[i] or yr < self.B or y.shape[-1] < self._N[i]:
                raise ValueError(f"layer {i}: x needs {self.B} x {self._K[i]}, y {self.B} x {self._N[i]}")
            self._px[i] = x.data_ptr()
            self._ldx[i] = x.stride(0) if x.dim() == 2 and x.shape[0] > 1 else x.shape[-1]
            self._py[i] = y.data_ptr()
            self._ldy[i] = y.stride(0) if y.dim() == 2 and y.shape[0] > 1 else y.shape[-1]
        ab = None
        if act_bits is not None:
            for i in range(self.n):
                _need_words(act_bits[i], self._K[i], f"act_bits[{i}]")
                self._pab[i] = None if act_bits[i] is None else act_bits[i].data_ptr()
            ab = self._pab
        _check("spw_spmv_group", lib().spw_spmv_group(
            self.n, self._harr, self._pbufs, self._px, self._ldx, ab, self._py, self._ldy,
            self.B, float(threshold), _ptr(self.ws), _nbytes(self.ws), _stream(stream)))
        return ys


def spw_s24_bytes(N: int, K: int) -> int:
    return int(lib().spw_s24_bytes(int(N), int(K)))


def spw_split24(W: torch.Tensor, mask: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """2:4 + residual split: (s24 uint8 buffer of the 2:4 part, residual mask uint8 N x K);
    see spw_split24 in include/spw.h."""
    W2, ldw = _rows(_half(W, "W"), "W")
    N, K = W2.shape
    m2, ldm = _mask_like(mask, N, K)
    s24 = torch.empty(spw_s24_bytes(N, K), dtype=torch.uint8, device=W.device)
    mask_r = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    _check("spw_split24", lib().spw_split24(_ptr(W2), ldw, _ptr(m2), ldm, N, K, _ptr(s24), _nbytes(s24, "s24"),
                                            _ptr(mask_r), K, _stream(stream)))
    return s24, mask_r


def spw_spmm24_workspace_bytes(hdr_r, M: int) -> int:
    return int(lib().spw_spmm24_workspace_bytes(ctypes.byref(_hdr(hdr_r)), int(M)))


def spw_spmm24_plan(hdr_r, M: int, sm_count: int = 0) -> dict:
    info = spw_spmm_plan_info()
    _check("spw_spmm24_plan", lib().spw_spmm24_plan(ctypes.byref(_hdr(hdr_r)), int(M), int(sm_count),
                                                    ctypes.byref(info)))
    return {name: getattr(info, name) for name, _ in info._fields_}


def spw_spmm24(hdr_r, buf_r: torch.Tensor, s24: torch.Tensor, X: torch.Tensor,
               Y: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Prefill on the 2:4 + residual split: Y = X . (S + R)^T, S on sparse tensor cores."""
    h = _hdr(hdr_r)
    X2, ldx = _rows(_half(X, "X"), "X")
    M = X2.shape[0]
    if Y is None:
        Y = torch.empty((M, h.N), dtype=torch.float16, device=X.device)
    Y2, ldy = _rows(_half(Y, "Y"), "Y")
    _need_buf(buf_r, h, "buf_r")
    _need(X2, M, h.K, "X")
    _need(Y2, M, h.N, "Y")
    need = spw_spmm24_workspace_bytes(h, M)
    if ws is None and need:
        ws = torch.zeros(need, dtype=torch.uint8, device=X.device)
    _check("spw_spmm24", lib().spw_spmm24(
        ctypes.byref(h), _ptr(buf_r), _ptr(s24), _nbytes(s24, "s24"), _ptr(X2), M, ldx, _ptr(Y2), ldy,
        _ptr(ws), _nbytes(ws), _stream(stream)))
    return Y


class SparseLinear24:
    """A weight held as its 2:4 part (sparse tensor cores) plus a TCB residual: a holder
    for spw_split24, spw_compress and spw_spmm24 (it adds no arithmetic)."""

    def __init__(self, W: torch.Tensor, mask: torch.Tensor, stream=None):
        self.N, self.K = W.shape
        self.s24, self.mask_r = spw_split24(W, mask, stream)
        self.buf_r, self.hdr_r = spw_compress(W, self.mask_r, stream=stream)

    def spmm(self, X, Y=None, ws=None, stream=None):
        return spw_spmm24(self.hdr_r, self.buf_r, self.s24, X, Y, ws, stream)


class SparseLinear:
    """A compressed weight with its header and per-batch decode workspaces (a holder for
    the calls above; it adds no arithmetic)."""

    def __init__(self, W: torch.Tensor, mask: torch.Tensor, stream=None):
        self.N, self.K = W.shape
        self.buf, self.hdr = spw_compress(W, mask, stream=stream)
        self._ws = {}

    def workspace(self, B: int) -> torch.Tensor:
        if B not in self._ws:
            self._ws[B] = torch.zeros(max(spw_spmv_workspace_bytes(self.hdr, B), 16),
                                      dtype=torch.uint8, device=self.buf.device)
        return self._ws[B]

    def spmv(self, x, threshold=0.0, act_bits=None, y=None, stream=None):
        x2 = x if x.dim() == 2 else x.unsqueeze(0)
        return spw_spmv(self.hdr, self.buf, x2, threshold, act_bits, y,
                        self.workspace(x2.shape[0]), stream)

    def spmv_auto(self, x, threshold=0.0, act_bits=None, y=None, stream=None):
        x2 = x if x.dim() == 2 else x.unsqueeze(0)
        B = x2.shape[0]
        if ("auto", B) not in self._ws:
            self._ws[("auto", B)] = torch.zeros(max(spw_spmv_auto_workspace_bytes(self.hdr, B), 16),
                                                dtype=torch.uint8, device=self.buf.device)
        return spw_spmv_auto(self.hdr, self.buf, x2, threshold, act_bits, y,
                             self._ws[("auto", B)], stream)

    def spmm(self, X, Y=None, stream=None):
        return spw_spmm(self.hdr, self.buf, X, Y, stream=stream)

    def spmm_tokens(self, X, threshold=0.0, Y=None, ws=None, stream=None):
        return spw_spmm_tokens(self.hdr, self.buf, X, threshold, Y, ws, stream=stream)

    def decompress(self, out=None, stream=None):
        return spw_decompress(self.hdr, self.buf, out, stream)
