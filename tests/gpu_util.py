"""Helpers for the GPU parity tests: numpy <-> CUDA tensors, oracle comparisons."""
import numpy as np
import pytest
import torch

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

# Tolerance on max|y - y_ref| / max|y_ref| for products (fp16 inputs, fp32 accumulation),
# as fixed for this path.
TOL = 5e-3


def dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return torch.from_numpy(a.view(np.int16).copy()).cuda().view(torch.float16)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).cuda().view(torch.float16)
    if a.dtype == np.uint32:
        return torch.from_numpy(a.view(np.int32).copy()).cuda()
    return torch.from_numpy(a.copy()).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach()
    if t.dtype == torch.float16:
        return t.view(torch.int16).cpu().numpy().view(np.float16)
    if t.dtype == torch.int32:
        return t.cpu().numpy().view(np.uint32)
    return t.cpu().numpy()


def padded_rows(a: np.ndarray, ld: int) -> torch.Tensor:
    """Device copy of a 2-D fp16 array whose rows sit at stride ld (>= row length)."""
    rows, cols = a.shape
    buf = np.zeros((rows, ld), dtype=a.dtype)
    buf[:, :cols] = a
    return dev(buf)[:, :cols]


def half_bits(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float16).view(np.uint16)
