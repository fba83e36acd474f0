"""The C-ABI library loads and exports every symbol include/spw.h declares, and its
host-side argument checks return status codes without touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

from spmm_tiled_column_b200 import build as spw_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spw.h")


@pytest.fixture(scope="module")
def spw():
    spw_build.build()
    import spmm_tiled_column_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(spw_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("spw_compress", "spw_decompress", "spw_spmv", "spw_spmm",
                     "spw_select_threshold", "spw_select_topk", "spw_format_query"):
        assert required in names


def test_every_declared_symbol_is_exported(spw):
    lib = ctypes.CDLL(spw_build.LIB)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    # and the binding knows every one of them
    assert set(declared_functions()) <= set(spw.SIGNATURES)


def test_struct_layout_matches_header(spw):
    assert ctypes.sizeof(spw.spw_format) == 80
    assert spw.spw_format.max_tile_units.offset == 72


def test_status_strings_and_version(spw):
    L = spw.lib()
    assert L.spw_version() == 100
    for code in range(8):
        assert L.spw_status_string(code).decode().startswith("SPW_")
    assert L.spw_status_string(99).decode() == "unknown spw status"


def test_wait_limit_setting(spw):
    # The timeout hook is host state: 0 and values above the default (2e9 cycles) restore
    # the default; each call returns the previous limit.
    L = spw.lib()
    assert L.spw_set_wait_limit_cycles(0) == 2_000_000_000
    assert L.spw_set_wait_limit_cycles(5000) == 2_000_000_000
    assert L.spw_set_wait_limit_cycles(3 * 10**9) == 5000
    assert L.spw_set_wait_limit_cycles(0) == 2_000_000_000


def test_column_fetch_setting(spw):
    L = spw.lib()
    assert L.spw_set_column_fetch(2) == 0
    assert L.spw_set_column_fetch(1) == 2
    assert L.spw_set_column_fetch(3) == -1 and L.spw_set_column_fetch(-1) == -1
    assert L.spw_set_column_fetch(0) == 1


def valid_header(spw, N=128, K=128):
    h = spw.spw_format()
    h.magic, h.version, h.N, h.K, h.TN, h.TK = 0x31424354, 1, N, K, 64, 64
    h.n_strips, h.n_ktiles = (N + 63) // 64, (K + 63) // 64
    T = h.n_strips * h.n_ktiles
    h.off_bitmaps = 256
    h.off_tileptr = -(-(256 + 8 * 64 * T) // 256) * 256
    h.off_values = -(-(h.off_tileptr + 4 * (T + 1)) // 256) * 256
    h.bytes_total = h.off_values + 16 * T
    h.nnz, h.max_tile_units = T * 8, 1
    return h


def test_host_validation_without_gpu(spw):
    L = spw.lib()
    h = valid_header(spw)
    P = ctypes.c_void_p
    good = P(0x10000)
    odd = P(0x10008)
    s = P(0)
    ws_n = ctypes.c_uint64(1 << 20)
    # spmv argument errors
    assert L.spw_spmv(None, good, good, 1, 128, 0.0, None, good, 128, good, ws_n, s) == 1
    assert L.spw_spmv(ctypes.byref(h), None, good, 1, 128, 0.0, None, good, 128, good, ws_n, s) == 1
    for B in (0, 17):
        assert L.spw_spmv(ctypes.byref(h), good, good, B, 128, 0.0, None, good, 128, good, ws_n, s) == 1
    for t in (-1.0, float("nan"), float("inf")):
        assert L.spw_spmv(ctypes.byref(h), good, good, 1, 128, t, None, good, 128, good, ws_n, s) == 1
    assert L.spw_spmv(ctypes.byref(h), good, good, 2, 100, 0.0, None, good, 128, good, ws_n, s) == 1
    assert L.spw_spmv(ctypes.byref(h), good, good, 2, 132, 0.0, None, good, 128, good, ws_n, s) == 1
    assert L.spw_spmv(ctypes.byref(h), odd, good, 1, 128, 0.0, None, good, 128, good, ws_n, s) == 2
    assert L.spw_spmv(ctypes.byref(h), good, good, 1, 128, 0.0, odd, good, 128, good, ws_n, s) == 2
    # header errors
    bad = valid_header(spw)
    bad.magic = 0
    assert L.spw_spmv(ctypes.byref(bad), good, good, 1, 128, 0.0, None, good, 128, good, ws_n, s) == 4
    bad = valid_header(spw)
    bad.off_values += 256
    assert L.spw_decompress(ctypes.byref(bad), good, good, 128, s) == 4
    bad = valid_header(spw)
    bad.TN = 32
    assert L.spw_spmm(ctypes.byref(bad), good, good, 4, 128, good, 128, None, 0, s) == 4
    # selection
    assert L.spw_select_threshold(None, 1, 128, 128, 0.0, good, good, s) == 1
    assert L.spw_select_threshold(good, 1, 128, 128, -0.5, good, good, s) == 1
    assert L.spw_select_threshold(odd, 1, 128, 128, 0.5, good, good, s) == 2
    assert L.spw_select_topk(good, 1, 128, 128, 129, good, good, s) == 1
    assert L.spw_select_topk(good, 1, 128, 128, -1, good, good, s) == 1
    assert L.spw_select_topk(good, 1, 30000, 30000, 10, good, good, s) == 5
    # format
    n1, n2 = ctypes.c_uint64(), ctypes.c_uint64()
    assert L.spw_format_query(good, 0, 128, 128, ctypes.byref(n1), ctypes.byref(n2), s) == 1
    assert L.spw_format_query(good, 4, 128, 100, ctypes.byref(n1), ctypes.byref(n2), s) == 1
    assert L.spw_spmm(ctypes.byref(h), good, good, 4, 132, good, 128, None, 0, s) == 1
    assert L.spw_format_query(odd, 4, 128, 128, ctypes.byref(n1), ctypes.byref(n2), s) == 2
    assert L.spw_compress(good, 128, good, 128, 128, 128, good, 100, None, s) == 3
    assert L.spw_compress(good, 120, good, 128, 128, 128, good, 1 << 20, None, s) == 1
    assert L.spw_format_read(good, 10, None, s) == 1
    # device status
    assert L.spw_last_device_status(s, None) == 1


def test_tensor_core_decode_and_ffn_host_validation_without_gpu(spw):
    L = spw.lib()
    h = valid_header(spw)
    P = ctypes.c_void_p
    good, odd, s = P(0x10000), P(0x10008), P(0)
    ws_n = ctypes.c_uint64(1 << 20)
    # tensor-core decode: every argument error is found before any device call
    bad = valid_header(spw)
    bad.version = 2
    assert L.spw_spmv_tc(ctypes.byref(bad), good, good, 1, 128, 0.0, None, good, 128, good, ws_n, s) == 4
    for B in (0, 17):
        assert L.spw_spmv_tc(ctypes.byref(h), good, good, B, 128, 0.0, None, good, 128, good, ws_n, s) == 1
    assert L.spw_spmv_tc(ctypes.byref(h), None, good, 1, 128, 0.0, None, good, 128, good, ws_n, s) == 1
    for t in (-1.0, float("nan"), float("inf")):
        assert L.spw_spmv_tc(ctypes.byref(h), good, good, 1, 128, t, None, good, 128, good, ws_n, s) == 1
    assert L.spw_spmv_tc(ctypes.byref(h), good, good, 2, 132, 0.0, None, good, 128, good, ws_n, s) == 1
    assert L.spw_spmv_tc(ctypes.byref(h), good, good, 1, 128, 0.0, None, good, 127, good, ws_n, s) == 1
    assert L.spw_spmv_tc(ctypes.byref(h), good, odd, 1, 128, 0.0, None, good, 128, good, ws_n, s) == 2
    # fused FFN: header, batch and gate/up shape checks come first
    other = valid_header(spw, N=192)
    args = (good, good, 1, 128, 0.0, good, 128, good, good, ws_n, s)
    assert L.spw_spmv_ffn(None, good, ctypes.byref(h), *args) == 1
    assert L.spw_spmv_ffn(ctypes.byref(h), good, ctypes.byref(bad), *args) == 4
    assert L.spw_spmv_ffn(ctypes.byref(h), good, ctypes.byref(other), *args) == 1
    for B in (0, 17):
        assert L.spw_spmv_ffn(ctypes.byref(h), good, ctypes.byref(h), good, good, B, 128, 0.0,
                              good, 128, good, good, ws_n, s) == 1
    assert L.spw_spmv_ffn_workspace_bytes(ctypes.byref(h), ctypes.byref(other), 1) == 0


def test_grouping_and_2of4_host_validation_without_gpu(spw):
    L = spw.lib()
    h = valid_header(spw)
    P = ctypes.c_void_p
    good, odd, s = P(0x10000), P(0x10008), P(0)
    big = ctypes.c_uint64(1 << 30)
    # token grouping: arguments, limits and alignment are checked before any launch
    assert L.spw_group_tokens(None, 4, 128, 128, 0.0, 2, good, 128, good, good, good, big, s) == 1
    assert L.spw_group_tokens(good, 0, 128, 128, 0.0, 2, good, 128, good, good, good, big, s) == 1
    assert L.spw_group_tokens(good, 4, 128, 128, 0.0, 0, good, 128, good, good, good, big, s) == 1
    assert L.spw_group_tokens(good, 4, 128, 128, -1.0, 2, good, 128, good, good, good, big, s) == 1
    assert L.spw_group_tokens(good, 4, 128, 128, 0.0, 2, good, 130, good, good, good, big, s) == 1
    assert L.spw_group_tokens(good, 4, 128, 100, 0.0, 2, good, 128, good, good, good, big, s) == 1
    assert L.spw_group_tokens(good, 4, 16385, 16392, 0.0, 2, good, 16392, good, good, good, big, s) == 5
    assert L.spw_group_tokens(good, 16385, 128, 128, 0.0, 2, good, 128, good, good, good, big, s) == 5
    assert L.spw_group_tokens(good, 4, 128, 128, 0.0, 2, good, 128, odd, good, good, big, s) == 2
    assert L.spw_group_tokens(good, 4, 128, 128, 0.0, 2, good, 128, good, good, good,
                              ctypes.c_uint64(16), s) == 3
    assert L.spw_group_tokens_workspace_bytes(4, 128) > 0
    assert L.spw_group_tokens_workspace_bytes(4, 16385) == 0
    # grouped prefill
    ws = ctypes.c_uint64(1 << 30)
    assert L.spw_spmm_tokens(ctypes.byref(h), good, good, 0, 128, 0.0, good, 128, good, ws, s) == 0
    assert L.spw_spmm_tokens(ctypes.byref(h), None, good, 4, 128, 0.0, good, 128, good, ws, s) == 1
    assert L.spw_spmm_tokens(ctypes.byref(h), good, good, 4, 128, 0.0, good, 128, None, ws, s) == 1
    for t in (-1.0, float("nan"), float("inf")):
        assert L.spw_spmm_tokens(ctypes.byref(h), good, good, 4, 128, t, good, 128, good, ws, s) == 1
    assert L.spw_spmm_tokens(ctypes.byref(h), good, good, 4, 132, 0.0, good, 128, good, ws, s) == 1
    assert L.spw_spmm_tokens(ctypes.byref(h), good, odd, 4, 128, 0.0, good, 128, good, ws, s) == 2
    assert L.spw_spmm_tokens(ctypes.byref(h), good, good, 16385, 128, 0.0, good, 128, good, ws, s) == 5
    # 2:4 split and prefill
    assert L.spw_s24_bytes(128, 128) == 4 * 5120 + 1024
    assert L.spw_split24(None, 128, good, 128, 128, 128, good, big, good, 128, s) == 1
    assert L.spw_split24(good, 100, good, 128, 128, 128, good, big, good, 128, s) == 1
    assert L.spw_split24(good, 128, good, 128, 128, 128, odd, big, good, 128, s) == 2
    assert L.spw_split24(good, 128, good, 128, 128, 128, good, ctypes.c_uint64(100), good, 128, s) == 3
    n24 = ctypes.c_uint64(4 * 5120 + 1024)
    assert L.spw_spmm24(ctypes.byref(h), good, good, n24, good, 0, 128, good, 128, None, 0, s) == 0
    assert L.spw_spmm24(ctypes.byref(h), good, None, n24, good, 4, 128, good, 128, None, 0, s) == 1
    assert L.spw_spmm24(ctypes.byref(h), good, odd, n24, good, 4, 128, good, 128, None, 0, s) == 2
    assert L.spw_spmm24(ctypes.byref(h), good, good, ctypes.c_uint64(4 * 5120), good, 4, 128, good, 128,
                        None, 0, s) == 3
    assert L.spw_spmm24(ctypes.byref(h), good, good, n24, good, 4, 132, good, 128, None, 0, s) == 1
    bad = valid_header(spw)
    bad.magic = 0
    assert L.spw_spmm24(ctypes.byref(bad), good, good, n24, good, 4, 128, good, 128, None, 0, s) == 4


def test_auto_decode_path_choice_without_gpu(spw):
    # The choice depends on the batch alone: the CUDA-core decode below the boundary, the
    # tensor-core decode from it up to 16 rows; argument errors of the path taken come back
    # before any device call.
    L = spw.lib()
    h = valid_header(spw)
    P = ctypes.c_void_p
    good, odd, s = P(0x10000), P(0x10008), P(0)
    ws_n = ctypes.c_uint64(1 << 20)
    paths = [L.spw_spmv_auto_path(B) for B in range(1, 17)]
    assert set(paths) <= {0, 1} and paths[0] == 0 and paths[-1] == 1
    first_tc = paths.index(1)
    assert all(p == 1 for p in paths[first_tc:])  # one boundary, monotone in B
    for B in (0, 17, -3):
        assert L.spw_spmv_auto_path(B) == -1
        assert L.spw_spmv_auto_workspace_bytes(ctypes.byref(h), B) == 0
        assert L.spw_spmv_auto(ctypes.byref(h), good, good, B, 128, 0.0, None, good, 128, good, ws_n, s) == 1
    for B in (1, first_tc + 1, 16):
        assert L.spw_spmv_auto(None, good, good, B, 128, 0.0, None, good, 128, good, ws_n, s) == 1
        assert L.spw_spmv_auto(ctypes.byref(h), good, good, B, 128, float("nan"), None, good, 128,
                               good, ws_n, s) == 1
        assert L.spw_spmv_auto(ctypes.byref(h), good, odd, B, 128, 0.0, None, good, 128, good, ws_n, s) == 2
    bad = valid_header(spw)
    bad.magic = 0
    assert L.spw_spmv_auto(ctypes.byref(bad), good, good, 16, 128, 0.0, None, good, 128, good, ws_n, s) == 4
    assert spw.spw_spmv_auto_path(16) == 1 and spw.spw_spmv_auto_path(0) == -1


class _FakeDeviceTensor:
    """Stands in for a CUDA tensor in the size checks (they read only these three)."""
    is_cuda = True

    def __init__(self, n, element_size=4):
        self.n, self.es = n, element_size

    def numel(self):
        return self.n

    def element_size(self):
        return self.es


def test_binding_refuses_host_tensors_and_short_buffers_without_gpu(spw):
    # The library writes through raw pointers and cannot see tensor sizes or devices, so
    # the binding refuses host tensors and short output / workspace buffers before any
    # library call.
    import torch
    host_x = torch.zeros((2, 64), dtype=torch.float16)
    with pytest.raises(ValueError):
        spw.spw_select_threshold(host_x, 0.0)
    with pytest.raises(ValueError):
        spw.spw_compress(host_x, torch.ones((2, 64), dtype=torch.uint8))
    with pytest.raises(ValueError):
        spw._nbytes(torch.zeros(16, dtype=torch.uint8), "ws")
    with pytest.raises(ValueError):
        spw._need_words(torch.zeros(4, dtype=torch.int32), 64)
    with pytest.raises(TypeError):
        spw._mask_like(torch.zeros((2, 64), dtype=torch.uint8), 2, 64)
    F = _FakeDeviceTensor
    assert spw._nbytes(None) == 0 and spw._nbytes(F(10, 2)) == 20
    spw._need_words(F(2), 64)
    with pytest.raises(ValueError):
        spw._need_words(F(1), 64)
    spw._need_words(F(3), 65)
    with pytest.raises(ValueError):
        spw._need_words(F(5, 1), 33)  # 5 bytes hold one word, two are needed
    spw._need_u32(F(4), 4, "idx")
    with pytest.raises(ValueError):
        spw._need_u32(F(3), 4, "idx")


def test_header_compiles_as_plain_c_and_cpp(tmp_path):
    # the boundary is a C ABI: the header must stand alone in C11 and C++17, warning-free
    src = tmp_path / "use_spw.c"
    src.write_text('#include "spw.h"\nint main(void) { return spw_version() > 0 ? 0 : 1; }\n')
    import subprocess
    inc = os.path.join(ROOT, "include")
    for cmd in (["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror"],
                ["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-x", "c++"]):
        proc = subprocess.run(cmd + ["-fsyntax-only", "-I", inc, str(src)], capture_output=True, text=True)
        assert proc.returncode == 0, proc.stderr


def test_plain_c_program_links_and_calls_the_library(spw, tmp_path):
    # a C caller (no Python, no torch) links libspw.so and calls host-side entry points
    import subprocess
    src = tmp_path / "caller.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "spw.h"
int main(void) {
    if (spw_version() != 100) return 1;
    if (strcmp(spw_status_string(SPW_OK), "SPW_OK") != 0) return 2;
    if (spw_spmv_auto_path(16) != 1 || spw_spmv_auto_path(1) != 0 || spw_spmv_auto_path(0) != -1) return 3;
    if (spw_s24_bytes(128, 128) != 4 * 5120 + 1024) return 4;
    if (spw_spmv(NULL, NULL, NULL, 1, 128, 0.0f, NULL, NULL, 128, NULL, 0, NULL) != SPW_ERR_INVALID_ARG)
        return 5;
    puts("ok");
    return 0;
}
''')
    exe = tmp_path / "caller"
    libdir = os.path.dirname(spw_build.LIB)
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir,
                    "-l:libspw.so", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    proc = subprocess.run([str(exe)], capture_output=True, text=True)
    assert proc.returncode == 0 and proc.stdout.strip() == "ok", (proc.returncode, proc.stderr)
