"""The bench's measurement helpers (CPU).

decode_bytes is the numerator of the reported GB/s and of the roofline fraction: the
values and bitmap words of the active columns plus activations read and outputs
written.  It is checked against a count taken independently from the oracle's TCB
buffer (the bitmap words of active columns, popcounted).  code_sha256 decides whether
the committed DRAM-traffic capture still describes the decode kernel: comment and
whitespace edits must not change it, code edits (string literals included) must."""
import importlib.util
import os

import numpy as np
import pytest

import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def count_from_buffer(buf, N, K, active):
    """Kept weights and bitmap words of the active columns, read from a TCB v1 buffer."""
    off_bitmaps = int(buf[48:56].view(np.uint64)[0])  # header: 8 u32, nnz, bytes_total, then the offsets
    n_strips, n_ktiles = -(-N // 64), -(-K // 64)
    words = buf[off_bitmaps:off_bitmaps + 8 * n_strips * n_ktiles * 64].view(np.uint64)
    words = words.reshape(n_strips, n_ktiles * 64)[:, :K]
    kept = sum(bin(int(w)).count("1") for w in words[:, active].ravel())
    return kept, n_strips * int(active.sum())


@pytest.mark.parametrize("N,K,B,t,zero", [(200, 300, 1, 0.0, 0.5), (130, 70, 3, 0.4, 0.3),
                                          (64, 4097, 2, 0.0, 0.0)])
def test_decode_bytes_counts_active_columns(bench, N, K, B, t, zero):
    W = workloads.weight(N, K, "metric")
    mask = workloads.random_mask(N, K, 0.5, "metric")
    x = workloads.zero_random(workloads.normal_act(B, K, "metric"), zero, "metric")
    bits, _ = oracle.select_threshold(x, t)
    active = np.array([(bits[k // 32] >> (k % 32)) & 1 for k in range(K)], dtype=bool)
    kept, bitmap_words = count_from_buffer(oracle.tcb_encode(W, mask), N, K, active)
    want = 2 * kept + 8 * bitmap_words + 2 * B * K + 2 * B * N
    assert bench.decode_bytes(W, mask, x, t) == want


def test_code_hash_ignores_comments_only(bench):
    src = b'// header\nint f(int a) { /* note */ return a + 1; }\nconst char* s = "// kept";\n'
    h = bench.code_sha256(src)
    assert bench.code_sha256(src.replace(b"// header", b"// other words")) == h
    assert bench.code_sha256(src.replace(b"/* note */", b"")) == h
    assert bench.code_sha256(src.replace(b"return a + 1;", b"return  a+1 ;")) == h
    assert bench.code_sha256(src.replace(b"a + 1", b"a + 2")) != h
    assert bench.code_sha256(src.replace(b'"// kept"', b'"// Kept"')) != h
