"""Checks of the seeded input generators (the workload recipe, not the method)."""
import numpy as np

import workloads


def test_seeds_are_stable_and_distinct():
    a = workloads.weight(8, 8, "x")
    b = workloads.weight(8, 8, "x")
    c = workloads.weight(8, 8, "y")
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)
    assert workloads.seed_of("cfg", 1) == workloads.seed_of("cfg", 1)


def test_magnitude_mask_keeps_largest_per_row():
    W = workloads.weight(64, 4096, "m")
    for s, keep in ((0.5, 2048), (0.6, 1639), (0.7, 1229), (0.4, 2458), (0.8, 820)):
        m = workloads.magnitude_mask(W, s)
        assert (m.sum(axis=1) == keep).all()
        mag = np.abs(W.astype(np.float64))
        assert (np.where(m == 1, mag, np.inf).min(axis=1) >=
                np.where(m == 0, mag, -np.inf).max(axis=1)).all()


def test_zero_smallest_counts_and_threshold():
    x = workloads.silu_gate_up_act(4, 11008, "z")
    for a in (0.0, 0.3, 0.5, 0.7):
        zx, t = workloads.zero_smallest(x, a)
        nz = int(np.floor(a * 11008 + 1e-9))
        # the zeroed count can exceed nz only by entries that were already zero
        assert ((zx == 0).sum(axis=1) >= nz).all()
        kept = np.abs(zx.astype(np.float64))
        kept[zx == 0] = np.inf
        assert np.allclose(kept.min(axis=1), t) or a == 0.0


def test_shapes():
    assert workloads.LLAMA7B_LAYERS["down"] == (4096, 11008)
    assert workloads.LLAMA13B_SHAPES["gate_up"] == (13824, 5120)


def test_magnitude_mask_ties_go_to_lower_index():
    W = np.array([[1, -1, 2, 1, 0, -2]], dtype=np.float16)
    np.testing.assert_array_equal(workloads.magnitude_mask(W, 0.5)[0], [1, 0, 1, 0, 0, 1])
    np.testing.assert_array_equal(workloads.magnitude_mask(W, 0.0)[0], [1] * 6)
    np.testing.assert_array_equal(workloads.magnitude_mask(W, 1.0)[0], [0] * 6)
    # NaN-free magnitude order on fp16 bits matches the numeric order
    W = workloads.weight(4, 300, "tie")
    m = workloads.magnitude_mask(W, 0.3)
    mag = np.abs(W.astype(np.float64))
    for r in range(4):
        order = sorted(range(300), key=lambda c: (-mag[r, c], c))[:300 - 90]
        assert set(np.nonzero(m[r])[0]) == set(order)
