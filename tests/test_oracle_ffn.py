"""Pins for the oracle's FFN activation ("Reduced Matrix Multiplication" §4.2, §3.2).

binary16 rounding is checked against numpy's float64 -> float16 conversion and against
exact round trips; SiLU(g) * u against values fixed outside the oracle: the identity
SiLU(x) - SiLU(-x) = x (so h(x, x) + h(-x, -x) = x^2), its limits, zeros, and a worked
value from e^-1.  A sign error in the exponent, a dropped factor or a wrong rounding
fails one of them."""
import math

import numpy as np
import pytest

import oracle


def test_round_to_half_matches_numpy():
    rng = np.random.default_rng(11)
    v = rng.standard_normal(200000) * 10.0 ** rng.integers(-10, 6, 200000)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(oracle.round_to_half(v).view(np.uint16), ref)


def test_round_to_half_round_trip_and_ties():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    h = bits.view(np.float16)
    finite = np.isfinite(h)
    d = h[finite].astype(np.float64)
    np.testing.assert_array_equal(oracle.round_to_half(d).view(np.uint16), bits[finite])
    # midpoints between neighbouring positive finite values round to the even neighbour
    pos = np.arange(0x0000, 0x7BFF, dtype=np.uint16)
    lo = pos.view(np.float16).astype(np.float64)
    hi = (pos + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2.0
    got = oracle.round_to_half(mid).view(np.uint16)
    even = np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint16)
    np.testing.assert_array_equal(got, even)
    # overflow, infinities, NaN, signed zero
    special = np.array([65504.0, 65519.99, 65520.0, np.inf, -np.inf, -0.0, 2.0 ** -25,
                        2.0 ** -25 * (1 + 2 ** -20)])
    got = oracle.round_to_half(special).view(np.uint16)
    np.testing.assert_array_equal(got, [0x7BFF, 0x7BFF, 0x7C00, 0x7C00, 0xFC00, 0x8000, 0x0000, 0x0001])
    assert np.isnan(oracle.round_to_half(np.array([np.nan]))[0])


def test_silu_mul_worked_value():
    # SiLU(1) * 2 = 2 / (1 + e^-1) = 1.46211715726..., nearest binary16 1.4619140625
    h = oracle.silu_mul(np.array([[1.0]], np.float16), np.array([[2.0]], np.float16))
    assert float(h[0, 0]) == 1.4619140625
    assert abs(2.0 / (1.0 + math.exp(-1.0)) - 1.4619140625) < 2.0 ** -11


def test_silu_odd_part_identity():
    # h(x, x) + h(-x, -x) = x * SiLU(x) + x * (x - SiLU(x)) = x^2, up to two roundings
    x = np.linspace(-12.0, 12.0, 4001).astype(np.float16)
    x = x[x != 0]
    a = oracle.silu_mul(x[None, :], x[None, :])[0].astype(np.float64)
    b = oracle.silu_mul(-x[None, :], -x[None, :])[0].astype(np.float64)
    x2 = x.astype(np.float64) ** 2
    assert np.all(np.abs(a + b - x2) <= x2 * 2.0 ** -10 + 2.0 ** -24)
    assert np.all(a >= 0) and np.all(b >= 0)  # x * SiLU(x) >= 0 for every x


def test_silu_limits_and_zeros():
    g = np.array([[20.0, 30.0, 100.0, -20.0, -30.0, 0.0, 3.0]], np.float16)
    u = np.array([[1.0, 1.0, 1.0, 1.0, 1.0, 5.0, 0.0]], np.float16)
    h = oracle.silu_mul(g, u)[0].astype(np.float64)
    np.testing.assert_array_equal(h[:3], [20.0, 30.0, 100.0])  # SiLU(v) -> v
    assert np.all(np.abs(h[3:5]) < 2.0 ** -20)                 # SiLU(v) -> 0
    assert h[5] == 0.0 and h[6] == 0.0
    assert np.isnan(oracle.silu_mul(np.array([[np.nan]], np.float16), np.array([[1.0]], np.float16))[0, 0])


def test_ffn_identity_gate_and_up():
    # W_gate = I, W_up = 2 I: g = x, u = 2 x, so h = fp16(SiLU(x) * 2 x); the column set
    # is the threshold rule on h
    K = 96
    x = np.linspace(-6.0, 6.0, K).astype(np.float16)[None, :]
    eye = np.eye(K, dtype=np.float16)
    mask = np.eye(K, dtype=np.uint8)
    h, bits = oracle.ffn(eye, mask, (2 * eye).astype(np.float16), mask, x, 0.5)
    xd = x.astype(np.float64)[0]
    want = (xd / (1.0 + np.exp(-xd)) * (2.0 * xd)).astype(np.float16)
    np.testing.assert_array_equal(h[0].view(np.uint16), want.view(np.uint16))
    keep = (want.astype(np.float64) != 0) & ~(np.abs(want.astype(np.float64)) < 0.5)
    got = np.array([(bits[k // 32] >> (k % 32)) & 1 for k in range(K)], dtype=bool)
    np.testing.assert_array_equal(got, keep)
