"""Pins of the oracle's GELU (erf form), the activation between the MLP linears
of the fused MLP pair: the standard normal CDF at printed points, the odd-part
identity GELU(h) - GELU(-h) = h, the asymptotes, and the bf16 rounding against
brute force."""
import math

import numpy as np

import oracle


def test_normal_cdf_points():
    # GELU(h) = h Phi(h); Phi(1) and Phi(2) are textbook values of the normal CDF
    np.testing.assert_allclose(oracle.gelu_f64(np.array([1.0, 2.0, -1.0])),
                               [0.8413447460685429, 2 * 0.9772498680518208, -(1 - 0.8413447460685429)],
                               rtol=1e-15, atol=1e-16)
    assert oracle.gelu_f64(np.array([0.0]))[0] == 0.0


def test_negative_tail():
    # Phi(-10) = 7.6198530241604696e-24, Phi(-8) = 6.2209605742717841e-16 (normal CDF tables)
    np.testing.assert_allclose(oracle.gelu_f64(np.array([-10.0, -8.0])),
                               [-10 * 7.6198530241604696e-24, -8 * 6.2209605742717841e-16], rtol=1e-13)
    # the tail is kept through the bf16 rounding: bf16 has binary32's exponent range
    assert oracle.bf16_to_f32(oracle.gelu_bf16(oracle.f32_to_bf16(np.array([-9.25], np.float32))))[0] < 0


def test_odd_part_identity_and_asymptotes():
    h = np.linspace(-9.0, 9.0, 1801)
    g = oracle.gelu_f64(h)
    np.testing.assert_allclose(g - oracle.gelu_f64(-h), h, rtol=0, atol=1e-14)
    big = np.array([12.0, 30.0, 1e4])
    np.testing.assert_array_equal(oracle.gelu_f64(big), big)
    assert np.all(np.abs(oracle.gelu_f64(-big)) < 1e-30)
    # near zero GELU(h) = h/2 + h^2/sqrt(2 pi) + O(h^4)
    t = np.array([1e-6, -1e-6])
    np.testing.assert_allclose(oracle.gelu_f64(t), t / 2 + t * t / math.sqrt(2 * math.pi), rtol=1e-9)


def test_bf16_rounding_brute_force():
    rng = np.random.default_rng(0)
    hb = rng.integers(0, 1 << 16, 4000).astype(np.uint16)
    hb = hb[np.isfinite(oracle.bf16_to_f32(hb)) & (np.abs(oracle.bf16_to_f32(hb)) < 1e30)]
    got = oracle.gelu_bf16(hb)
    for h, gbits in zip(hb[:600], got[:600]):
        x = float(oracle.bf16_to_f32(np.array([h]))[0])
        g = 0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0)))
        if g == 0.0:
            assert oracle.bf16_to_f32(np.array([gbits]))[0] == 0.0
            continue
        # nearest bf16 by exhaustive search over the neighbours of the truncation
        u = int(np.array([g], np.float32).view(np.uint32)[0]) >> 16
        cands = np.array([(u + d) & 0xFFFF for d in (-1, 0, 1, 2)], np.uint16)
        vals = oracle.bf16_to_f32(cands).astype(np.float64)
        keep = np.isfinite(vals) & (np.sign(vals) * np.sign(g) >= 0)
        cands, vals = cands[keep], vals[keep]
        err = np.abs(vals - g)
        best = cands[err == err.min()]
        if best.size > 1:  # a tie: the even mantissa
            best = best[(best & 1) == 0]
        assert gbits == best[0], (h, g, gbits)
