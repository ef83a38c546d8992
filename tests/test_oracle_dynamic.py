"""Pins of the dynamic per-tensor NVFP4 activation scale in the oracle (a first
pass takes the largest |x^| of the tensor being quantized; the block quantizer
then runs with g_x = the smallest power of two >= that / (6 * 448)).

They rest on facts independent of the oracle's own code: the static scale of
prepare applies the same formula to the per-channel calibration maxima, so
calibrating on the very input must give the same scale (rounding is monotone);
a power-of-two rescaling of the input must leave every code and block scale
unchanged and scale g_x and y exactly; and the scale is fixed by a brute-force
search over exponents."""
import math

import numpy as np
import pytest

import oracle
import workloads as wl


def _layer(M=40, K=256, N=96, r=16):
    layer = wl.small_layer(M, K, N, r, "nvfp4")
    X, W, b = wl.make_layer_inputs(layer)
    return layer, X, W, b


def _dynamic(prep):
    d = dict(prep)
    d["g_x"] = 0.0
    return d


def test_dynamic_equals_static_calibrated_on_the_same_input():
    _, X, W, b = _layer()
    prep = oracle.prepare(W, b, oracle.calib_absmax(X), 0.5, 16, "nvfp4")
    st = oracle.quantize_act(X, prep)
    dy = oracle.quantize_act(X, _dynamic(prep))
    assert dy["g_x"] == prep["g_x"] == st["g_x"]
    for k in ("codes", "scales", "t"):
        np.testing.assert_array_equal(dy[k], st[k])
    np.testing.assert_array_equal(oracle.forward(X, _dynamic(prep)), oracle.forward(X, prep))


@pytest.mark.parametrize("k", [-6, 3, 9])
def test_dynamic_scale_follows_a_power_of_two_rescaling(k):
    """x -> 2^k x (exact in bf16 here): codes and block scales unchanged, g_x
    and t times 2^k, and with a zero bias y times 2^k exactly."""
    _, X, W, _ = _layer()
    prep = _dynamic(oracle.prepare(W, None, oracle.calib_absmax(X), 0.5, 16, "nvfp4"))
    Xs = wl.f32_to_bf16_bits(oracle.bf16_to_f32(X) * np.float32(2.0 ** k))
    np.testing.assert_array_equal(oracle.bf16_to_f32(Xs), oracle.bf16_to_f32(X) * np.float32(2.0 ** k))
    a, b = oracle.quantize_act(X, prep), oracle.quantize_act(Xs, prep)
    assert b["g_x"] == a["g_x"] * 2.0 ** k
    np.testing.assert_array_equal(b["codes"], a["codes"])
    np.testing.assert_array_equal(b["scales"], a["scales"])
    np.testing.assert_array_equal(oracle.bf16_to_f32(b["t"]), oracle.bf16_to_f32(a["t"]) * np.float32(2.0 ** k))
    ya, yb = oracle.forward_from_act(a, prep), oracle.forward_from_act(b, prep)
    np.testing.assert_array_equal(oracle.bf16_to_f32(yb), oracle.bf16_to_f32(ya) * np.float32(2.0 ** k))


def test_static_scale_does_not_follow_a_rescaling():
    """The reason for the dynamic variant: with the calibrated static scale, an
    input 2^9 times larger than the calibration saturates the block scales."""
    _, X, W, _ = _layer()
    prep = oracle.prepare(W, None, oracle.calib_absmax(X), 0.5, 16, "nvfp4")
    Xs = wl.f32_to_bf16_bits(oracle.bf16_to_f32(X) * np.float32(512.0))
    yd_ref = oracle.bf16_to_f32(oracle.forward(Xs, _dynamic(prep))).astype(np.float64)
    yd_st = oracle.bf16_to_f32(oracle.forward(Xs, prep)).astype(np.float64)
    e_dyn = np.linalg.norm(yd_ref - 512.0 * oracle.bf16_to_f32(oracle.forward(X, prep)))
    e_st = np.linalg.norm(yd_st - 512.0 * oracle.bf16_to_f32(oracle.forward(X, prep)))
    assert e_st > 10 * max(e_dyn, 1e-30)


def _brute_scale(amax):
    if amax == 0:
        return 1.0
    e = -160
    while 2688.0 * 2.0 ** e < amax:  # exact comparisons: 2688 * 2^e is exact in binary64
        e += 1
    return 2.0 ** e


@pytest.mark.parametrize("amax", [0.0, 1.0, 2688.0, 2688.0 * 2 ** -20, math.nextafter(2688.0, 1e9),
                                  math.nextafter(2688.0, 0.0), 3.0e-7, 65504.0, 1.7e38])
def test_tensor_scale_is_the_smallest_power_of_two_covering_amax(amax):
    a = np.float32(amax)
    x = np.array([[0.0, -float(a), float(a) / 3.0]], np.float32)
    assert oracle.act_tensor_scale(x) == _brute_scale(float(a))
