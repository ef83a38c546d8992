"""Pins of the INT8 tensorwise W8A8 oracle against the format definition and
plain arithmetic: a layer built so that every step is exact equals the dense
product; a loop-level brute force in Python integers; the quantizer's error is
at most half a step, it is odd-symmetric and maps +-max|v| to +-127; an all-zero
input gives codes 0 and y = bias."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl
from fp_exact import f32_of_bits, fl32

bf = oracle.bf16_to_f32


def _bf16(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_w8a8_exact_layer_equals_dense_product():
    """Power-of-two scales and grid values make every step exact (127 * 2^e is
    exact in bf16's 8 significant bits), so the layer equals bf16(x W^T + b)."""
    rng = np.random.default_rng(21)
    M, K, N = 5, 96, 7
    qx = rng.integers(-127, 128, (M, K))
    qw = rng.integers(-127, 128, (N, K))
    qx[0, 0], qw[0, 0] = 127, -127  # the tensors reach max|v| = 127 * step
    X = _bf16(qx * 2.0 ** -9)
    W = _bf16(qw * 2.0 ** -12)
    assert np.array_equal(bf(X), (qx * 2.0 ** -9).astype(np.float32))
    b = _bf16(rng.standard_normal(N) * 0.01)
    prep = oracle.w8a8_prepare(W, b)
    act = oracle.w8a8_quantize_act(X)
    assert prep["s_w"] == np.float32(2.0 ** -12) and act["s_x"] == np.float32(2.0 ** -9)
    np.testing.assert_array_equal(prep["wcodes"], qw)
    np.testing.assert_array_equal(act["codes"], qx)
    ref = oracle.f64_to_bf16(bf(X).astype(np.float64) @ bf(W).astype(np.float64).T + bf(b).astype(np.float64))
    np.testing.assert_array_equal(oracle.w8a8_forward(X, prep), ref)


def test_w8a8_forward_brute_force_tiny():
    rng = np.random.default_rng(22)
    M, K, N = 3, 32, 4
    X = _bf16(rng.standard_normal((M, K)))
    W = _bf16(rng.standard_normal((N, K)) * 0.05)
    b = _bf16(rng.standard_normal(N) * 0.01)
    prep = oracle.w8a8_prepare(W, b)
    act = oracle.w8a8_quantize_act(X)
    y = oracle.w8a8_forward(X, prep)
    for m in range(M):
        for n in range(N):
            acc = sum(int(act["codes"][m, k]) * int(prep["wcodes"][n, k]) for k in range(K))
            v = float(act["s_x"]) * float(prep["s_w"]) * acc + float(bf(b)[n])
            assert y[m, n] == oracle.f64_to_bf16(np.array([v]))[0]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_w8_quantizer_properties(seed):
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal((17, 64)) * rng.uniform(0.01, 100)).astype(np.float32)
    s = oracle.w8_tensor_scale(v)
    assert s == np.float32(np.float32(np.abs(v).max()) / np.float32(127))
    q = oracle.quant_w8(v, s)
    np.testing.assert_array_equal(oracle.quant_w8(-v, s), -q)  # odd symmetry
    i = np.unravel_index(np.argmax(np.abs(v)), v.shape)
    assert abs(int(q[i])) == 127
    err = np.abs(q.astype(np.float64) * float(s) - v.astype(np.float64))
    assert np.all(err <= 0.5 * float(s) * (1 + 2.0 ** -20))  # half a step (the reciprocal is rounded)


def test_w8_code_uses_the_binary32_reciprocal():
    """Worked example of the reading q = rne(fl32(v * fl32(1/s))), s = fl32(max|v| / 127):
    for these two binary32 values the exact quotient v / s is -110.500004..., which a
    division would round to -111; the binary32 reciprocal gives -110."""
    amax, v = f32_of_bits(0x3FBA4BF1), f32_of_bits(0xBFA217BF)
    s = fl32(amax / 127)
    assert round(fl32(v * fl32(1 / s))) == -110 and round(v / s) == -111
    x = np.array([[float(amax), float(v)]], np.float32)
    assert Fraction(float(oracle.w8_tensor_scale(x))) == s
    q = oracle.quant_w8(x, oracle.w8_tensor_scale(x))
    assert q[0, 0] == 127 and q[0, 1] == -110


def test_w8_ties_round_to_even():
    """With s = 2^-3 every value (k + 1/2) / 8 is an exact tie; the codes take the even
    neighbour (0.5 -> 0, 1.5 -> 2, -2.5 -> -2, ...)."""
    k = np.arange(-127, 126)
    x = np.concatenate([[127 / 8.0], (k + 0.5) / 8.0]).astype(np.float32)[None, :]
    s = oracle.w8_tensor_scale(x)
    assert s == np.float32(0.125)
    q = oracle.quant_w8(x, s)[0, 1:]
    want = [round(Fraction(int(j)) + Fraction(1, 2)) for j in k]
    np.testing.assert_array_equal(q, want)


def test_w8a8_output_rounds_once():
    """y is formed in binary64 and rounded once: with unit scales and an integer product
    of 2^24 + 2^16 + 1 (above the bf16 tie at 2^24 + 2^16), y rounds up to 2^24 + 2^17
    (0x4B81); a binary32 detour would land on the tie and give 2^24."""
    qx = np.array([127] * 1044 + [127, 13], np.int8)
    qw = np.array([127] * 1044 + [32, 1], np.int8)
    assert int(qx.astype(np.int64) @ qw.astype(np.int64)) == 2**24 + 2**16 + 1
    act = dict(codes=qx[None, :], s_x=np.float32(1.0))
    prep = dict(wcodes=qw[None, :], s_w=np.float32(1.0), bias=np.zeros(1, np.uint16))
    assert oracle.w8a8_forward_from_act(act, prep)[0, 0] == 0x4B81


def test_w8a8_zero_input_gives_bias():
    W = _bf16(np.random.default_rng(3).standard_normal((6, 64)))
    b = _bf16(np.arange(6) * 0.25)
    prep = oracle.w8a8_prepare(W, b)
    X = np.zeros((2, 64), np.uint16)
    act = oracle.w8a8_quantize_act(X)
    assert act["s_x"] == 0 and not act["codes"].any()
    np.testing.assert_array_equal(oracle.w8a8_forward(X, prep), np.tile(b, (2, 1)))
