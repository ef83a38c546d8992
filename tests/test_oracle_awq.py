"""Pins of the awq_w4a16 oracle (4-bit weights, 16-bit activations) against what
the definition and the mathematics fix, independently of the oracle's own code:
exactly representable layers, a loop-level brute force from the nibble format,
the unit-scale reduction to plain group-INT4, and the method's claim that the
activation-aware scale protects the weights of outlier channels."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl
from fp_exact import bf16 as bf16_exact
from fp_exact import f32_of_bits, fl32

bf = oracle.bf16_to_f32


def _bf16(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


def _nibble_decode(codes):
    """Two's-complement nibbles, element 2i in the low half of byte i (format definition)."""
    lo = (codes & 0x0F).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    q = np.empty((codes.shape[0], 2 * codes.shape[1]), np.int64)
    q[:, 0::2], q[:, 1::2] = lo, hi
    return np.where(q >= 8, q - 16, q)


def _f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def test_awq_exact_layer_equals_dense_product():
    """Channel scales that are powers of two (mean|x_j| = 4^k_j, alpha = 1/2, so
    s_j = 2^k_j) and weights with W s exactly on the INT4 grid of each group make
    every step exact: the layer must equal bf16(x W^T + b) computed directly."""
    rng = np.random.default_rng(5)
    M, K, N = 4, 128, 6
    k = rng.integers(-2, 3, K)  # s_j = 2^k_j
    X = _bf16(rng.choice([-1.0, 1.0], (M, K)) * (4.0 ** k)[None, :])
    e = rng.integers(3, 7, (N, K // 64))  # group step 2^-e
    c = rng.integers(-7, 8, (N, K))
    c[:, ::64] = 7  # every group reaches amax = 7 * step, so its fp16 scale is the step exactly
    Ws = c * (2.0 ** -np.repeat(e, 64, axis=1))  # W diag(s), on the grid
    W = _bf16(Ws / (2.0 ** k)[None, :])
    b = _bf16(rng.standard_normal(N) * 0.1)
    prep = oracle.awq_prepare(W, b, X, alphas=(0.5,))
    np.testing.assert_array_equal(prep["s"], (2.0 ** k).astype(np.float32))
    np.testing.assert_array_equal(prep["inv_s"], (2.0 ** -k).astype(np.float32))
    np.testing.assert_array_equal(_nibble_decode(prep["wcodes"]), c)
    np.testing.assert_array_equal(_f16(prep["wscales"]), 2.0 ** -e)
    y_ref = oracle.f64_to_bf16(bf(X).astype(np.float64) @ bf(W).astype(np.float64).T + bf(b).astype(np.float64))
    np.testing.assert_array_equal(oracle.awq_forward(X, prep), y_ref)


def test_awq_statistic_is_the_channel_mean():
    """Worked example: the activation-aware statistic is mean |x| per input channel
    (not the maximum), and s = mean^alpha with s = 1 for an all-zero channel."""
    X = _bf16([[1.0, -2.0, 0.0, 0.5], [3.0, 6.0, 0.0, -0.5], [-2.0, 4.0, 0.0, 1.5]])
    np.testing.assert_allclose(oracle.awq_mean_abs(X), [2.0, 4.0, 0.0, 2.5 / 3], rtol=1e-15)
    s, s_f, inv = oracle.awq_channel_scales(oracle.awq_mean_abs(X), 0.5)
    np.testing.assert_allclose(s, [np.sqrt(2.0), 2.0, 1.0, np.sqrt(2.5 / 3)], rtol=1e-15)
    W = _bf16(np.random.default_rng(9).standard_normal((3, 64 * 1))[:, :4].repeat(16, axis=1) * 0.05)
    Xw = np.tile(X, (1, 16))
    prep = oracle.awq_prepare(W, None, Xw, alphas=(1.0,))
    np.testing.assert_array_equal(prep["s"], np.tile(np.float32([2.0, 4.0, 1.0, 2.5 / 3]), 16))


def test_awq_smoothed_input_is_binary32():
    """The smoothed activation is one binary32 product fl32(x * inv_s) before the binary64
    sum: with x = 3 and this inv_s, 3 * inv_s lies just above the bf16 tie 1.03515625 and
    rounds onto it in binary32, so y = bf16(tie) = 1.03125 (the even neighbour, 0x3F84);
    the unrounded product would give 1.0390625."""
    inv = f32_of_bits(0x3EB0AAAB)
    tie = fl32(3 * inv)
    assert tie == 1 + Fraction(9, 256) and 3 * inv > tie
    assert bf16_exact(tie) == Fraction(33, 32) and bf16_exact(3 * inv) == 1 + Fraction(5, 128)
    K = 64
    inv_s = np.ones(K, np.float32)
    inv_s[0] = float(inv)
    wcodes = np.zeros((1, K // 2), np.uint8)
    wcodes[0, 0] = 0x01  # q = 1 at k = 0
    prep = dict(N=1, K=K, inv_s=inv_s, wcodes=wcodes, wscales=np.array([[0x3C00]], np.uint16),
                bias=np.zeros(1, np.uint16))
    X = np.zeros((1, K), np.uint16)
    X[0, 0] = 0x4040  # 3.0
    assert oracle.awq_forward(X, prep)[0, 0] == 0x3F84


def test_awq_forward_brute_force_tiny():
    """Loop-level evaluation from the stored codes and scales (no matrix routines)."""
    rng = np.random.default_rng(6)
    M, K, N = 2, 64, 3
    X = _bf16(rng.standard_normal((M, K)))
    W = _bf16(rng.standard_normal((N, K)) * 0.05)
    b = _bf16(rng.standard_normal(N) * 0.01)
    prep = oracle.awq_prepare(W, b, X)
    q = _nibble_decode(prep["wcodes"])
    S = _f16(prep["wscales"])
    xf = bf(X)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for kk in range(K):
                xh = float(np.float32(xf[m, kk]) * np.float32(prep["inv_s"][kk]))  # binary32 product
                acc += xh * (q[n, kk] * S[n, kk // 64])
            acc += float(bf(b)[n])
            assert oracle.awq_forward(X, prep)[m, n] == oracle.f64_to_bf16(np.array([acc]))[0]


def test_awq_unit_scale_is_plain_group_int4():
    """alpha = 0 makes every s_j = 1: the layer is group-INT4 weight-only
    quantization, with scales fp16(amax/7) and round-half-even codes."""
    rng = np.random.default_rng(7)
    M, K, N = 3, 256, 5
    X = _bf16(rng.standard_normal((M, K)))
    W = _bf16(rng.standard_normal((N, K)) * 0.05)
    prep = oracle.awq_prepare(W, None, X, alphas=(0.0,))
    assert np.all(prep["s"] == 1.0) and np.all(prep["inv_s"] == 1.0)
    wf = bf(W).reshape(N, K // 64, 64)  # binary32, as the quantizer works
    amax = np.abs(wf).max(axis=2)
    S = (amax / np.float32(7.0)).astype(np.float16)  # binary32 quotient, then fp16 round-to-nearest-even
    np.testing.assert_array_equal(_f16(prep["wscales"]), S.astype(np.float64))
    inv = (np.float32(1.0) / S.astype(np.float32))  # correctly rounded binary32 reciprocal
    q = np.clip(np.rint(wf * inv[:, :, None]), -8, 7).reshape(N, K)
    np.testing.assert_array_equal(_nibble_decode(prep["wcodes"]), q)


def test_awq_zero_channel_keeps_unit_scale():
    _, s_f, inv = oracle.awq_channel_scales(np.array([0.0, 4.0, 0.25]), 0.5)
    np.testing.assert_array_equal(s_f, np.array([1.0, 2.0, 0.5], np.float32))
    np.testing.assert_array_equal(inv, np.array([1.0, 0.5, 2.0], np.float32))


def test_awq_scale_helps_on_outlier_channels():
    """On inputs with a few large channels (the FLUX-style x50 outliers) the
    searched scale must beat plain W4A16 (alpha = 0) clearly."""
    rng = np.random.default_rng(8)
    M, K, N = 64, 512, 128
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.choice(K, 6, replace=False)] *= 50.0
    X = _bf16(x)
    W = _bf16(rng.standard_normal((N, K)) * 0.02)
    prep = oracle.awq_prepare(W, None, X)
    err0 = oracle.awq_output_error(X, W, oracle.awq_mean_abs(X), 0.0)
    assert prep["alpha"] > 0.0
    assert prep["err"] < 0.8 * err0, (prep["alpha"], prep["err"], err0)
