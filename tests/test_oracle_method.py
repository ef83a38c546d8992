"""Pins for the oracle's method steps against closed forms, invariants, brute
force and independent library routines (numpy matmul / eigvalsh)."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl
from fp_exact import fl32


def _bf(x):
    return oracle.bf16_to_f32(x).astype(np.float64)


# ----------------------------------------------------------------------------- smoothing
def test_smoothing_closed_forms():
    rng = np.random.default_rng(0)
    ax = rng.uniform(0.1, 50, 64).astype(np.float32)
    aw = rng.uniform(0.01, 0.1, 64).astype(np.float32)
    ax[3] = 0.0
    aw[5] = 0.0
    ld, lf, il = oracle.smooth_factors(ax, aw, 0.0)
    ok = (ax > 0) & (aw > 0)
    assert np.allclose(ld[ok], 1.0 / aw[ok].astype(np.float64), rtol=1e-15)
    ld, lf, il = oracle.smooth_factors(ax, aw, 1.0)
    assert np.allclose(ld[ok], ax[ok], rtol=1e-15)
    assert ld[3] == 1.0 and ld[5] == 1.0
    ld, lf, il = oracle.smooth_factors(ax, aw, 0.5)
    assert np.allclose(ld[ok], np.sqrt(ax[ok].astype(np.float64) / aw[ok]), rtol=1e-14)
    assert np.array_equal(lf, ld.astype(np.float32))
    assert np.array_equal(il, (1.0 / ld).astype(np.float32))


def test_smoothing_preserves_product():
    layer = wl.small_layer(64, 256, 128, 16, "int4")
    X, W, b = wl.make_layer_inputs(layer)
    amax_x = oracle.calib_absmax(X)
    amax_w = np.abs(oracle.bf16_to_f32(W)).max(axis=0)
    ld, lf, il = oracle.smooth_factors(amax_x, amax_w, 0.5)
    xhat = oracle.smooth_act(X, il).astype(np.float64)
    What = _bf(W) * lf.astype(np.float64)[None, :]
    ref = _bf(X) @ _bf(W).T
    got = xhat @ What.T
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-6
    # outlier channels get lambda > typical: the smoothed activation max is flattened
    assert np.abs(xhat).max(axis=0).max() / np.median(np.abs(xhat).max(axis=0)) < \
        np.abs(_bf(X)).max(axis=0).max() / np.median(np.abs(_bf(X)).max(axis=0))


# ----------------------------------------------------------------------------- SVD split
def test_svd_recovers_known_spectrum():
    rng = np.random.default_rng(1)
    N, K = 48, 32
    Q1, _ = np.linalg.qr(rng.standard_normal((N, N)))
    Q2, _ = np.linalg.qr(rng.standard_normal((K, K)))
    sig = np.sort(rng.uniform(0.1, 10, K))[::-1]
    What = Q1[:, :K] @ np.diag(sig) @ Q2.T
    L1, L2, S = oracle.svd_lowrank_factors(What, 8)
    assert np.allclose(S, sig, rtol=1e-12)
    exact_r = Q1[:, :8] @ np.diag(sig[:8]) @ Q2[:, :8].T
    assert np.linalg.norm((L1 @ L2).T - exact_r) < 1e-10 * np.linalg.norm(What)
    # balanced split: columns of L1 and rows of L2 carry sqrt(sigma) each
    assert np.allclose(np.linalg.norm(L1, axis=0), np.sqrt(sig[:8]), rtol=1e-12)
    assert np.allclose(np.linalg.norm(L2, axis=1), np.sqrt(sig[:8]), rtol=1e-12)


def test_eckart_young_and_monotone_in_rank():
    rng = np.random.default_rng(2)
    N, K = 96, 64
    What = rng.standard_normal((N, K)) * 0.02
    What[:, [3, 17]] *= 40.0  # smoothed outlier columns
    ev = np.sort(np.linalg.eigvalsh(What.T @ What))[::-1]  # independent routine
    prev = np.inf
    for r in [0, 1, 2, 4, 8, 16, 32, 64]:
        if r:
            L1, L2, S = oracle.svd_lowrank_factors(What, r)
            err = np.linalg.norm(What - (L1 @ L2).T) ** 2
        else:
            err = np.linalg.norm(What) ** 2
        assert err == pytest.approx(ev[r:].sum(), rel=1e-9, abs=1e-20)
        assert err <= prev * (1 + 1e-12)
        prev = err
    L1, L2, S = oracle.svd_lowrank_factors(What, min(N, K))
    assert np.linalg.norm(What - (L1 @ L2).T) <= 1e-12 * np.linalg.norm(What)


def test_prepare_residual_uses_rounded_factors():
    layer = wl.small_layer(64, 256, 128, 32, "nvfp4")
    X, W, b = wl.make_layer_inputs(layer)
    p = oracle.prepare(W, b, oracle.calib_absmax(X), 0.5, 32, "nvfp4")
    What = _bf(W) * p["lam"].astype(np.float64)[None, :]
    recon = (_bf(p["L1"]) @ _bf(p["L2"])).T + p["R"].astype(np.float64)
    # R is W^ - (L1 L2)^T with the bf16 factors, rounded once to binary32
    assert np.max(np.abs(recon - What)) <= np.max(np.abs(What)) * 2.0**-24 * 1.01
    # full rank: the residual is only the bf16 rounding noise of the factors
    pf = oracle.prepare(W, b, oracle.calib_absmax(X), 0.5, 128, "nvfp4")
    assert np.linalg.norm(pf["R"]) < 0.02 * np.linalg.norm(What)
    # the layer's bias passes through unchanged; no bias means zeros
    assert np.array_equal(p["bias"], b) and b.any()
    assert not oracle.prepare(W, None, oracle.calib_absmax(X), 0.5, 32, "nvfp4")["bias"].any()


# ----------------------------------------------------------------------------- quantizers
def test_int4_roundtrip_exact_codes():
    rng = np.random.default_rng(3)
    rows, K = 8, 256
    c = rng.integers(-7, 8, (rows, K))
    c[:, ::64] = 7  # make amax = 7 S in every group, so S = fp16(amax / 7) is exact
    S = 2.0 ** rng.integers(-6, 4, (rows, K // 64))
    v = (c * np.repeat(S, 64, axis=1)).astype(np.float32)
    codes, scales = oracle.quant_int4(v)
    assert np.array_equal(oracle.f16_to_f32(scales).astype(np.float64), S)
    lo = (codes & 0xF).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    q = np.empty((rows, K), np.int64)
    q[:, 0::2], q[:, 1::2] = lo, hi
    q[q >= 8] -= 16
    assert np.array_equal(q, c)
    assert np.array_equal(oracle.dequant(codes, scales, "int4"), v.astype(np.float64))


def test_int4_error_bound_and_zero_group():
    rng = np.random.default_rng(4)
    v = (rng.standard_normal((16, 512)) * np.exp(rng.uniform(-8, 3, (16, 1)))).astype(np.float32)
    v[2, 64:128] = 0.0
    codes, scales = oracle.quant_int4(v)
    S = np.repeat(oracle.f16_to_f32(scales).astype(np.float64), 64, axis=1)
    dq = oracle.dequant(codes, scales, "int4")
    assert np.all(np.abs(dq - v) <= 0.5 * S * (1 + 1e-6) + 1e-30)
    assert np.all(codes[2, 32:64] == 0) and scales[2, 1] == 0
    # scale is amax / 7 up to one fp16 rounding
    amax = np.abs(v.astype(np.float64)).reshape(16, 8, 64).max(axis=2)
    assert np.all(np.abs(oracle.f16_to_f32(scales) - amax / 7) <= amax / 7 * 2.0**-11 * 1.001 + 2.0**-25)


def test_nvfp4_roundtrip_on_grid():
    rng = np.random.default_rng(5)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    rows, K, g = 4, 128, 2.0**-3
    idx = rng.integers(0, 8, (rows, K))
    sgn = rng.choice([-1.0, 1.0], (rows, K))
    idx[:, ::16] = 7  # block amax = 6 d, so sb = e4m3(6 d / (6 g)) = d / g exactly
    sb = oracle.e4m3_to_f32(rng.integers(0x20, 0x60, (rows, K // 16)).astype(np.uint8)).astype(np.float64)
    v = (sgn * grid[idx] * np.repeat(sb * g, 16, axis=1)).astype(np.float32)
    codes, scales = oracle.quant_nvfp4(v, g)
    assert np.array_equal(oracle.e4m3_to_f32(scales).astype(np.float64), sb)
    assert np.array_equal(oracle.dequant(codes, scales, "nvfp4", g), v.astype(np.float64))


def test_nvfp4_error_bound():
    rng = np.random.default_rng(6)
    v = (rng.standard_normal((16, 256)) * 3).astype(np.float32)
    v[:, 7] *= 30
    g = oracle.pow2_scale(float(np.abs(v).max()))
    assert g >= np.abs(v).max() / 2688 and g / 2 < np.abs(v).max() / 2688
    codes, scales = oracle.quant_nvfp4(v, g)
    assert scales.max() <= 0x7E  # never saturated when g comes from the tensor max
    d = np.repeat(oracle.e4m3_to_f32(scales).astype(np.float64) * g, 16, axis=1)
    dq = oracle.dequant(codes, scales, "nvfp4", g)
    # spacing of E2M1 at |v|/d: 0.5 below 2, 1 in [2,4), 2 in [4,6]; error <= half spacing
    a = np.abs(v) / d
    half = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0)) * d
    assert np.all(np.abs(dq - v) <= half * (1 + 1e-6))


def test_nvfp4_zero_scale_blocks_have_zero_codes():
    """A block whose amax / (6 g) rounds to the E4M3 zero (below half the smallest
    subnormal, 2^-10) has scale 0, and every code of it is +0 (0x0) -- for an all-zero
    block and for tiny nonzero values of either sign alike."""
    g = 1.0
    v = np.zeros((3, 64), np.float32)
    v[1, 16:32] = np.linspace(-0.005, 0.004, 16)  # amax / 6 < 2^-10
    v[2, 48:64] = -0.0051
    v[0, 0:16] = np.linspace(-3, 3, 16)  # a normal block beside them
    codes, scales = oracle.quant_nvfp4(v, g)
    assert scales[0, 0] != 0
    zero_blocks = [(0, 1), (0, 2), (0, 3), (1, 0), (1, 1), (1, 2), (1, 3), (2, 0), (2, 1), (2, 2), (2, 3)]
    for r, blk in zero_blocks:
        assert scales[r, blk] == 0
        assert not codes[r, 8 * blk:8 * blk + 8].any(), (r, blk)


def test_int4_code_uses_the_binary32_reciprocal():
    """Worked example of the INT4 reading code = rne(fl32(x * fl32(1/S))): with S = fp16
    0x3D25 = 1317/1024 and x = 3.5 S exactly, the exact quotient is the tie 3.5 (a
    division would round it to 4), while the binary32 reciprocal puts the product just
    below the tie: code 3."""
    S = Fraction(1317, 1024)
    x = Fraction(7, 2) * S
    p = fl32(x * fl32(1 / S))
    assert p < Fraction(7, 2) and round(p) == 3 and round(x / S) == 4
    v = np.zeros((1, 64), np.float32)
    v[0, 0], v[0, 1] = float(7 * S), float(x)  # the group's amax makes fp16(amax / 7) = S exactly
    codes, scales = oracle.quant_int4(v)
    assert oracle.f16_to_f32(scales)[0, 0] == float(S)
    q = _unpack_int4(codes)
    assert q[0, 0] == 7 and q[0, 1] == 3


def test_nvfp4_code_uses_the_binary32_reciprocal():
    """Worked example of the NVFP4 reading code = e2m1_rne(fl32(x * fl32(1/d))): with the
    block scale d = 1.875 (E4M3 0x3F, g = 1) and x = 1.25 d, the exact quotient is the
    tie 1.25 between 1 and 1.5 (a division would round to the even neighbour 1), while
    the binary32 reciprocal lands just above it: 1.5, code 0x3."""
    d = Fraction(15, 8)
    x = Fraction(5, 4) * d
    assert fl32(x * fl32(1 / d)) > Fraction(5, 4)
    v = np.zeros((1, 16), np.float32)
    v[0, 0], v[0, 1] = float(6 * d), float(x)  # amax / 6 = d exactly
    codes, scales = oracle.quant_nvfp4(v, 1.0)
    assert scales[0, 0] == 0x3F
    assert codes[0, 0] & 0xF == 0x7 and codes[0, 0] >> 4 == 0x3  # 6 and 1.5 (E2M1: sign, 2 exponent bits, 1 mantissa bit)


def test_tensor_scales_are_tight():
    """g is the smallest power of two with 6 * 448 * g >= amax of the tensor it scales,
    so the block holding that amax gets an E4M3 scale in [224, 448]: for the weight
    residual (g_w from |R|) and, on the calibration input itself, for the activations
    (static g_x from the smoothed calibration maxima)."""
    layer = wl.small_layer(64, 512, 128, 32, "nvfp4")
    X, W, b = wl.make_layer_inputs(layer)
    p = oracle.prepare(W, b, oracle.calib_absmax(X), 0.5, 32, "nvfp4")
    sw = oracle.e4m3_to_f32(p["wscales"]).astype(np.float64)
    assert 224.0 <= sw.max() <= 448.0, sw.max()
    act = oracle.quantize_act(X, p)
    sx = oracle.e4m3_to_f32(act["scales"]).astype(np.float64)
    assert 224.0 <= sx.max() <= 448.0, sx.max()


def test_pow2_scale():
    assert oracle.pow2_scale(2688.0) == 1.0
    assert oracle.pow2_scale(2688.0 * 1.0001) == 2.0
    assert oracle.pow2_scale(0.0) == 1.0
    assert oracle.pow2_scale(1.0) == 2.0**-11


# ----------------------------------------------------------------------------- W4A4 product
def _unpack_int4(codes):
    q = np.empty((codes.shape[0], 2 * codes.shape[1]), np.int64)
    q[:, 0::2], q[:, 1::2] = codes & 0xF, codes >> 4
    q[q >= 8] -= 16
    return q


def test_int4_group_acc_equals_matmul():
    rng = np.random.default_rng(7)
    M, N, K = 24, 40, 256
    xc = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    wc = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    acc = oracle.int4_group_acc(xc, wc)
    qx, qw = _unpack_int4(xc), _unpack_int4(wc)
    for g in range(K // 64):
        assert np.array_equal(acc[g], qx[:, g * 64:(g + 1) * 64] @ qw[:, g * 64:(g + 1) * 64].T)


def test_int4_subnormal_scales_saturate_codes():
    """Groups whose amax / 7 lies among the fp16 subnormals: the scale rounds down
    to 2^-24, so |v| / S reaches 7.35-10.15 and the codes must saturate.  Every
    code is the member of [-8, 7] nearest to fl32(v * fl32(1/S)) (brute force
    over all 16 codes, ties to the even code)."""
    rng = np.random.default_rng(8)
    rows, K = 6, 256
    v = np.empty((rows, K), np.float32)
    for r in range(rows):
        for g in range(K // 64):
            amax = 7.0 * rng.uniform(1.05, 1.45) * 2.0**-24  # amax / 7 rounds down to 2^-24 in fp16
            x = rng.uniform(-1.0, 1.0, 64) * amax
            x[0], x[1] = amax, -amax
            v[r, g * 64:(g + 1) * 64] = x
    codes, scales = oracle.quant_int4(v)
    S = oracle.f16_to_f32(scales).astype(np.float64)
    assert np.all(S == 2.0**-24)
    q = _unpack_int4(codes)
    inv = np.float32(1.0) / np.float32(2.0**-24)
    p = (v * inv).astype(np.float64)
    assert (p > 7.5).any() and (p < -8.5).any()  # both ends of the code range are exercised
    cand = np.arange(-8, 8)
    for pv, qv in zip(p.ravel(), q.ravel()):
        d = np.abs(pv - cand)
        best = cand[d == d.min()]
        if best.size > 1:
            best = best[best % 2 == 0]
        assert qv == best[0], (pv, qv)
    assert (q == 7).any() and (q == -8).any()


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_forward_equals_dequantized_matmul(fmt):
    layer = wl.small_layer(40, 256, 96, 16, fmt)
    X, W, b = wl.make_layer_inputs(layer)
    p = oracle.prepare(W, b, oracle.calib_absmax(X), 0.5, 16, fmt)
    act = oracle.quantize_act(X, p)
    y, yd = oracle.forward_from_act(act, p, want_f64=True)
    g_x, g_w = p["g_x"], p["g_w"]
    dqx = oracle.dequant(act["codes"], act["scales"], fmt, g_x)
    dqw = oracle.dequant(p["wcodes"], p["wscales"], fmt, g_w)
    ref = dqx @ dqw.T + _bf(act["t"]) @ _bf(p["L2"]) + _bf(p["bias"])[None, :]
    assert np.max(np.abs(yd - ref)) <= 1e-12 * np.max(np.abs(ref))
    assert np.array_equal(y, oracle.f64_to_bf16(yd))


def test_lowrank_down_matches_matmul():
    layer = wl.small_layer(32, 512, 64, 32, "nvfp4")
    X, W, b = wl.make_layer_inputs(layer)
    p = oracle.prepare(W, b, oracle.calib_absmax(X), 0.5, 32, "nvfp4")
    xhat = oracle.smooth_act(X, p["inv_lambda"])
    t = oracle.lowrank_down(xhat, p["L1"])
    ref = oracle.f64_to_bf16(_bf(oracle.f32_to_bf16(xhat)) @ _bf(p["L1"]))
    assert np.array_equal(t, ref)


def test_lowrank_down_rounds_once():
    """t is the binary64 sum rounded once to bf16: 1 + 2^-8 + 2^-30 lies above the bf16
    tie at 1 + 2^-8 and rounds up, where a detour through binary32 would land on the tie
    and round to 1.  The tie itself rounds to the even neighbour, 1."""
    xhat = np.array([[1.0, 2.0**-8, 2.0**-30], [1.0, 2.0**-8, 0.0]], np.float32)
    L1 = oracle.f64_to_bf16(np.ones((3, 1)))
    t = oracle.lowrank_down(xhat, L1)
    assert t[0, 0] == 0x3F81 and t[1, 0] == 0x3F80


def test_output_rounds_once_from_binary64():
    """y is formed in binary64 and rounded once to bf16: with zero codes (main term 0),
    t = (1, 2^-8, 2^-30), L2 = 1 and no bias, y = 1 + 2^-8 + 2^-30 exactly, which rounds
    up to 0x3F81 (a binary32 detour would give the tie and 0x3F80)."""
    K, N, r = 64, 1, 3
    prep = dict(N=N, K=K, rank=r, fmt=oracle.INT4, g_x=1.0, g_w=1.0,
                wcodes=np.zeros((N, K // 2), np.uint8), wscales=np.zeros((N, 1), np.uint16),
                L2=oracle.f64_to_bf16(np.ones((r, N))), bias=np.zeros(N, np.uint16))
    act = dict(codes=np.zeros((1, K // 2), np.uint8), scales=np.zeros((1, 1), np.uint16),
               t=oracle.f64_to_bf16(np.array([[1.0, 2.0**-8, 2.0**-30]])), g_x=1.0)
    y, yd = oracle.forward_from_act(act, prep, want_f64=True)
    assert yd[0, 0] == 1.0 + 2.0**-8 + 2.0**-30
    assert y[0, 0] == 0x3F81


# ----------------------------------------------------------------------------- method invariants
def _layer_err(X, W, b, rank, fmt, alpha=0.5):
    p = oracle.prepare(W, b, oracle.calib_absmax(X), alpha, rank, fmt)
    y = _bf(oracle.forward(X, p))
    ref = _bf(X) @ _bf(W).T + _bf(b)[None, :]
    return np.linalg.norm(y - ref) / np.linalg.norm(ref)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_error_decreases_with_rank_and_full_rank_is_near_exact(fmt):
    layer = wl.small_layer(64, 128, 128, 0, fmt)
    X, W, b = wl.make_layer_inputs(layer)
    errs = [_layer_err(X, W, b, r, fmt) for r in (0, 32, 64, 128)]
    assert all(errs[i + 1] < errs[i] for i in range(3)), errs
    assert errs[-1] < 0.02, errs  # only bf16 roundings of x^, t, L1, L2 remain


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_svdquant_beats_plain_w4a4_on_outliers(fmt):
    layer = wl.small_layer(128, 256, 256, 32, fmt, outlier_frac=0.02, outlier_scale=40.0)
    X, W, b = wl.make_layer_inputs(layer)
    plain = _layer_err(X, W, b, 0, fmt, alpha=0.0)  # alpha=0 -> lambda = 1/amax_w only
    svdq = _layer_err(X, W, b, 32, fmt, alpha=0.5)
    assert svdq < 0.5 * plain, (svdq, plain)


def test_workload_generator_is_deterministic_and_shaped():
    layer = wl.WORKLOADS["c1_int4_128x1024x1024_r32"][0]
    X1, W1, b1 = wl.make_layer_inputs(layer)
    X2, W2, b2 = wl.make_layer_inputs(layer)
    assert np.array_equal(X1, X2) and np.array_equal(W1, W2) and np.array_equal(b1, b2)
    assert layer.n_outliers == 10
    ch = wl.outlier_channels(layer)
    amax = np.abs(oracle.bf16_to_f32(X1)).max(axis=0)
    assert np.all(amax[ch] > 30) and np.median(amax) < 5
    assert abs(oracle.bf16_to_f32(W1).std() - 0.02) < 0.001
