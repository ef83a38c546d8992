"""CPU checks of the C-ABI library: it loads, exports every declared symbol,
computes sizes and layouts, and its host-side prepare/pack agree with the oracle
and the format definitions.  No kernel runs here."""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

import diffusion_transformer_w4a4_b200 as svdq
import oracle
import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svdq.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from diffusion_transformer_w4a4_b200 import build

    build.build()
    return svdq.lib()


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", svdq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (svdq_[a-z0-9_]+)", out))
    assert set(names) <= exported
    # the binding mirrors the C names
    for n in names:
        assert hasattr(svdq, n), n


def test_status_strings(lib):
    assert svdq.svdq_status_string(0) == "SVDQ_OK"
    assert "sm_100a" in svdq.svdq_status_string(svdq.SVDQ_ERR_UNSUPPORTED_DEVICE)
    assert svdq.svdq_status_string(99).startswith("SVDQ_ERR")
    assert svdq.svdq_abi_version() == 2


def test_shape_validation(lib):
    assert svdq.svdq_packed_size(1024, 1024, 32, "int4") > 0
    for bad in [(1024, 1000, 32, "int4"), (1000, 1024, 32, "nvfp4"), (1024, 1024, 24, "int4"),
                (1024, 1024, 144, "nvfp4"), (1024, 1024, 32, 7), (16, 256, 32, "int4")]:
        with pytest.raises(svdq.SvdqError) as e:
            svdq.svdq_packed_size(*bad)
        assert e.value.status == svdq.SVDQ_ERR_INVALID_ARG


def test_canonical_sizes(lib):
    s = svdq.svdq_canonical_sizes(384, 512, 32, "nvfp4")
    assert s == [512 * 4, 512 * 4, 512 * 32 * 2, 32 * 384 * 2, 384 * 256, 384 * 32, 384 * 2]
    s = svdq.svdq_canonical_sizes(384, 512, 32, "int4")
    assert s[5] == 384 * 8 * 2


def test_device_check_without_gpu(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is visible")
    assert svdq.svdq_device_check(0) == svdq.SVDQ_ERR_UNSUPPORTED_DEVICE


def _run_env(code: str, **env):
    e = dict(os.environ, **env)
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=e, cwd=ROOT)


def test_fault_injection_env():
    code = ("import numpy as np, diffusion_transformer_w4a4_b200 as s\n"
            "W=np.zeros((32,256),np.uint16)\n"
            "try:\n s.svdq_prepare(W,None,np.ones(256,np.float32),0.5,16,'int4'); print('OK')\n"
            "except s.SvdqError as e: print('ERR', e.status)\n"
            "print('DEV', s.svdq_device_check(0))\n")
    r = _run_env(code, SVDQ_FAULT="alloc")
    assert "ERR 3" in r.stdout, r.stderr
    r = _run_env(code, SVDQ_FAULT="nan_input")
    assert "ERR 5" in r.stdout, r.stderr
    r = _run_env(code, SVDQ_FAULT="bad_arch")
    assert "DEV 2" in r.stdout, r.stderr


def test_prepare_rejects_non_finite(lib):
    W = np.zeros((32, 256), np.uint16)
    W[3, 5] = 0x7FC0  # NaN
    with pytest.raises(svdq.SvdqError) as e:
        svdq.svdq_prepare(W, None, np.ones(256, np.float32), 0.5, 16, "int4")
    assert e.value.status == svdq.SVDQ_ERR_NUMERIC
    with pytest.raises(svdq.SvdqError):
        svdq.svdq_prepare(np.zeros((32, 256), np.uint16), None, np.full(256, np.inf, np.float32), 0.5, 16, "int4")


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_product_prepare_agrees_with_oracle(lib, fmt):
    layer = wl.small_layer(256, 512, 384, 32, fmt)
    X, W, b = wl.make_layer_inputs(layer)
    amax = oracle.calib_absmax(X)
    ours = svdq.svdq_prepare(W, b, amax, 0.5, 32, fmt)
    ref = oracle.prepare(W, b, amax, 0.5, 32, fmt)
    # smoothing factors: same formula, within one binary32 ulp
    assert np.all(np.abs(ours["lambda_"] - ref["lam"]) <= np.spacing(ref["lam"]))
    assert np.all(np.abs(ours["inv_lambda"] - ref["inv_lambda"]) <= np.spacing(ref["inv_lambda"]))
    # rank-32 branch.  The synthetic weights have a few outlier-driven singular
    # values above a flat random-matrix bulk, so the bulk part of a rank-32
    # subspace is not determined to 1e-3 by any SVD.  Gate on what is fixed:
    # near-optimal truncation (Eckart-Young, from the oracle's spectrum) and
    # agreement on the gap-separated leading directions.
    bf = lambda h: oracle.bf16_to_f32(h).astype(np.float64)
    P1 = bf(ours["L1"]) @ bf(ours["L2"])
    What = bf(W) * ref["lam"].astype(np.float64)[None, :]
    S = ref["sing"]
    assert np.linalg.norm(What - P1.T) ** 2 <= np.sum(S[32:] ** 2) * 1.005
    k = int(np.sum(S > 1.5 * S[32]))
    assert k >= 3
    U, s_, Vt = np.linalg.svd(What, full_matrices=False)
    Pk = (U[:, :k] * s_[:k]) @ Vt[:k]
    proj = U[:, :k] @ U[:, :k].T
    assert np.linalg.norm(proj @ P1.T - Pk) / np.linalg.norm(Pk) <= 5e-3
    # the residual differs with the bulk subspace, so compare what the layer
    # reconstructs: branch + dequantized residual vs the smoothed weight
    assert ours["g_x"] == ref["g_x"]
    def recon_err(c):
        dq = oracle.dequant(c["wcodes"], c["wscales"], fmt, c["g_w"])
        return np.linalg.norm(What - (bf(c["L1"]) @ bf(c["L2"])).T - dq) / np.linalg.norm(What)
    e_ours, e_ref = recon_err(ours), recon_err(ref)
    assert e_ours <= 1.05 * e_ref, (e_ours, e_ref)
    np.testing.assert_array_equal(ours["bias"], b)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_product_prepare_degenerate_inputs(lib, fmt):
    """A zero weight channel and a zero activation channel get lambda = 1; an all-zero
    weight gives a zero branch, zero codes and scales and g_w = 1 (nothing non-finite);
    at full rank the branch reconstructs the smoothed weight as well as the oracle's."""
    bf = lambda h: oracle.bf16_to_f32(h).astype(np.float64)
    X, W, b = wl.make_layer_inputs(wl.small_layer(64, 256, 128, 16, fmt))
    W = W.copy()
    W[:, 7] = 0
    amax = oracle.calib_absmax(X).copy()
    amax[11] = 0.0
    ours = svdq.svdq_prepare(W, b, amax, 0.5, 16, fmt)
    assert ours["lambda_"][7] == 1.0 and ours["lambda_"][11] == 1.0
    assert ours["inv_lambda"][7] == 1.0 and ours["inv_lambda"][11] == 1.0
    zero = svdq.svdq_prepare(np.zeros_like(W), None, amax, 0.5, 16, fmt)
    assert np.isfinite(bf(zero["L1"])).all() and np.isfinite(bf(zero["L2"])).all()
    assert not (bf(zero["L1"]) @ bf(zero["L2"])).any()
    assert not zero["wcodes"].any() and not np.asarray(zero["wscales"]).any()
    assert zero["g_w"] == 1.0
    X, W, b = wl.make_layer_inputs(wl.small_layer(64, 256, 128, 128, fmt))
    amax = oracle.calib_absmax(X)
    full = svdq.svdq_prepare(W, b, amax, 0.5, 128, fmt)
    ref = oracle.prepare(W, b, amax, 0.5, 128, fmt)
    What = bf(W) * ref["lam"].astype(np.float64)[None, :]
    err = lambda c: np.linalg.norm(What - (bf(c["L1"]) @ bf(c["L2"])).T) / np.linalg.norm(What)
    assert err(full) <= 1.01 * err(ref) + 1e-12 and err(ref) < 0.01


def test_product_svd_on_adversarial_spectra(lib):
    """The product's truncated SVD (randomized subspace iteration) on the two spectra
    that are hardest for it: a weight of exact rank 8 at r = 16 must be reconstructed
    as well as by the oracle's full SVD (only bf16 rounding of the factors remains),
    and a flat spectrum (no gap, slowest convergence) must still come within 1 % of
    the Eckart-Young optimum."""
    bf = lambda h: oracle.bf16_to_f32(h).astype(np.float64)
    rng = np.random.default_rng(0)
    N, K = 192, 256
    amax = (np.abs(rng.standard_normal(K)) + 0.5).astype(np.float32)
    W = wl.f32_to_bf16_bits((rng.standard_normal((N, 8)) @ rng.standard_normal((8, K)) * 0.01).astype(np.float32))
    ours = svdq.svdq_prepare(W, None, amax, 0.5, 16, "int4")
    ref = oracle.prepare(W, None, amax, 0.5, 16, "int4")
    What = bf(W) * ref["lam"].astype(np.float64)[None, :]
    err = lambda c: np.linalg.norm(What - (bf(c["L1"]) @ bf(c["L2"])).T) / np.linalg.norm(What)
    assert err(ours) <= 1.01 * err(ref) and err(ref) < 0.01
    Q1, _ = np.linalg.qr(rng.standard_normal((N, N)))
    Q2, _ = np.linalg.qr(rng.standard_normal((K, K)))
    W = wl.f32_to_bf16_bits((Q1 @ np.diag(np.linspace(1.0, 0.98, N)) @ Q2[:, :N].T * 0.05).astype(np.float32))
    ours = svdq.svdq_prepare(W, None, amax, 0.5, 32, "int4")
    ref = oracle.prepare(W, None, amax, 0.5, 32, "int4")
    What = bf(W) * ref["lam"].astype(np.float64)[None, :]
    trunc = np.linalg.norm(What - (bf(ours["L1"]) @ bf(ours["L2"])).T) ** 2
    assert trunc <= 1.01 * np.sum(ref["sing"][32:] ** 2)


def test_product_codecs_match_oracle_via_prepare_rank0(lib):
    # rank 0 and alpha 0: the residual is W * lambda exactly, so the weight codes
    # and scales come from identical binary32 inputs on both sides and must be
    # bit-identical (quantizer parity of the host code).
    for fmt in ("int4", "nvfp4"):
        layer = wl.small_layer(64, 512, 256, 0, fmt)
        X, W, b = wl.make_layer_inputs(layer)
        amax = oracle.calib_absmax(X)
        ours = svdq.svdq_prepare(W, b, amax, 0.0, 0, fmt)
        ref = oracle.prepare(W, b, amax, 0.0, 0, fmt)
        np.testing.assert_array_equal(ours["wcodes"], ref["wcodes"])
        np.testing.assert_array_equal(ours["wscales"], ref["wscales"])


def _sf_offset(row, block, katoms, tile_rows):
    tile, rin = row // tile_rows, row % tile_rows
    apt = (tile_rows + 127) // 128
    a, ra = rin // 128, rin % 128
    return ((tile * katoms + block // 4) * apt + a) * 512 + (ra % 32) * 16 + ((ra // 32) % 4) * 4 + block % 4


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_pack_layout(lib, fmt):
    N, K, r = 400, 512, 48
    rng = np.random.default_rng(0)
    c = svdq._canonical_arrays(N, K, r, fmt)
    c["inv_lambda"][:] = rng.uniform(0.5, 2, K)
    c["L1"][:] = oracle.f32_to_bf16(rng.standard_normal((K, r)).astype(np.float32))
    c["L2"][:] = oracle.f32_to_bf16(rng.standard_normal((r, N)).astype(np.float32))
    c["wcodes"][:] = rng.integers(0, 256, c["wcodes"].shape)
    c["wscales"][:] = rng.integers(0, 0x7E if fmt == "nvfp4" else 0x7BFF, c["wscales"].shape)
    c["bias"][:] = oracle.f32_to_bf16(rng.standard_normal(N).astype(np.float32))
    c["g_x"], c["g_w"] = 2.0**-4, 2.0**-13
    blob = svdq.svdq_pack(c)
    # region offsets, 1024-aligned, in the documented order
    o = 0
    def take(nbytes):
        nonlocal o
        start = o
        o = (o + nbytes + 1023) // 1024 * 1024
        return start
    wc_bytes = N * K if fmt == "int4" else N * K // 2
    o_il, o_l1, o_l2, o_b, o_wc = take(K * 4), take(r * K * 2), take(N * r * 2), take(N * 4), take(wc_bytes)
    o_ws = o
    assert blob.size == (o + (N * K // 64 * 4 if fmt == "int4" else (N + 191) // 192 * (K // 64) * 1024) + 1023) // 1024 * 1024
    assert np.array_equal(blob[o_il:o_il + 4 * K].view(np.float32), c["inv_lambda"])
    assert np.array_equal(blob[o_l1:o_l1 + 2 * r * K].view(np.uint16).reshape(r, K), c["L1"].T)
    l2t = oracle.bf16_to_f32(blob[o_l2:o_l2 + 2 * N * r].view(np.uint16).reshape(N, r)).astype(np.float64)
    scale = 1.0 / (c["g_x"] * c["g_w"]) if fmt == "nvfp4" else 1.0
    assert np.array_equal(l2t, oracle.bf16_to_f32(c["L2"]).T.astype(np.float64) * scale)
    assert np.array_equal(blob[o_b:o_b + 4 * N].view(np.float32), oracle.bf16_to_f32(c["bias"]))
    if fmt == "int4":
        # one E4M3 byte per code, holding the code's integer value exactly
        wb = blob[o_wc:o_wc + N * K].reshape(N, K)
        nib = np.stack([c["wcodes"] & 15, c["wcodes"] >> 4], axis=-1).reshape(N, K).astype(np.int64)
        vals = np.where(nib >= 8, nib - 16, nib).astype(np.float32)
        assert np.array_equal(wb, oracle.f32_to_e4m3(vals.reshape(-1)).reshape(N, K))
    else:
        assert np.array_equal(blob[o_wc:o_wc + N * K // 2].reshape(N, K // 2), c["wcodes"])
    if fmt == "int4":
        ws = blob[o_ws:o_ws + N * K // 64 * 4].view(np.float32).reshape(K // 64, N)
        assert np.array_equal(ws, c["wscales"].T.view(np.float16).astype(np.float32))
    else:
        rows, blocks = np.meshgrid(np.arange(N), np.arange(K // 16), indexing="ij")
        offs = _sf_offset(rows, blocks, K // 64, 192)
        assert np.array_equal(blob[o_ws + offs], c["wscales"])
        # padding rows of the last 192-row tile stay zero
        used = np.zeros(blob.size - o_ws, bool)
        used[offs.ravel()] = True
        assert np.all(blob[o_ws:][~used] == 0)


def test_pack_dynamic_activation_scale_folds_only_the_weight_scale(lib):
    """g_x = 0 selects the per-call activation scale: the packed L2 carries
    1/g_w only (the quantizer stores t / g_x), everything else is unchanged."""
    N, K, r = 208, 256, 16
    rng = np.random.default_rng(4)
    c = svdq._canonical_arrays(N, K, r, "nvfp4")
    c["inv_lambda"][:] = rng.uniform(0.5, 2, K)
    c["L1"][:] = oracle.f32_to_bf16(rng.standard_normal((K, r)).astype(np.float32))
    c["L2"][:] = oracle.f32_to_bf16(rng.standard_normal((r, N)).astype(np.float32))
    c["wcodes"][:] = rng.integers(0, 256, c["wcodes"].shape)
    c["wscales"][:] = rng.integers(0, 0x7E, c["wscales"].shape)
    c["g_x"], c["g_w"] = 0.0, 2.0**-11
    dyn = svdq.svdq_pack(c)
    c["g_x"] = 1.0
    st = svdq.svdq_pack(c)
    assert np.array_equal(dyn, st)  # with g_x = 1 the static fold is the same 1/g_w
    c["g_x"] = 2.0**-3
    st3 = svdq.svdq_pack(c)
    l2_off = (K * 4 + 1023) // 1024 * 1024 + (r * K * 2 + 1023) // 1024 * 1024
    l2d = oracle.bf16_to_f32(dyn[l2_off:l2_off + 2 * N * r].view(np.uint16))
    l23 = oracle.bf16_to_f32(st3[l2_off:l2_off + 2 * N * r].view(np.uint16))
    assert np.array_equal(l23, l2d * np.float32(8.0))
    c["g_x"] = -1.0
    with pytest.raises(svdq.SvdqError):
        svdq.svdq_pack(c)


def test_pack_rejects_non_power_of_two_scales(lib):
    c = svdq._canonical_arrays(32, 256, 16, "nvfp4")
    c["g_x"], c["g_w"] = 0.3, 1.0
    with pytest.raises(svdq.SvdqError):
        svdq.svdq_pack(c)


# ----------------------------------------------------------------------------- awq_w4a16
def test_awq_shape_validation(lib):
    assert svdq.svdq_awq_packed_size(18432, 3072) > 0
    for bad in [(16, 100), (0, 64), (16, 32), (16, 12288 + 64)]:
        with pytest.raises(svdq.SvdqError) as e:
            svdq.svdq_awq_packed_size(*bad)
        assert e.value.status == svdq.SVDQ_ERR_INVALID_ARG


def test_awq_prepare_rejects_non_finite(lib):
    W = np.zeros((16, 64), np.uint16)
    X = np.zeros((2, 64), np.uint16)
    X[1, 3] = 0x7FC0  # bf16 NaN
    with pytest.raises(svdq.SvdqError) as e:
        svdq.svdq_awq_prepare(W, None, X)
    assert e.value.status == svdq.SVDQ_ERR_NUMERIC


@pytest.mark.parametrize("shape", [(2, 256, 48), (64, 512, 96)])
def test_awq_product_prepare_agrees_with_oracle(lib, shape):
    """The library's activation-aware preparation picks the oracle's alpha (or
    one whose error ties it to 1e-9 relative) and then the same codes and scales
    (its error sums run in another order; the scales use the same pow)."""
    M, K, N = shape
    rng = np.random.default_rng(11)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.choice(K, 3, replace=False)] *= 50.0
    X = wl.f32_to_bf16_bits(x)
    W = wl.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    b = wl.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32) * 0.01)
    ours = svdq.svdq_awq_prepare(W, b, X)
    ref = oracle.awq_prepare(W, b, X)
    if np.float32(ours["alpha"]) != np.float32(ref["alpha"]):  # the ABI stores alpha as binary32
        a = min(oracle.AWQ_ALPHAS, key=lambda g: abs(g - ours["alpha"]))
        e_ours = oracle.awq_output_error(X, W, oracle.awq_mean_abs(X), a)
        assert abs(e_ours - ref["err"]) <= 1e-9 * ref["err"], (ours["alpha"], ref["alpha"])
        ref = dict(ref)
        _, ref["s"], ref["inv_s"] = oracle.awq_channel_scales(oracle.awq_mean_abs(X), a)
        ref["wcodes"], ref["wscales"] = oracle.awq_quant_weights(W, ref["s"])
    np.testing.assert_array_equal(ours["s"], ref["s"])
    np.testing.assert_array_equal(ours["inv_s"], ref["inv_s"])
    np.testing.assert_array_equal(ours["wcodes"], ref["wcodes"])
    np.testing.assert_array_equal(ours["wscales"], ref["wscales"])
    np.testing.assert_array_equal(ours["bias"], b)


@pytest.mark.parametrize("K", [192, 256])
def test_awq_pack_layout(lib, K):
    N = 40
    rng = np.random.default_rng(12)
    c = svdq._awq_arrays(N, K)
    c["inv_s"][:] = rng.uniform(0.5, 2, K)
    c["s"][:] = 1.0 / c["inv_s"]
    c["wcodes"][:] = rng.integers(0, 256, c["wcodes"].shape)
    c["wscales"][:] = rng.integers(0, 0x7BFF, c["wscales"].shape)
    c["bias"][:] = oracle.f32_to_bf16(rng.standard_normal(N).astype(np.float32))
    blob = svdq.svdq_awq_pack(c)
    o = 0
    def take(nbytes):
        nonlocal o
        start = o
        o = (o + nbytes + 1023) // 1024 * 1024
        return start
    G = K // 64
    ld = (G + 7) // 8 * 8  # scale rows padded to a multiple of 8 entries
    o_is, o_b, o_ws, o_wc, o_st = take(K * 4), take(N * 4), take(N * ld * 2), take(N * K // 2), take(16)
    assert blob.size == o
    assert np.all(blob[o_st:] == 0)
    assert np.array_equal(blob[o_is:o_is + 4 * K].view(np.float32), c["inv_s"])
    assert np.array_equal(blob[o_b:o_b + 4 * N].view(np.float32), oracle.bf16_to_f32(c["bias"]))
    ws = blob[o_ws:o_ws + N * ld * 2].view(np.uint16).reshape(N, ld)
    assert np.array_equal(ws[:, :G], c["wscales"])
    assert np.all(ws[:, G:] == 0)
    assert np.array_equal(blob[o_wc:o_wc + N * K // 2].reshape(N, K // 2), c["wcodes"] ^ 0x88)  # offset binary nibbles


# ----------------------------------------------------------------------------- int8 tensorwise W8A8
def test_w8a8_shape_validation(lib):
    assert svdq.svdq_w8a8_packed_size(3072, 12288) > 0
    for bad in [(12, 128), (0, 128), (16, 64), (16, 200)]:
        with pytest.raises(svdq.SvdqError):
            svdq.svdq_w8a8_packed_size(*bad)


@pytest.mark.parametrize("shape", [(24, 128), (200, 384)])
def test_w8a8_product_prepare_agrees_with_oracle(lib, shape):
    N, K = shape
    rng = np.random.default_rng(31)
    w = rng.standard_normal((N, K)).astype(np.float32) * 0.02
    w[3, 5] = 0.5  # a large entry sets the scale
    W = wl.f32_to_bf16_bits(w)
    codes, s_w = svdq.svdq_w8a8_prepare(W)
    ref = oracle.w8a8_prepare(W)
    assert np.float32(s_w) == ref["s_w"]
    np.testing.assert_array_equal(codes, ref["wcodes"])


def test_w8a8_prepare_rejects_non_finite(lib):
    W = wl.f32_to_bf16_bits(np.ones((8, 128), np.float32))
    W[2, 3] = 0x7F80  # +inf
    with pytest.raises(svdq.SvdqError):
        svdq.svdq_w8a8_prepare(W)


def test_w8a8_pack_layout(lib):
    N, K = 40, 256
    rng = np.random.default_rng(32)
    codes = rng.integers(-127, 128, (N, K)).astype(np.int8)
    b = oracle.f32_to_bf16(rng.standard_normal(N).astype(np.float32))
    blob = svdq.svdq_w8a8_pack(codes, b)
    o_wc = (N * 4 + 1023) // 1024 * 1024
    assert blob.size == (o_wc + N * K + 1023) // 1024 * 1024
    assert np.array_equal(blob[:4 * N].view(np.float32), oracle.bf16_to_f32(b))
    assert np.array_equal(blob[o_wc:o_wc + N * K].view(np.int8).reshape(N, K), codes)
    assert np.all(svdq.svdq_w8a8_pack(codes)[:4 * N] == 0)  # no bias: zeros
