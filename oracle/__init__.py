"""Oracle for the svdq_w4a4 linear layer: plain, slow, obviously correct CPU code.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import this package.  It shares no code with the
CUDA library in diffusion_transformer_w4a4_b200/ and never imports it.

The per-element arithmetic (number codecs, quantizers, the W4A4 product, the
output) lives in svdq_oracle.c (binary64 unless the method fixes binary32);
this file adds the host-side preparation, where numpy's LAPACK SVD in binary64
serves as the SVD step, and thin ctypes marshalling.

Method source: "Hugging Face встроила Nunchaku в Diffusers ..." (iitog.ru),
paragraph "Суть метода" (smoothing, 16-bit low-rank branch from the weight,
4-bit residual, W4A4), and the paragraph after it (svdq_w4a4 in INT4 and NVFP4
variants); "SVDQuant ускоряет Krea 2 вдвое ..." (ainews.so), section
"Решение: INT8 и W4A4" (no calibration dataset; low-rank branches compensate).
Beyond the svdq_w4a4 layer: the awq_w4a16 runtime layer the same iitog.ru page
names for normalization / modulation layers (awq_*), the per-call (dynamic)
per-tensor NVFP4 activation scale (act_tensor_scale, selected by g_x = 0), and
the INT8 tensorwise W8A8 layer the ainews.so section compares (w8a8_*), each
pinned in its own tests/test_oracle_*.py, and the GELU between a block's MLP
linears (gelu_bf16, for the fused MLP pair; pinned in test_oracle_gelu.py).

The pins themselves are tested: tests/test_oracle_mutants.py plants plausible
mistakes in copies of this oracle (compile_source / bind load a mutated copy of
svdq_oracle.c; single Python steps are replaced) and requires a pin to catch each.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svdq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

INT4, NVFP4 = 1, 2
_FMT = {"int4": INT4, "nvfp4": NVFP4, INT4: INT4, NVFP4: NVFP4}
E4M3_MAX = 448.0
E2M1_MAX = 6.0


def compile_source(src: str, out: str) -> None:
    """gcc with the flags the oracle's arithmetic relies on (no fused
    multiply-add, no fast-math)."""
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                           "-shared", "-fPIC", "-o", out, src, "-lm"])


def build(force: bool = False) -> str:
    """Compile svdq_oracle.c into liboracle.so when it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        compile_source(_SRC, tmp)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = bind(ctypes.CDLL(build()))
    return _lib


def bind(L):
    """Declare the C signatures on a loaded copy of the oracle library."""
    i64, f32, f64, vp, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
    L.orc_f64_to_bf16.restype = ctypes.c_uint16
    L.orc_f64_to_bf16.argtypes = [f64]
    L.orc_f32_to_bf16.restype = ctypes.c_uint16
    L.orc_f32_to_bf16.argtypes = [f32]
    L.orc_f32_to_f16.restype = ctypes.c_uint16
    L.orc_f32_to_f16.argtypes = [f32]
    L.orc_f32_to_e4m3_satfinite.restype = ctypes.c_uint8
    L.orc_f32_to_e4m3_satfinite.argtypes = [f32]
    L.orc_f32_to_e2m1_satfinite.restype = ctypes.c_uint8
    L.orc_f32_to_e2m1_satfinite.argtypes = [f32]
    for name in ("orc_vec_f64_to_bf16", "orc_vec_f32_to_bf16", "orc_vec_f32_to_f16", "orc_vec_f16_to_f32",
                 "orc_vec_f32_to_e4m3", "orc_vec_e4m3_to_f32", "orc_vec_f32_to_e2m1", "orc_vec_e2m1_to_f32"):
        getattr(L, name).argtypes = [i64, vp, vp]
        getattr(L, name).restype = None
    L.orc_smooth_factors.argtypes = [i64, vp, vp, f64, vp, vp, vp]
    L.orc_smooth_act.argtypes = [i64, i64, vp, vp, vp]
    L.orc_quant_int4_rows.argtypes = [i64, i64, vp, vp, vp]
    L.orc_quant_nvfp4_rows.argtypes = [i64, i64, vp, f32, vp, vp]
    L.orc_dequant_int4_rows.argtypes = [i64, i64, vp, vp, vp]
    L.orc_dequant_nvfp4_rows.argtypes = [i64, i64, vp, vp, f32, vp]
    L.orc_lowrank_down.argtypes = [i64, i64, i64, vp, vp, vp]
    L.orc_int4_group_acc.argtypes = [i64, i64, i64, vp, vp, vp]
    L.orc_forward_out.argtypes = [i64, i64, i64, i64, i32, vp, vp, vp, vp, f32, f32, vp, vp, vp, vp, vp]
    L.orc_num_threads.restype = i32
    return L


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ----------------------------------------------------------------------------- codecs
def _vec(fn, x, in_dtype, out_dtype):
    x = np.ascontiguousarray(x, dtype=in_dtype)
    out = np.empty(x.shape, dtype=out_dtype)
    getattr(lib(), fn)(x.size, _p(x), _p(out))
    return out


def f64_to_bf16(x): return _vec("orc_vec_f64_to_bf16", x, np.float64, np.uint16)
def f32_to_bf16(x): return _vec("orc_vec_f32_to_bf16", x, np.float32, np.uint16)
def f32_to_f16(x): return _vec("orc_vec_f32_to_f16", x, np.float32, np.uint16)
def f16_to_f32(x): return _vec("orc_vec_f16_to_f32", x, np.uint16, np.float32)
def f32_to_e4m3(x): return _vec("orc_vec_f32_to_e4m3", x, np.float32, np.uint8)
def e4m3_to_f32(x): return _vec("orc_vec_e4m3_to_f32", x, np.uint8, np.float32)
def f32_to_e2m1(x): return _vec("orc_vec_f32_to_e2m1", x, np.float32, np.uint8)
def e2m1_to_f32(x): return _vec("orc_vec_e2m1_to_f32", x, np.uint8, np.float32)


def bf16_to_f32(h):
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------- GELU
def gelu_f64(h: np.ndarray) -> np.ndarray:
    """GELU in its erf form, h Phi(h) = h/2 (1 + erf(h / sqrt 2)), in binary64 (the
    activation between a diffusion transformer block's MLP linears).  Evaluated
    as h/2 erfc(-h / sqrt 2), the same value: 1 + erf(x) cancels to 0 in binary64
    once x < -5.9 or so, erfc keeps the tail."""
    from scipy.special import erfc

    h = np.asarray(h, np.float64)
    return 0.5 * h * erfc(-h / math.sqrt(2.0))


def gelu_bf16(h_bits: np.ndarray) -> np.ndarray:
    """bf16 bits -> bf16 bits of GELU(h), computed in binary64 and rounded once
    (round to nearest even)."""
    return f64_to_bf16(np.ascontiguousarray(gelu_f64(bf16_to_f32(h_bits))))


# ----------------------------------------------------------------------------- smoothing
def calib_absmax(X_bf16: np.ndarray) -> np.ndarray:
    """Calibration statistic: per input channel max |x| over the layer's own input
    (no calibration dataset -- "Решение: INT8 и W4A4")."""
    return np.abs(bf16_to_f32(X_bf16)).max(axis=0).astype(np.float32)


def smooth_factors(amax_x: np.ndarray, amax_w: np.ndarray, alpha: float):
    """lambda_j = amax_x[j]^alpha / amax_w[j]^(1-alpha) (1 if either is 0).
    Returns (lambda in binary64, lambda in binary32, 1/lambda in binary32)."""
    K = amax_x.size
    amax_x = np.ascontiguousarray(amax_x, np.float32)
    amax_w = np.ascontiguousarray(amax_w, np.float32)
    ld = np.empty(K, np.float64)
    lf = np.empty(K, np.float32)
    il = np.empty(K, np.float32)
    lib().orc_smooth_factors(K, _p(amax_x), _p(amax_w), float(alpha), _p(ld), _p(lf), _p(il))
    return ld, lf, il


def smooth_act(X_bf16: np.ndarray, inv_lambda: np.ndarray) -> np.ndarray:
    X = np.ascontiguousarray(X_bf16, np.uint16)
    M, K = X.shape
    out = np.empty((M, K), np.float32)
    lib().orc_smooth_act(M, K, _p(X), _p(np.ascontiguousarray(inv_lambda, np.float32)), _p(out))
    return out


# ----------------------------------------------------------------------------- quantizers
def quant_int4(v: np.ndarray):
    """INT4, groups of 64 along K: returns (codes [rows, K/2] u8, scales [rows, K/64] fp16 bits)."""
    v = np.ascontiguousarray(v, np.float32)
    rows, K = v.shape
    assert K % 64 == 0
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 64), np.uint16)
    lib().orc_quant_int4_rows(rows, K, _p(v), _p(codes), _p(scales))
    return codes, scales


def quant_nvfp4(v: np.ndarray, g: float):
    """NVFP4, blocks of 16 along K: returns (codes [rows, K/2] u8, scales [rows, K/16] E4M3 bits)."""
    v = np.ascontiguousarray(v, np.float32)
    rows, K = v.shape
    assert K % 16 == 0
    codes = np.empty((rows, K // 2), np.uint8)
    scales = np.empty((rows, K // 16), np.uint8)
    lib().orc_quant_nvfp4_rows(rows, K, _p(v), float(g), _p(codes), _p(scales))
    return codes, scales


def dequant(codes, scales, fmt, g=1.0):
    codes = np.ascontiguousarray(codes, np.uint8)
    rows, K2 = codes.shape
    out = np.empty((rows, 2 * K2), np.float64)
    if _FMT[fmt] == INT4:
        lib().orc_dequant_int4_rows(rows, 2 * K2, _p(codes), _p(np.ascontiguousarray(scales, np.uint16)), _p(out))
    else:
        lib().orc_dequant_nvfp4_rows(rows, 2 * K2, _p(codes), _p(np.ascontiguousarray(scales, np.uint8)), float(g), _p(out))
    return out


def pow2_scale(amax: float) -> float:
    """Per-tensor NVFP4 scale: the smallest power of two g with g >= amax / (6 * 448),
    i.e. the largest block scale amax_b/(6 g) stays <= 448 (E4M3 max) and
    every block value / (scale * g) stays <= 6 (E2M1 max).  1.0 for an all-zero tensor."""
    a = float(amax) / (E2M1_MAX * E4M3_MAX)
    if a <= 0.0:
        return 1.0
    m, e = math.frexp(a)  # a = m * 2^e, m in [0.5, 1)
    k = e - 1 if m == 0.5 else e
    return math.ldexp(1.0, k)


# ----------------------------------------------------------------------------- prepare
def svd_lowrank_factors(What: np.ndarray, rank: int):
    """Truncated SVD of the smoothed weight W^ [N, K] = U S V^T (binary64 LAPACK).
    L1 = V_r S_r^(1/2) [K, r], L2 = S_r^(1/2) U_r^T [r, N], so L1 L2 ~ W^T.
    Sign convention: the largest-magnitude entry of each column of U is positive.
    Returns (L1, L2, singular values) in binary64."""
    U, S, Vt = np.linalg.svd(What, full_matrices=False)
    r = int(rank)
    Ur, Sr, Vr = U[:, :r].copy(), S[:r], Vt[:r].T.copy()
    for j in range(r):
        i = int(np.argmax(np.abs(Ur[:, j])))
        if Ur[i, j] < 0:
            Ur[:, j] *= -1.0
            Vr[:, j] *= -1.0
    sq = np.sqrt(Sr)
    return Vr * sq[None, :], (Ur * sq[None, :]).T.copy(), S


def smoothed_weight(W_bf16: np.ndarray, amax_x: np.ndarray, alpha: float):
    """Steps 1-2 of prepare: lambda from the channel maxima and W^ = W * lambda
    (binary64 product of the binary32 lambda).  Returns (W^, (lambda_d, lambda_f,
    1/lambda_f))."""
    Wf = bf16_to_f32(np.ascontiguousarray(W_bf16, np.uint16))
    amax_w = np.abs(Wf).max(axis=0).astype(np.float32)
    lams = smooth_factors(amax_x, amax_w, alpha)
    return Wf.astype(np.float64) * lams[1].astype(np.float64)[None, :], lams


def prepare(W_bf16: np.ndarray, bias_bf16, amax_x: np.ndarray, alpha: float, rank: int, fmt, svd=None):
    """Offline preparation of one layer ("Суть метода"):
      1. lambda from the activation and weight channel maxima (smoothing),
      2. W^ = W * lambda,
      3. rank-r split of W^ by SVD into bf16 L1 [K, r] and L2 [r, N],
      4. residual R = W^ - (L1 L2)^T with the rounded factors, rounded to binary32,
      5. 4-bit group quantization of R (INT4 or NVFP4).
    `svd` may carry a precomputed (L1, L2, S) of the same W^ (same lambda), so
    that several ranks reuse one decomposition; it is truncated to `rank`."""
    fmt = _FMT[fmt]
    N, K = W_bf16.shape
    What, (lam_d, lam_f, inv_lam) = smoothed_weight(W_bf16, amax_x, alpha)
    r = int(rank)
    if r > 0:
        if svd is None:
            L1d, L2d, S = svd_lowrank_factors(What, r)
        else:
            L1d, L2d, S = svd[0][:, :r], svd[1][:r], svd[2]
        L1 = f64_to_bf16(np.ascontiguousarray(L1d))
        L2 = f64_to_bf16(np.ascontiguousarray(L2d))
        R = What - (bf16_to_f32(L1).astype(np.float64) @ bf16_to_f32(L2).astype(np.float64)).T
    else:
        L1 = np.zeros((K, 0), np.uint16)
        L2 = np.zeros((0, N), np.uint16)
        S = None
        R = What
    R32 = np.ascontiguousarray(R.astype(np.float32))
    out = dict(N=N, K=K, rank=r, fmt=fmt, alpha=float(alpha), lambda_d=lam_d, lam=lam_f, inv_lambda=inv_lam,
               L1=L1, L2=L2, sing=S, R=R32,
               bias=(np.zeros(N, np.uint16) if bias_bf16 is None else np.ascontiguousarray(bias_bf16, np.uint16)))
    if fmt == INT4:
        out["wcodes"], out["wscales"] = quant_int4(R32)
        out["g_w"] = 1.0
        out["g_x"] = 1.0
    else:
        g_w = pow2_scale(float(np.abs(R32).max()) if R32.size else 0.0)
        out["wcodes"], out["wscales"] = quant_nvfp4(R32, g_w)
        out["g_w"] = g_w
        # Static activation scale from the calibration statistic: max over channels of
        # the largest smoothed activation, |x^| = float(amax_x * inv_lambda).
        xhat_max = float((np.asarray(amax_x, np.float32) * inv_lam).max()) if K else 0.0
        out["g_x"] = pow2_scale(xhat_max)
    return out


# ----------------------------------------------------------------------------- forward
def lowrank_down(xhat: np.ndarray, L1: np.ndarray) -> np.ndarray:
    xhat = np.ascontiguousarray(xhat, np.float32)
    M, K = xhat.shape
    r = L1.shape[1]
    t = np.zeros((M, r), np.uint16)
    if r:
        lib().orc_lowrank_down(M, K, r, _p(xhat), _p(np.ascontiguousarray(L1, np.uint16)), _p(t))
    return t


def act_tensor_scale(xhat: np.ndarray) -> float:
    """Dynamic per-tensor NVFP4 activation scale: pow2_scale of the largest |x^|
    of the tensor being quantized (a first pass over the whole activation, then
    the block quantizer with that scale).  The static scale of prepare is the
    same formula applied to the calibration statistic instead."""
    return pow2_scale(float(np.abs(np.asarray(xhat, np.float32)).max()) if np.size(xhat) else 0.0)


def quantize_act(X_bf16: np.ndarray, prep: dict):
    """Activation side of the layer: smoothing, 4-bit group quantization and the
    low-rank down-projection t = bf16(bf16(x^) L1).  Returns dict(xhat, codes,
    scales, t, g_x); g_x is the activation per-tensor scale used (NVFP4: the
    prepared static one, or, when prep["g_x"] is 0, the dynamic one of this X)."""
    xhat = smooth_act(X_bf16, prep["inv_lambda"])
    if prep["fmt"] == INT4:
        g = 1.0
        codes, scales = quant_int4(xhat)
    else:
        g = prep["g_x"] if prep["g_x"] != 0 else act_tensor_scale(xhat)
        codes, scales = quant_nvfp4(xhat, g)
    return dict(xhat=xhat, codes=codes, scales=scales, t=lowrank_down(xhat, prep["L1"]), g_x=g)


def forward_from_act(act: dict, prep: dict, want_f64: bool = False):
    """y = main + t L2 + b in binary64, rounded to bf16 (see svdq_oracle.c)."""
    codes = np.ascontiguousarray(act["codes"], np.uint8)
    M = codes.shape[0]
    N, K, r = prep["N"], prep["K"], prep["rank"]
    y = np.empty((M, N), np.uint16)
    yd = np.empty((M, N), np.float64) if want_f64 else None
    t = np.ascontiguousarray(act["t"], np.uint16) if r else np.zeros((M, 1), np.uint16)
    L2 = np.ascontiguousarray(prep["L2"], np.uint16) if r else np.zeros((1, N), np.uint16)
    sc_dtype = np.uint16 if prep["fmt"] == INT4 else np.uint8
    lib().orc_forward_out(M, N, K, r, prep["fmt"], _p(codes), _p(np.ascontiguousarray(act["scales"], sc_dtype)),
                          _p(np.ascontiguousarray(prep["wcodes"], np.uint8)),
                          _p(np.ascontiguousarray(prep["wscales"], sc_dtype)),
                          float(act.get("g_x", prep["g_x"])), float(prep["g_w"]), _p(t), _p(L2), _p(prep["bias"]),
                          _p(yd) if want_f64 else None, _p(y))
    return (y, yd) if want_f64 else y


def forward(X_bf16: np.ndarray, prep: dict, want_f64: bool = False):
    return forward_from_act(quantize_act(X_bf16, prep), prep, want_f64)


def int4_group_acc(xcodes: np.ndarray, wcodes: np.ndarray) -> np.ndarray:
    """INT4 per-group integer accumulators acc[g, m, n] = sum_{k in g} qx[m,k] qw[n,k]."""
    xcodes = np.ascontiguousarray(xcodes, np.uint8)
    wcodes = np.ascontiguousarray(wcodes, np.uint8)
    M, N, K = xcodes.shape[0], wcodes.shape[0], 2 * xcodes.shape[1]
    acc = np.empty((K // 64, M, N), np.int32)
    lib().orc_int4_group_acc(M, N, K, _p(xcodes), _p(wcodes), _p(acc))
    return acc


# ----------------------------------------------------------------------------- awq_w4a16
# The second runtime layer of the pages ("Hugging Face встроила Nunchaku в
# Diffusers ...", paragraph on Nunchaku Lite): 4-bit weights with 16-bit
# activations for precision-sensitive normalization / modulation layers (adaLN in
# FLUX).  The pages name AWQ and say nothing more; the readings here are:
#   - activation-aware per-input-channel scale s_j = mean|x_j|^alpha (1 where the
#     mean is 0), alpha from the grid 0, 0.05, ..., 1 minimising the layer's
#     output error on its own calibration input (the AWQ form);
#   - weights W diag(s) quantized with the same INT4 group-64 quantizer as the
#     svdq_w4a4 residual (symmetric, fp16 scale);
#   - forward y = (f32(x) * inv_s) . dequant(Q4(W diag(s)))^T + b, the activation
#     product in binary32 (as in the smoothing step), the rest exact in binary64,
#     rounded once to bf16.
AWQ_ALPHAS = tuple(i / 20.0 for i in range(21))


def awq_mean_abs(X_bf16: np.ndarray) -> np.ndarray:
    """Calibration statistic of the activation-aware scale: mean |x| per input channel (binary64)."""
    return np.abs(bf16_to_f32(X_bf16).astype(np.float64)).mean(axis=0)


def awq_channel_scales(mean_abs: np.ndarray, alpha: float):
    """s_j = mean|x_j|^alpha in binary64 (1 where the mean is 0); returns (s, float32(s), float32(1/float32(s)))."""
    m = np.asarray(mean_abs, np.float64)
    s = np.ones_like(m)
    nz = m > 0
    s[nz] = m[nz] ** float(alpha)
    s_f = s.astype(np.float32)
    inv = (1.0 / s_f.astype(np.float64)).astype(np.float32)
    return s, s_f, inv


def awq_quant_weights(W_bf16: np.ndarray, s_f32: np.ndarray):
    """Q4(W diag(s)): the scaled weight rounded to binary32, then INT4 groups of 64 (codes, fp16 scales)."""
    Wf = bf16_to_f32(np.ascontiguousarray(W_bf16, np.uint16)).astype(np.float64)
    Ws = (Wf * np.asarray(s_f32, np.float32).astype(np.float64)[None, :]).astype(np.float32)
    return quant_int4(Ws)


def awq_forward(X_bf16: np.ndarray, prep: dict, want_f64: bool = False):
    """y = (f32(x) * inv_s) . (q * S)^T + b in binary64 from the binary32 x^, rounded to bf16."""
    xhat = smooth_act(X_bf16, prep["inv_s"]).astype(np.float64)
    deq = dequant(prep["wcodes"], prep["wscales"], INT4)
    yd = xhat @ deq.T + bf16_to_f32(prep["bias"]).astype(np.float64)[None, :]
    y = f64_to_bf16(np.ascontiguousarray(yd))
    return (y, yd) if want_f64 else y


def awq_output_error(X_bf16: np.ndarray, W_bf16: np.ndarray, mean_abs: np.ndarray, alpha: float) -> float:
    """Squared output error sum_mn (x^ . deq^T - x . W^T)^2 (no bias) of one grid point, binary64."""
    _, s_f, inv = awq_channel_scales(mean_abs, alpha)
    codes, scales = awq_quant_weights(W_bf16, s_f)
    xhat = smooth_act(X_bf16, inv).astype(np.float64)
    ref = bf16_to_f32(X_bf16).astype(np.float64) @ bf16_to_f32(W_bf16).astype(np.float64).T
    return float(((xhat @ dequant(codes, scales, INT4).T - ref) ** 2).sum())


def awq_prepare(W_bf16: np.ndarray, bias_bf16, X_calib_bf16: np.ndarray, alphas=AWQ_ALPHAS):
    """Activation-aware preparation of one awq_w4a16 layer: the first alpha of the
    grid with the smallest output error on the calibration input wins."""
    W = np.ascontiguousarray(W_bf16, np.uint16)
    N, K = W.shape
    mabs = awq_mean_abs(X_calib_bf16)
    best = None
    for a in alphas:
        err = awq_output_error(X_calib_bf16, W, mabs, a)
        if best is None or err < best[1]:
            best = (a, err)
    a = best[0]
    _, s_f, inv = awq_channel_scales(mabs, a)
    codes, scales = awq_quant_weights(W, s_f)
    return dict(N=N, K=K, alpha=float(a), err=best[1], s=s_f, inv_s=inv, wcodes=codes, wscales=scales,
                bias=(np.zeros(N, np.uint16) if bias_bf16 is None else np.ascontiguousarray(bias_bf16, np.uint16)))


# ----------------------------------------------------------------------------- int8 tensorwise W8A8
# The INT8 tensorwise W8A8 layer the Krea page ("SVDQuant ускоряет Krea 2 вдвое ...",
# section "Решение: INT8 и W4A4") compares with W4A4: symmetric 8-bit codes with one
# scale per tensor, for the weight (fixed at preparation) and for the activation
# (taken from the tensor being quantized at every call: a first pass for its
# largest |x|, then the quantizer).  No smoothing and no low-rank branch.
W8_QMAX = 127


def w8_tensor_scale(v: np.ndarray) -> np.float32:
    """s = fl32(max|v| / 127) (0 for an all-zero tensor)."""
    v = np.asarray(v, np.float32)
    amax = np.float32(np.abs(v).max()) if v.size else np.float32(0.0)
    return np.float32(amax / np.float32(W8_QMAX))


def quant_w8(v: np.ndarray, s: np.float32) -> np.ndarray:
    """Codes clamp(rne(v * fl32(1/s)), -127, 127) as int8, the product in binary32
    (all zero when s is 0)."""
    v = np.asarray(v, np.float32)
    if s == 0:
        return np.zeros(v.shape, np.int8)
    inv = np.float32(np.float32(1.0) / np.float32(s))
    q = np.rint((v * inv).astype(np.float32))
    return np.clip(q, -W8_QMAX, W8_QMAX).astype(np.int8)


def w8a8_prepare(W_bf16: np.ndarray, bias_bf16=None) -> dict:
    W = np.ascontiguousarray(W_bf16, np.uint16)
    N, K = W.shape
    w = bf16_to_f32(W)
    s_w = w8_tensor_scale(w)
    return dict(N=N, K=K, s_w=s_w, wcodes=quant_w8(w, s_w),
                bias=(np.zeros(N, np.uint16) if bias_bf16 is None else np.ascontiguousarray(bias_bf16, np.uint16)))


def w8a8_quantize_act(X_bf16: np.ndarray) -> dict:
    x = bf16_to_f32(np.ascontiguousarray(X_bf16, np.uint16))
    s_x = w8_tensor_scale(x)
    return dict(codes=quant_w8(x, s_x), s_x=s_x)


def w8a8_forward_from_act(act: dict, prep: dict, want_f64: bool = False):
    """y = bf16(s_x s_w (qx . qw^T) + b): the integer product exactly (int64), the
    rest in binary64."""
    acc = act["codes"].astype(np.int64) @ prep["wcodes"].astype(np.int64).T
    yd = float(act["s_x"]) * float(prep["s_w"]) * acc.astype(np.float64) + \
        bf16_to_f32(prep["bias"]).astype(np.float64)[None, :]
    y = f64_to_bf16(np.ascontiguousarray(yd))
    return (y, yd) if want_f64 else y


def w8a8_forward(X_bf16: np.ndarray, prep: dict, want_f64: bool = False):
    return w8a8_forward_from_act(w8a8_quantize_act(X_bf16), prep, want_f64)
