"""Shared helpers for the GPU parity tests: oracle-prepared layers on the device,
workspace read-back into canonical layouts, and the output tolerance.

The prepared weights fed to the CUDA path come from the ORACLE's prepare (never
the other way round); svdq_pack only re-lays them out."""
from __future__ import annotations

import functools

import numpy as np

import oracle
import workloads as wl

# Tolerances.
# t: the oracle sums bf16(x^) L1 exactly (binary64) and rounds once to bf16; the
#    GPU sums in fp32 in tensor-core order.  Any fp32 summation order of K terms
#    is within gamma_K * sum|terms| of the exact sum (gamma_K ~ K u, u = 2^-24;
#    taken as K 2^-23 to cover truncating accumulators), plus one bf16 ulp of
#    the final rounding.
# Y: the stated gates rel-L2 <= 1e-3 and max-abs 2e-2, with the elementwise
#    bound widened by exactly one bf16 ulp of the oracle value: two correct fp32
#    accumulation orders of the same exact sum round to neighbouring bf16 values
#    once |y| >= 4, where one bf16 ulp (1/32) already exceeds 2e-2.  Nothing
#    else widens the gate; the fp32 forward-error bound of the arithmetic
#    (y_error_bound) is reported beside it as a diagnostic only.
REL_L2 = 1e-3
MAX_ABS = 2e-2


def int4_bytes_to_packed(b: np.ndarray) -> np.ndarray:
    """Device INT4 codes (one E4M3 byte per code, the byte of the code's
    integer value) -> canonical packed two's-complement nibbles, element 2i in
    the low nibble.  A byte that is not the E4M3 encoding of an integer in
    [-8, 7] (a negative zero included) decodes to an out-of-range marker so the
    bit-exact comparison fails."""
    v = oracle.e4m3_to_f32(b.reshape(-1)).reshape(b.shape).astype(np.float64)
    ok = (v == np.round(v)) & (v >= -8) & (v <= 7) & ~((b & 0x7F) == 0) | (b == 0)
    assert ok.all(), f"{(~ok).sum()} device INT4 code bytes are not canonical E4M3 integers"
    n = (v.astype(np.int64) & 15).astype(np.uint8)
    return (n[:, 0::2] | (n[:, 1::2] << 4)).astype(np.uint8)


def bf(h):
    return oracle.bf16_to_f32(h).astype(np.float64)


def bf16_ulp(x):
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0**-126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def t_sum_bound(act: dict, prep: dict):
    """fp32 summation bound of t = bf16(x^) L1, per element [M, r]."""
    K = prep["K"]
    if not prep["rank"]:
        return np.zeros((act["xhat"].shape[0], 0))
    S = np.abs(bf(oracle.f32_to_bf16(act["xhat"]))) @ np.abs(bf(prep["L1"]))
    return K * 2.0**-23 * S


def y_error_bound(act: dict, prep: dict):
    """Forward-error allowance of y (beyond the final bf16 rounding) for the rows of `act`."""
    K = prep["K"]
    fmt = prep["fmt"]
    gx = prep["g_x"] if fmt == oracle.NVFP4 else 1.0
    gw = prep["g_w"] if fmt == oracle.NVFP4 else 1.0
    dqx = np.abs(oracle.dequant(act["codes"], act["scales"], fmt, gx))
    dqw = np.abs(oracle.dequant(prep["wcodes"], prep["wscales"], fmt, gw))
    bound = (K + prep["rank"]) * 2.0**-23 * (dqx @ dqw.T)
    if prep["rank"]:
        t = bf(act["t"])
        dt = bf16_ulp(t) + t_sum_bound(act, prep)
        L2 = np.abs(bf(prep["L2"]))
        bound += dt @ L2 + (K + prep["rank"]) * 2.0**-23 * (np.abs(t) @ L2)
    return bound


def y_stats(y_gpu_bits, y_orc_bits, diag=None):
    g, o = bf(y_gpu_bits), bf(y_orc_bits)
    d = np.abs(g - o)
    lim = MAX_ABS + bf16_ulp(o)
    s = dict(rel_l2=float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30)), max_abs=float(d.max()),
             n_over_abs=int(np.sum(d > MAX_ABS)), n_over_abs_ulp=int(np.sum(d > lim)),
             n_flip=int(np.sum(g != o)), worst_excess=float(np.max(d - lim)),
             nonfinite=int(np.sum(~np.isfinite(g))))
    if diag is not None:  # how much of the fp32 forward-error allowance the result uses
        s["max_err_over_fp32_bound"] = float(np.max(np.maximum(d - bf16_ulp(o), 0.0) / np.maximum(diag, 1e-300)))
    return s


def assert_y_close(y_gpu_bits, y_orc_bits, act=None, prep=None):
    """rel-L2 <= 1e-3 and |dy| <= 2e-2 + 1 bf16 ulp(|y_oracle|) on every element."""
    diag = y_error_bound(act, prep) if act is not None else None
    s = y_stats(y_gpu_bits, y_orc_bits, diag)
    assert s["nonfinite"] == 0, s
    assert s["rel_l2"] <= REL_L2, s
    assert s["n_over_abs_ulp"] == 0, s
    return s


def check_layer_output(gl, X, prep, y, rows=None):
    """Parity of one svdq_w4a4 forward whose workspace still holds its quantized
    activations: codes and scales bit-exact on every row; the GPU's t within its
    summation bound (assert_t_close); Y on `rows` (all by default) within the
    stated gate given the GPU's own t (the low-rank input teacher-forced: a t
    one bf16 ulp away from the oracle's, which its own gate allows, moves y by
    that ulp times L2, more than 2e-2 where |t| is large); and the fully
    independent oracle output (its own t) within rel-L2 1e-3, its statistics
    reported."""
    M = X.shape[0]
    got = gl.read_act(M)
    ref = oracle.quantize_act(X, prep)
    if "g_x" in got and prep["fmt"] == oracle.NVFP4:
        assert got["g_x"] == ref["g_x"], (got["g_x"], ref["g_x"])
    np.testing.assert_array_equal(got["codes"], ref["codes"])
    np.testing.assert_array_equal(got["scales"], ref["scales"])
    st = assert_t_close(got["t"], ref["t"], ref, prep) if prep["rank"] else {}
    rows = np.arange(M) if rows is None else np.asarray(rows)
    sub = {k: (v[rows] if np.ndim(v) else v) for k, v in ref.items()}
    taught = dict(sub, t=got["t"][rows])
    s = assert_y_close(y[rows], oracle.forward_from_act(taught, prep), taught, prep)
    ind = y_stats(y[rows], oracle.forward_from_act(sub, prep))
    assert ind["rel_l2"] <= REL_L2, ind
    s.update(indep_rel_l2=ind["rel_l2"], indep_max_abs=ind["max_abs"], indep_n_over_abs_ulp=ind["n_over_abs_ulp"])
    s.update(st)
    return s


def tile_rows(M, seed, spread=40, tile=128):
    """Sampled output rows: one seeded row inside every 128-row M tile (the ragged
    last tile included), the first/last rows of the first two tiles and of the
    tail, and a seeded spread."""
    rng = np.random.default_rng(seed)
    starts = np.arange(0, M, tile)
    per_tile = starts + rng.integers(0, np.minimum(tile, M - starts))
    fixed = [r for r in (0, 1, 127, 128, 255, M - 129, M - 128, M - 1) if 0 <= r < M]
    return np.unique(np.concatenate([fixed, per_tile, rng.choice(M, min(M, spread), replace=False)]))


def assert_t_close(t_gpu, t_orc, act=None, prep=None):
    g, o = bf(t_gpu), bf(t_orc)
    lim = bf16_ulp(np.maximum(np.abs(g), np.abs(o)))
    if act is not None:
        lim = lim + t_sum_bound(act, prep)
    bad = np.abs(g - o) > lim
    assert not bad.any(), (int(bad.sum()), float(np.abs(g - o).max()))
    return dict(t_flip_frac=float(np.mean(g != o)), t_max_abs=float(np.abs(g - o).max()) if g.size else 0.0)


@functools.lru_cache(maxsize=16)
def oracle_layer(layer: wl.Layer, seed: int = 0, alpha: float = 0.5):
    X, W, b = wl.make_layer_inputs(layer, seed)
    amax = oracle.calib_absmax(X)
    prep = oracle.prepare(W, b, amax, alpha, layer.rank, layer.fmt)
    return X, W, b, prep


def canonical_from_oracle(prep: dict) -> dict:
    return dict(N=prep["N"], K=prep["K"], rank=prep["rank"], fmt=prep["fmt"], alpha=prep["alpha"],
                g_x=prep["g_x"], g_w=prep["g_w"], lambda_=prep["lam"], inv_lambda=prep["inv_lambda"],
                L1=prep["L1"], L2=prep["L2"], wcodes=prep["wcodes"], wscales=prep["wscales"], bias=prep["bias"])


def sf_offset(row, block, katoms, tile_rows):
    tile, rin = row // tile_rows, row % tile_rows
    apt = (tile_rows + 127) // 128
    a, ra = rin // 128, rin % 128
    return ((tile * katoms + block // 4) * apt + a) * 512 + (ra % 32) * 16 + ((ra // 32) % 4) * 4 + block % 4


class GpuLayer:
    """An oracle-prepared layer resident on cuda:0 behind the C ABI."""

    def __init__(self, prep: dict):
        import torch

        import diffusion_transformer_w4a4_b200 as svdq

        self.svdq = svdq
        self.prep = prep
        self.lin = svdq.SvdqLinear(canonical_from_oracle(prep), device="cuda:0")
        self.torch = torch

    def x_dev(self, X):
        return self.torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).view(self.torch.bfloat16).to("cuda:0")

    def quantize(self, X):
        """Run the activation quantizer only; return canonical codes, scales, t."""
        torch, svdq = self.torch, self.svdq
        M = X.shape[0]
        ws = self.lin.workspace(M)
        svdq.svdq_quantize_act(self.lin.handle, self.x_dev(X), M, ws)
        torch.cuda.synchronize()
        return self.read_act(M)

    def read_act(self, M):
        svdq = self.svdq
        ws = self.lin.workspace(M).cpu().numpy()
        off, sz = svdq.svdq_workspace_layout(self.lin.handle, M)
        K, r = self.prep["K"], self.prep["rank"]
        if self.prep["fmt"] == oracle.NVFP4:
            codes = ws[off[0]:off[0] + sz[0]].reshape(M, K // 2)
        else:
            codes = int4_bytes_to_packed(ws[off[0]:off[0] + sz[0]].reshape(M, K))
        if self.prep["fmt"] == oracle.NVFP4:
            rows, blocks = np.meshgrid(np.arange(M), np.arange(K // 16), indexing="ij")
            scales = ws[off[1]:][sf_offset(rows, blocks, K // 64, 128)]
        else:
            scales = ws[off[1]:off[1] + sz[1]].view(np.uint16).reshape(K // 64, -1)[:, :M].T.copy()
        t = ws[off[2]:off[2] + sz[2]].view(np.uint16).reshape(M, r) if r else np.zeros((M, 0), np.uint16)
        g_x = self.prep["g_x"]
        if self.prep["fmt"] == oracle.NVFP4 and g_x == 0:
            # dynamic activation scale: the quantizer leaves g_x in the control block
            # (word 1) and stores t / g_x; undo the exact power-of-two scaling
            g_x = float(ws[off[3] + 4:off[3] + 8].view(np.float32)[0])
            t = oracle.f32_to_bf16(oracle.bf16_to_f32(t) * np.float32(g_x))
        return dict(codes=codes.copy(), scales=scales, t=t.copy(), g_x=g_x)

    def forward(self, X):
        torch = self.torch
        y = self.lin.forward(self.x_dev(X))
        torch.cuda.synchronize()
        return y.view(torch.int16).cpu().numpy().view(np.uint16)

    def status(self, M):
        return self.lin.status(M)
