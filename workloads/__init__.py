"""Seeded synthetic inputs for the svdq_w4a4 linear layer.

This module only draws random tensors with the shapes and value distributions of
the FLUX-style layers that the layer is exercised on.  It holds none of the
layer's arithmetic (no smoothing, no SVD, no quantization), so that both the
oracle and the CUDA path can consume the same inputs without sharing any of the
method's code.

Distributions (one table entry per workload):
  * X   ~ N(0, 1), bf16, with a fixed set of "outlier" input channels multiplied
          by a constant factor for every token (1% x30 for the small layers,
          0.5% x50 for the FLUX-shaped ones).  The MLP down-projection input is
          GELU(z), z ~ N(0, 1), with no extra outliers (skewed, mostly >= 0).
  * W   ~ N(0, 0.02^2), bf16, nn.Linear layout [N, K].
  * b   ~ N(0, 0.01^2), bf16, [N].
Token count 4608 = 4096 image tokens (1024x1024 image, 16x16 patches of the
latent) + 512 text tokens, the FLUX 1024^2 setting; batch 2 doubles it.

Random streams come from numpy's PCG64 seeded by SeedSequence([seed, layer,
stream]); bf16 values are produced by round-to-nearest-even of float32 draws.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

INT4 = "int4"
NVFP4 = "nvfp4"

# stream ids
_S_X, _S_W, _S_BIAS, _S_OUTLIER, _S_GELU = 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class Layer:
    name: str
    M: int
    K: int
    N: int
    rank: int
    fmt: str
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    gelu_input: bool = False
    layer_id: int = 0

    @property
    def n_outliers(self) -> int:
        return int(round(self.outlier_frac * self.K))

    def with_(self, **kw) -> "Layer":
        return dataclasses.replace(self, **kw)


def _flux(M, K, N, rank, fmt, name, layer_id, gelu=False):
    if gelu:
        return Layer(name, M, K, N, rank, fmt, 0.0, 1.0, True, layer_id)
    return Layer(name, M, K, N, rank, fmt, 0.005, 50.0, False, layer_id)


# The five workloads.  Each entry is one linear layer (or a list of them).
WORKLOADS = {
    # single INT4 layer, 128 tokens, K=N=1024, rank 32, 1% outlier channels x30
    "c1_int4_128x1024x1024_r32": [Layer("c1", 128, 1024, 1024, 32, INT4, 0.01, 30.0, False, 0)],
    # same layer in NVFP4 at 1024 tokens, K=N=3072
    "c2_nvfp4_1024x3072x3072_r32": [Layer("c2", 1024, 3072, 3072, 32, NVFP4, 0.01, 30.0, False, 0)],
    # FLUX 1024^2 image block fused QKV projection
    "c3_qkv_4608x3072x9216_r32": [_flux(4608, 3072, 9216, 32, f, f"c3_{f}", 0) for f in (NVFP4, INT4)],
    # FLUX MLP pair: up-projection and down-projection (GELU input)
    "c4_mlp_4608x3072x12288_r32": [
        _flux(4608, 3072, 12288, 32, NVFP4, "c4up_nvfp4", 0),
        _flux(4608, 12288, 3072, 32, NVFP4, "c4dn_nvfp4", 1, gelu=True),
        _flux(4608, 3072, 12288, 32, INT4, "c4up_int4", 0),
        _flux(4608, 12288, 3072, 32, INT4, "c4dn_int4", 1, gelu=True),
    ],
}

# Full synthetic transformer block's linears at batch 2 (M = 9216): QKV, out-proj,
# MLP up, MLP down; NVFP4; rank swept over 16/32/64/128.
BLOCK_M = 9216
BLOCK_RANKS = (16, 32, 64, 128)


def block_layers(rank: int, M: int = BLOCK_M):
    return [
        _flux(M, 3072, 9216, rank, NVFP4, f"c5_qkv_r{rank}", 10),
        _flux(M, 3072, 3072, rank, NVFP4, f"c5_out_r{rank}", 11),
        _flux(M, 3072, 12288, rank, NVFP4, f"c5_up_r{rank}", 12),
        _flux(M, 12288, 3072, rank, NVFP4, f"c5_down_r{rank}", 13, gelu=True),
    ]


# awq_w4a16 layers: FLUX adaLN modulation linears.  Their input is the per-sample
# conditioning vector, so M is the batch (2 = the classifier-free-guidance pair);
# double-stream blocks map 3072 -> 6 x 3072, single-stream blocks 3072 -> 3 x 3072.
# Same value recipe as the FLUX-style svdq layers (N(0,1), 0.5 % channels x50).
AWQ = "awq"
AWQ_LAYERS = {
    "awq_flux_double_mod_2x3072x18432": _flux(2, 3072, 18432, 0, AWQ, "awq_double_mod", 20),
    "awq_flux_single_mod_2x3072x9216": _flux(2, 3072, 9216, 0, AWQ, "awq_single_mod", 21),
}


def _rng(seed: int, layer_id: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer_id, stream])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def outlier_channels(layer: Layer, seed: int = 0) -> np.ndarray:
    n = layer.n_outliers
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(_rng(seed, layer.layer_id, _S_OUTLIER).choice(layer.K, size=n, replace=False))


def make_x(layer: Layer, seed: int = 0, M: int | None = None) -> np.ndarray:
    """Activation X as bf16 bits, shape [M, K]."""
    M = layer.M if M is None else M
    if layer.gelu_input:
        z = _rng(seed, layer.layer_id, _S_GELU).standard_normal((M, layer.K), dtype=np.float32).astype(np.float64)
        from scipy.special import erf

        x = (0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))).astype(np.float32)
    else:
        x = _rng(seed, layer.layer_id, _S_X).standard_normal((M, layer.K), dtype=np.float32)
        ch = outlier_channels(layer, seed)
        if ch.size:
            x[:, ch] *= np.float32(layer.outlier_scale)
    return f32_to_bf16_bits(x)


def make_w(layer: Layer, seed: int = 0) -> np.ndarray:
    """Weight W as bf16 bits, nn.Linear layout [N, K]."""
    w = _rng(seed, layer.layer_id, _S_W).standard_normal((layer.N, layer.K), dtype=np.float32) * np.float32(0.02)
    return f32_to_bf16_bits(w)


def make_bias(layer: Layer, seed: int = 0) -> np.ndarray:
    b = _rng(seed, layer.layer_id, _S_BIAS).standard_normal(layer.N, dtype=np.float32) * np.float32(0.01)
    return f32_to_bf16_bits(b)


def make_layer_inputs(layer: Layer, seed: int = 0):
    """(X, W, bias) as bf16 bit arrays."""
    return make_x(layer, seed), make_w(layer, seed), make_bias(layer, seed)


def small_layer(M, K, N, rank, fmt, outlier_frac=0.01, outlier_scale=30.0, layer_id=0, gelu=False):
    """A layer with the same value distributions at an arbitrary (small) shape."""
    return Layer(f"small_{fmt}_{M}x{K}x{N}_r{rank}", M, K, N, rank, fmt,
                 0.0 if gelu else outlier_frac, 1.0 if gelu else outlier_scale, gelu, layer_id)
