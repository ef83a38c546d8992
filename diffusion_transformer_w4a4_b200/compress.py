"""Whole-model compression tool: target scan, calibration, quantization, packing.

"Hugging Face встроила Nunchaku в Diffusers ..." (iitog.ru), paragraph on the
compressor that ships with the runtime: a model is first scanned for the linear
layers to replace, then calibrated, quantized and packed into a checkpoint the
runtime loads; attention and MLP projections become svdq_w4a4 layers and the
precision-sensitive normalization / modulation (adaLN) layers become
awq_w4a16 layers (paragraph on Nunchaku Lite).

This module does those four steps over a model's list of linear layers, with
every numeric step in the library's own host code (svdq_prepare,
svdq_awq_prepare through the C ABI):

  scan(layers, rules)        -> one LayerPlan per layer: svdq_w4a4 / awq_w4a16 /
                                keep (left in bf16), by name pattern and by the
                                shapes the kernels accept
  calibrate(plan, inputs)    -> per layer, what its preparation needs from its own
                                inputs: the per-channel max |x| (svdq_w4a4) or a
                                bounded sample of input rows (awq_w4a16)
  quantize(...)              -> canonical prepared arrays per layer
  pack(path, ...)            -> one file: a JSON header and the canonical arrays,
                                each 1024-byte aligned
  load(path) / read_packed   -> device layers (SvdqLinear / AwqLinear) or the
                                canonical arrays on the host

The file holds the canonical (format-defined) arrays, not the device blobs, so
a checkpoint survives changes of the kernels' internal layout; `load` re-lays
them out with svdq_pack / svdq_awq_pack, which is a host permutation.

File layout ("svdq pack" version 1): 8-byte magic b"SVDQPACK", uint32 version,
uint32 header length H, H bytes of UTF-8 JSON, zero padding to 1024, then the
arrays.  The header lists, per layer, its name, kind, shape, rank, format,
scales and for every array its byte offset, byte count, dtype and shape.

Command line (synthetic model, no checkpoint needed):
  python -m diffusion_transformer_w4a4_b200.compress --synthetic-flux-block \
      --tokens 512 --rank 32 --fmt nvfp4 --out block.svdq
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import re
import struct

import numpy as np

MAGIC = b"SVDQPACK"
VERSION = 1
ALIGN = 1024

SVDQ = "svdq_w4a4"
AWQ = "awq_w4a16"
KEEP = "keep"

# Default target rules for diffusion-transformer layer names, tried in order:
# modulation / adaLN / normalization linears keep 16-bit activations (AWQ),
# attention and MLP projections become W4A4, everything else stays bf16.
DEFAULT_RULES = (
    (r"(^|\.)(norm\w*|adaln\w*|ada_ln\w*|mod\w*|modulation)(\.|$)", AWQ),
    (r"(^|\.)(attn|attention|self_attn|cross_attn)\.", SVDQ),
    (r"(^|\.)(ff|ff_context|mlp|ffn|feed_forward)(\.|$)", SVDQ),
    (r"(^|\.)(to_q|to_k|to_v|to_qkv|qkv|to_out|proj_mlp|proj_out|fc1|fc2|linear1|linear2)(\.|$)", SVDQ),
)


@dataclasses.dataclass
class LinearSpec:
    """One linear layer of a model: y = x W^T + b, W [N, K] and b [N] as bf16 bits."""

    name: str
    W: np.ndarray
    bias: np.ndarray | None = None

    @property
    def N(self) -> int:
        return int(self.W.shape[0])

    @property
    def K(self) -> int:
        return int(self.W.shape[1])


@dataclasses.dataclass
class LayerPlan:
    name: str
    kind: str  # SVDQ, AWQ or KEEP
    N: int
    K: int
    rank: int = 0
    fmt: str = ""
    reason: str = ""


def svdq_shape_ok(N: int, K: int, rank: int) -> bool:
    """Shapes the svdq_w4a4 kernels accept (see include/svdq.h)."""
    return K % 256 == 0 and N % 16 == 0 and N >= 16 and 0 <= rank <= min(K, N, 128) and rank % 16 == 0


def awq_shape_ok(N: int, K: int) -> bool:
    return K % 64 == 0 and 64 <= K <= 12288 and N >= 1


def scan(layers, rules=DEFAULT_RULES, rank: int = 32, fmt: str = "nvfp4") -> list[LayerPlan]:
    """Choose a target for every layer: the first rule whose pattern matches the
    name decides the kind; a layer whose shape the chosen kernel cannot take
    falls back to awq_w4a16 (if it fits) or stays in bf16.  The rank is clipped
    to what the layer's shape allows (a multiple of 16, at most min(K, N))."""
    plans = []
    for spec in layers:
        N, K = spec.N, spec.K
        kind, why = KEEP, "no rule matched"
        for pat, k in rules:
            m = re.search(pat, spec.name)
            if m:
                kind, why = k, f"name matches {m.group(0).strip('.')!r}"
                break
        r = 0
        if kind == SVDQ:
            r = min(rank, (min(K, N) // 16) * 16, 128)
            if not svdq_shape_ok(N, K, r):
                kind, why = (AWQ, "shape not supported by svdq_w4a4") if awq_shape_ok(N, K) else (
                    KEEP, "shape not supported by svdq_w4a4 or awq_w4a16")
                r = 0
        if kind == AWQ and not awq_shape_ok(N, K):
            kind, why = KEEP, "shape not supported by awq_w4a16"
        plans.append(LayerPlan(spec.name, kind, N, K, r if kind == SVDQ else 0, fmt if kind == SVDQ else "", why))
    return plans


def calibrate(plans, inputs: dict, awq_rows: int = 256) -> dict:
    """Per-layer calibration statistics from the layer's own inputs (bf16 bits
    [M, K], e.g. captured from a forward of the dense model): the per-input-channel
    max |x| for svdq_w4a4 layers, and up to `awq_rows` evenly spaced input rows for
    awq_w4a16 layers (the activation-aware scale search runs on them)."""
    stats = {}
    for p in plans:
        if p.kind == KEEP:
            continue
        x = np.ascontiguousarray(inputs[p.name], np.uint16)
        if x.ndim != 2 or x.shape[1] != p.K:
            raise ValueError(f"{p.name}: calibration input must be [M, {p.K}] bf16 bits")
        if p.kind == SVDQ:
            stats[p.name] = np.abs(_bf16_bits_to_f32(x)).max(axis=0).astype(np.float32)
        else:
            idx = np.unique(np.linspace(0, x.shape[0] - 1, min(awq_rows, x.shape[0])).round().astype(np.int64))
            stats[p.name] = np.ascontiguousarray(x[idx])
    return stats


def quantize(layers, plans, stats, alpha: float = 0.5) -> dict:
    """Canonical prepared arrays per layer, from the library's host preparation."""
    from . import svdq_awq_prepare, svdq_prepare

    specs = {s.name: s for s in layers}
    out = {}
    for p in plans:
        if p.kind == KEEP:
            continue
        s = specs[p.name]
        if p.kind == SVDQ:
            out[p.name] = svdq_prepare(s.W, s.bias, stats[p.name], alpha, p.rank, p.fmt)
        else:
            out[p.name] = svdq_awq_prepare(s.W, s.bias, stats[p.name])
    return out


_FMT_CODES = {"int4": 1, "nvfp4": 2}  # svdq_format values of include/svdq.h
_SVDQ_FIELDS = ("lambda_", "inv_lambda", "L1", "L2", "wcodes", "wscales", "bias")
_AWQ_FIELDS = ("s", "inv_s", "wcodes", "wscales", "bias")


def _align(n: int) -> int:
    return (n + ALIGN - 1) // ALIGN * ALIGN


def pack(path: str, plans, canon: dict, layers=None) -> dict:
    """Write the packed checkpoint; `layers` (optional) also stores the bf16
    weights of the layers kept in bf16 so the file describes the whole model.
    Returns the header."""
    specs = {s.name: s for s in (layers or [])}
    entries, blobs = [], []
    off = 0

    def add(arr):
        nonlocal off
        a = np.ascontiguousarray(arr)
        rec = [off, int(a.nbytes), a.dtype.str, list(a.shape)]
        blobs.append((off, a))
        off = _align(off + a.nbytes)
        return rec

    for p in plans:
        e = dataclasses.asdict(p)
        if p.kind == SVDQ:
            c = canon[p.name]
            e.update(alpha=float(c["alpha"]), g_x=float(c["g_x"]), g_w=float(c["g_w"]),
                     arrays={f: add(c[f]) for f in _SVDQ_FIELDS})
        elif p.kind == AWQ:
            c = canon[p.name]
            e.update(alpha=float(c["alpha"]), arrays={f: add(c[f]) for f in _AWQ_FIELDS})
        elif p.name in specs:
            sp = specs[p.name]
            arrays = {"W": add(sp.W)}
            if sp.bias is not None:
                arrays["bias"] = add(sp.bias)
            e.update(arrays=arrays)
        entries.append(e)
    header = {"format": "svdq pack", "version": VERSION, "align": ALIGN, "layers": entries}
    hbytes = json.dumps(header).encode()
    base = _align(len(MAGIC) + 8 + len(hbytes))
    with open(path, "wb") as f:
        f.write(MAGIC + struct.pack("<II", VERSION, len(hbytes)) + hbytes)
        f.write(b"\0" * (base - f.tell()))
        for o, a in blobs:
            f.seek(base + o)
            f.write(a.tobytes())
        f.truncate(base + off)
    return header


def read_packed(path: str):
    """(header, {name: canonical dict}) from a packed checkpoint, on the host.
    bf16 layers come back as {"W": ..., "bias": ...}."""
    raw = np.fromfile(path, dtype=np.uint8)
    if raw[:8].tobytes() != MAGIC:
        raise ValueError(f"{path}: not an svdq pack file")
    version, hlen = struct.unpack("<II", raw[8:16].tobytes())
    if version != VERSION:
        raise ValueError(f"{path}: pack version {version}, this reader knows {VERSION}")
    header = json.loads(raw[16:16 + hlen].tobytes().decode())
    base = _align(16 + hlen)
    out = {}
    for e in header["layers"]:
        arrays = {}
        for f, (o, n, dt, shape) in e.get("arrays", {}).items():
            arrays[f] = raw[base + o:base + o + n].view(np.dtype(dt)).reshape(shape).copy()
        if e["kind"] == SVDQ:
            arrays.update(N=e["N"], K=e["K"], rank=e["rank"], fmt=_FMT_CODES[e["fmt"]], alpha=e["alpha"],
                          g_x=e["g_x"], g_w=e["g_w"])
        elif e["kind"] == AWQ:
            arrays.update(N=e["N"], K=e["K"], alpha=e["alpha"])
        out[e["name"]] = arrays
    return header, out


def load(path: str, device=None) -> dict:
    """Device layers of a packed checkpoint: {name: SvdqLinear | AwqLinear | None}
    (None for layers kept in bf16)."""
    from . import AwqLinear, SvdqLinear

    header, canon = read_packed(path)
    layers = {}
    for e in header["layers"]:
        if e["kind"] == SVDQ:
            layers[e["name"]] = SvdqLinear(canon[e["name"]], device=device)
        elif e["kind"] == AWQ:
            layers[e["name"]] = AwqLinear(canon[e["name"]], device=device)
        else:
            layers[e["name"]] = None
    return layers


def compress(layers, inputs: dict, path: str, rank: int = 32, fmt: str = "nvfp4", alpha: float = 0.5,
             rules=DEFAULT_RULES):
    """scan -> calibrate -> quantize -> pack; returns (plans, canonical arrays)."""
    plans = scan(layers, rules, rank, fmt)
    stats = calibrate(plans, inputs)
    canon = quantize(layers, plans, stats, alpha)
    pack(path, plans, canon, layers)
    return plans, canon


# ----------------------------------------------------------------------------- synthetic model
def _bf16_bits_to_f32(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _f32_to_bf16_bits(a):
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def synthetic_flux_block(tokens: int = 512, seed: int = 0, width: int = 3072):
    """The linear layers of one synthetic FLUX-style double-stream block (image
    stream) with seeded weights ~ N(0, 0.02^2) and biases ~ N(0, 0.01^2), and
    calibration inputs from a dense bf16 forward of the block's linears on seeded
    tokens ~ N(0, 1) with 0.5 % of the channels scaled x50: the adaLN modulation
    linear (input: a per-sample conditioning vector, batch 2), the fused QKV
    projection, the attention output projection (its input: the Q slice standing
    in for the attention output), the MLP up-projection and, after a GELU, the
    MLP down-projection."""
    from scipy.special import erf

    D = width
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0x5D0A])))

    def spec(name, K, N):
        W = _f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
        b = _f32_to_bf16_bits(rng.standard_normal(N, dtype=np.float32) * np.float32(0.01))
        return LinearSpec(name, W, b)

    def tokens_in(M, K):
        x = rng.standard_normal((M, K), dtype=np.float32)
        ch = rng.choice(K, size=max(1, int(round(0.005 * K))), replace=False)
        x[:, ch] *= np.float32(50.0)
        return _f32_to_bf16_bits(x)

    def dense(x, sp):
        y = _bf16_bits_to_f32(x) @ _bf16_bits_to_f32(sp.W).T + _bf16_bits_to_f32(sp.bias)[None, :]
        return _f32_to_bf16_bits(np.ascontiguousarray(y, np.float32))

    layers = [spec("transformer_blocks.0.norm1.linear", D, 6 * D), spec("transformer_blocks.0.attn.to_qkv", D, 3 * D),
              spec("transformer_blocks.0.attn.to_out.0", D, D), spec("transformer_blocks.0.ff.net.0.proj", D, 4 * D),
              spec("transformer_blocks.0.ff.net.2", 4 * D, D)]
    mod, qkv, out, up, down = layers
    c = tokens_in(2, D)
    x = tokens_in(tokens, D)
    a = np.ascontiguousarray(dense(x, qkv)[:, :D])
    h_out = dense(a, out)
    g = _bf16_bits_to_f32(dense(h_out, up)).astype(np.float64)
    h_gelu = _f32_to_bf16_bits((0.5 * g * (1.0 + erf(g / np.sqrt(2.0)))).astype(np.float32))
    inputs = {mod.name: c, qkv.name: x, out.name: a, up.name: h_out, down.name: h_gelu}
    return layers, inputs


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--synthetic-flux-block", action="store_true", help="compress a seeded synthetic FLUX block")
    ap.add_argument("--tokens", type=int, default=512)
    ap.add_argument("--width", type=int, default=3072)
    ap.add_argument("--rank", type=int, default=32)
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "int4"])
    ap.add_argument("--alpha", type=float, default=0.5)
    ap.add_argument("--out", required=True)
    a = ap.parse_args(argv)
    if not a.synthetic_flux_block:
        ap.error("only the synthetic model is built in; use the Python API (compress) for a real one")
    layers, inputs = synthetic_flux_block(a.tokens, width=a.width)
    plans, _ = compress(layers, inputs, a.out, a.rank, a.fmt, a.alpha)
    for p in plans:
        print(f"{p.name:45s} {p.kind:10s} {p.K:6d} -> {p.N:6d} rank {p.rank:3d} {p.fmt:6s} ({p.reason})")
    print("wrote", a.out)


if __name__ == "__main__":
    main()
