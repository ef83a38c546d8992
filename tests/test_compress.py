"""The whole-model compression tool (scan -> calibrate -> quantize -> pack ->
read back) on the host: target choice by layer name and kernel shape limits,
calibration statistics, and a bit-exact round trip of every prepared array
through the packed file."""
import struct

import numpy as np
import pytest

from diffusion_transformer_w4a4_b200 import compress as cp


def _spec(name, K, N, seed=0):
    rng = np.random.default_rng(seed)
    W = cp._f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    return cp.LinearSpec(name, W, cp._f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32) * 0.01))


def test_scan_targets_by_name_and_shape():
    layers = [_spec("blocks.0.norm1.linear", 256, 1536), _spec("blocks.0.attn.to_qkv", 512, 1536),
              _spec("blocks.0.ff.net.2", 2048, 512), _spec("blocks.0.attn.to_out.0", 320, 512),
              _spec("blocks.0.attn.to_k", 512, 100), _spec("blocks.0.attn.to_v", 100, 64),
              _spec("pos_embed.proj", 512, 512), _spec("blocks.0.attn.to_q", 512, 32)]
    plans = {p.name: p for p in cp.scan(layers, rank=48, fmt="int4")}
    assert plans["blocks.0.norm1.linear"].kind == cp.AWQ
    assert plans["blocks.0.attn.to_qkv"].kind == cp.SVDQ and plans["blocks.0.attn.to_qkv"].rank == 48
    assert plans["blocks.0.attn.to_qkv"].fmt == "int4"
    assert plans["blocks.0.ff.net.2"].kind == cp.SVDQ
    # K = 320 is no multiple of 256: the W4A4 kernels cannot take it, AWQ can
    assert plans["blocks.0.attn.to_out.0"].kind == cp.AWQ
    # N = 100 is no multiple of 16 -> AWQ; K = 100 fits neither kernel -> bf16
    assert plans["blocks.0.attn.to_k"].kind == cp.AWQ
    assert plans["blocks.0.attn.to_v"].kind == cp.KEEP
    assert plans["pos_embed.proj"].kind == cp.KEEP
    # the rank is clipped to the layer (min(K, N) = 32)
    assert plans["blocks.0.attn.to_q"].kind == cp.SVDQ and plans["blocks.0.attn.to_q"].rank == 32


def test_calibration_statistics():
    x = cp._f32_to_bf16_bits(np.array([[1.0, -3.0], [-2.0, 0.5], [0.25, 2.5]], np.float32))
    x = np.repeat(x, 128, axis=1)  # K = 256
    layers = [_spec("a.attn.to_q", 256, 16), _spec("a.norm.linear", 256, 16)]
    plans = cp.scan(layers, rank=16)
    st = cp.calibrate(plans, {"a.attn.to_q": x, "a.norm.linear": x}, awq_rows=2)
    np.testing.assert_array_equal(st["a.attn.to_q"], np.repeat(np.array([2.0, 3.0], np.float32), 128))
    np.testing.assert_array_equal(st["a.norm.linear"], x[[0, 2]])


def test_pack_round_trip(tmp_path):
    layers, inputs = cp.synthetic_flux_block(tokens=48, width=256)
    layers.append(_spec("final_layer.proj_in", 256, 24))  # kept in bf16
    inputs["final_layer.proj_in"] = inputs[layers[1].name]
    path = str(tmp_path / "block.svdq")
    plans, canon = cp.compress(layers, inputs, path, rank=32, fmt="nvfp4")
    kinds = [p.kind for p in plans]
    assert kinds == [cp.AWQ, cp.SVDQ, cp.SVDQ, cp.SVDQ, cp.SVDQ, cp.KEEP]
    header, back = cp.read_packed(path)
    assert header["version"] == cp.VERSION and len(header["layers"]) == len(layers)
    for name, c in canon.items():
        for f, a in c.items():
            if isinstance(a, np.ndarray):
                np.testing.assert_array_equal(back[name][f], a, err_msg=f"{name}.{f}")
            else:
                assert back[name][f] == a, (name, f)
    np.testing.assert_array_equal(back["final_layer.proj_in"]["W"], layers[-1].W)
    raw = open(path, "rb").read()
    hlen = struct.unpack("<II", raw[8:16])[1]
    base = (16 + hlen + 1023) // 1024 * 1024
    for e in header["layers"]:
        for off, n, dt, shape in e.get("arrays", {}).values():
            assert off % 1024 == 0 and (base + off + n) <= len(raw)
    # the preparation is deterministic: a second run gives the same arrays
    again = cp.quantize(layers, plans, cp.calibrate(plans, inputs))
    for name, c in canon.items():
        for f, a in c.items():
            if isinstance(a, np.ndarray):
                np.testing.assert_array_equal(again[name][f], a, err_msg=f"{name}.{f}")


def test_rejects_foreign_files(tmp_path):
    p = tmp_path / "x.bin"
    p.write_bytes(b"NOTAPACK" + b"\0" * 64)
    with pytest.raises(ValueError):
        cp.read_packed(str(p))
    p.write_bytes(cp.MAGIC + struct.pack("<II", 99, 2) + b"{}")
    with pytest.raises(ValueError):
        cp.read_packed(str(p))
