"""GPU parity of the dynamic per-tensor NVFP4 activation scale (layers prepared
with g_x = 0: a first pass takes the tensor's largest |x^|, the quantizer derives
g_x from it, stores t / g_x, and the GEMM scales by g_x g_w).

The inputs are the calibration inputs times a factor that is not a power of
two, so the per-call scale differs from the one calibration would give.  Bar:
g_x, activation codes and scales bit-exact; t within its bound; bf16 Y within
the gate of svdq_cases.check_layer_output (sampled rows, one per 128-row tile,
at the FLUX-sized shape)."""
import numpy as np
import pytest

import oracle
import workloads as wl
from svdq_cases import GpuLayer, check_layer_output, oracle_layer, tile_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    import torch

    import diffusion_transformer_w4a4_b200 as svdq
    from diffusion_transformer_w4a4_b200 import build

    build.build()
    assert torch.cuda.is_available()
    assert svdq.svdq_device_check(0) == svdq.SVDQ_OK, "needs an sm_100a device"
    torch.cuda.set_device(0)


def _dynamic_case(layer, factor):
    X, W, b, prep = oracle_layer(layer)
    dyn = dict(prep)
    dyn["g_x"] = 0.0
    Xs = wl.f32_to_bf16_bits(oracle.bf16_to_f32(X) * np.float32(factor))
    return Xs, dyn


@pytest.mark.parametrize("M,K,N,rank,factor", [(1, 256, 192, 16, 3.0), (37, 512, 400, 32, 0.3),
                                               (300, 768, 576, 48, 7.5), (128, 1024, 384, 0, 1.7),
                                               (257, 256, 208, 64, 40.0), (513, 2048, 1152, 128, 0.05)])
def test_dynamic_scale_parity(M, K, N, rank, factor):
    layer = wl.small_layer(M, K, N, rank, "nvfp4", layer_id=3 * M + K)
    X, dyn = _dynamic_case(layer, factor)
    gl = GpuLayer(dyn)
    y = gl.forward(X)
    assert gl.status(M) == 0
    print(M, K, N, rank, factor, check_layer_output(gl, X, dyn, y))


@pytest.mark.parametrize("name,idx", [("c2_nvfp4_1024x3072x3072_r32", 0), ("c4_mlp_4608x3072x12288_r32", 0),
                                      ("c4_mlp_4608x3072x12288_r32", 1)], ids=["c2", "c4_up", "c4_down"])
def test_dynamic_scale_flux_shape_sampled_rows(name, idx):
    layer = wl.WORKLOADS[name][idx]
    X, dyn = _dynamic_case(layer, 6.0)
    gl = GpuLayer(dyn)
    M = layer.M
    y = gl.forward(X)
    assert gl.status(M) == 0
    print(name, idx, check_layer_output(gl, X, dyn, y, tile_rows(M, 3)))


def test_dynamic_scale_follows_the_input_from_call_to_call():
    """One layer, two calls on inputs 2^5 apart: the second call's g_x is 2^5
    times the first one's and its codes and scales are the same."""
    layer = wl.small_layer(200, 512, 256, 32, "nvfp4", layer_id=99)
    X, dyn = _dynamic_case(layer, 1.0)
    gl = GpuLayer(dyn)
    a = gl.quantize(X)
    b = gl.quantize(wl.f32_to_bf16_bits(oracle.bf16_to_f32(X) * np.float32(32.0)))
    assert gl.status(200) == 0
    assert b["g_x"] == 32.0 * a["g_x"]
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["scales"], b["scales"])


def test_dynamic_scale_all_zero_input():
    """max|x^| = 0: g_x = 1, every code and block scale 0, t = 0, and Y = bias."""
    layer = wl.small_layer(130, 512, 256, 32, "nvfp4", layer_id=5)
    X, dyn = _dynamic_case(layer, 1.0)
    X = np.zeros_like(X)
    gl = GpuLayer(dyn)
    y = gl.forward(X)
    assert gl.status(130) == 0
    got = gl.read_act(130)
    assert got["g_x"] == 1.0
    assert not got["codes"].any() and not got["scales"].any() and not got["t"].any()
    np.testing.assert_array_equal(y, oracle.forward(X, dyn))
