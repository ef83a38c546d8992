"""GPU parity of the CUDA path against the oracle, through the C ABI.

Bar: activation codes and scales bit-exact; t within one bf16 ulp; bf16 Y within
rel-L2 1e-3 and |dy| <= 2e-2 + 1 bf16 ulp (see svdq_cases).  Small shapes span
several tiles and ragged tails; the FLUX-sized workloads are checked on all
quantized activations and on sampled output rows."""
import numpy as np
import pytest

import oracle
import workloads as wl
from svdq_cases import GpuLayer, assert_t_close, check_layer_output, oracle_layer, tile_rows

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


def _check_act(gl, X, prep):
    got = gl.quantize(X)
    ref = oracle.quantize_act(X, prep)
    np.testing.assert_array_equal(got["codes"], ref["codes"])
    np.testing.assert_array_equal(got["scales"], ref["scales"])
    if prep["rank"]:
        assert_t_close(got["t"], ref["t"], ref, prep)
    return ref


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
@pytest.mark.parametrize("M,K,N,rank", [(1, 256, 192, 16), (37, 512, 400, 32), (300, 768, 576, 48),
                                        (128, 1024, 384, 0), (160, 512, 256, 128), (257, 256, 208, 64)])
def test_quantize_parity(fmt, M, K, N, rank):
    layer = wl.small_layer(M, K, N, rank, fmt, layer_id=M + K)
    X, W, b, prep = oracle_layer(layer)
    _check_act(GpuLayer(prep), X, prep)


@pytest.mark.parametrize("M,K,N,rank", [(128, 256, 192, 0), (128, 256, 192, 16), (300, 1024, 576, 32),
                                        (77, 512, 400, 48), (256, 768, 208, 128), (1, 256, 384, 32),
                                        (513, 2048, 1152, 64)])
def test_forward_nvfp4(M, K, N, rank):
    layer = wl.small_layer(M, K, N, rank, "nvfp4", layer_id=7 + M)
    X, W, b, prep = oracle_layer(layer)
    gl = GpuLayer(prep)
    y = gl.forward(X)
    assert gl.status(M) == 0
    print(M, K, N, rank, check_layer_output(gl, X, prep, y))


def test_forward_empty_and_reuse():
    layer = wl.small_layer(64, 256, 192, 16, "nvfp4")
    X, W, b, prep = oracle_layer(layer)
    gl = GpuLayer(prep)
    import torch

    y = gl.lin.forward(gl.x_dev(X[:0]))
    torch.cuda.synchronize()
    assert y.shape == (0, 192)
    # repeated calls on one workspace give identical results
    y1, y2 = gl.forward(X), gl.forward(X)
    np.testing.assert_array_equal(y1, y2)


@pytest.mark.parametrize("name", ["c2", "c3_nvfp4", "c4up_nvfp4", "c4dn_nvfp4"])
def test_flux_workloads_nvfp4(name):
    layers = {l.name: l for ls in wl.WORKLOADS.values() for l in ls}
    layer = layers[name]
    X, W, b, prep = oracle_layer(layer)
    gl = GpuLayer(prep)
    M = layer.M
    y = gl.forward(X)
    assert gl.status(M) == 0
    # every quantized activation bit-exact, t within its bound, sampled output rows
    print(name, check_layer_output(gl, X, prep, y, tile_rows(M, 1)))


def test_wait_timeout_reports_status():
    """A one-cycle wait limit makes the kernels give up on their first wait that
    is not already satisfied; they must report SVDQ_ERR_TIMEOUT, free what they
    hold and return, leaving the context usable."""
    import diffusion_transformer_w4a4_b200 as svdq

    layer = wl.small_layer(512, 1024, 768, 32, "nvfp4", layer_id=99)
    X, W, b, prep = oracle_layer(layer)
    gl = GpuLayer(prep)
    try:
        svdq.svdq_set_wait_limit(1)
        gl.forward(X)
        st = gl.status(512)
    finally:
        svdq.svdq_set_wait_limit(0)
    assert st == svdq.SVDQ_ERR_TIMEOUT
    import torch

    svdq.svdq_workspace_init(gl.lin.handle, 512, gl.lin.workspace(512))
    y = gl.forward(X)
    assert gl.status(512) == 0
    check_layer_output(gl, X, prep, y)


@pytest.mark.parametrize("M,K,N,rank", [(128, 256, 128, 0), (128, 256, 128, 16), (300, 1024, 576, 32),
                                        (77, 512, 400, 48), (256, 768, 208, 128), (1, 256, 384, 32)])
def test_forward_int4(M, K, N, rank):
    layer = wl.small_layer(M, K, N, rank, "int4", layer_id=11 + M)
    X, W, b, prep = oracle_layer(layer)
    gl = GpuLayer(prep)
    y = gl.forward(X)
    assert gl.status(M) == 0
    print(M, K, N, rank, check_layer_output(gl, X, prep, y))


@pytest.mark.parametrize("M,K,N", [(128, 256, 128), (300, 512, 400), (64, 1024, 256)])
def test_int4_group_accumulators_exact(M, K, N):
    """The int32 per-group accumulators of the INT4 GEMM equal the integer
    triple loop bit for bit."""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    layer = wl.small_layer(M, K, N, 16, "int4", layer_id=3 + M)
    X, W, b, prep = oracle_layer(layer)
    gl = GpuLayer(prep)
    act = gl.quantize(X)
    acc = torch.zeros(K // 64, M, N, dtype=torch.int32, device="cuda:0")
    svdq.svdq_int4_group_acc(gl.lin.handle, M, gl.lin.workspace(M), acc)
    torch.cuda.synchronize()
    assert gl.status(M) == 0
    ref = oracle.int4_group_acc(act["codes"], prep["wcodes"])
    np.testing.assert_array_equal(acc.cpu().numpy(), ref)


@pytest.mark.parametrize("name", ["c1", "c3_int4", "c4up_int4", "c4dn_int4"])
def test_flux_workloads_int4(name):
    layers = {l.name: l for ls in wl.WORKLOADS.values() for l in ls}
    layer = layers[name]
    X, W, b, prep = oracle_layer(layer)
    gl = GpuLayer(prep)
    M = layer.M
    y = gl.forward(X)
    assert gl.status(M) == 0
    print(name, check_layer_output(gl, X, prep, y, tile_rows(M, 2)))
