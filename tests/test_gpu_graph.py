"""CUDA-graph capture of the forward entry points.  Each forward is run eagerly on
a side stream for two inputs, then captured once (its kernels -- programmatic
dependent launches included -- and the workspace control-block reset become
graph nodes), and the graph is replayed after each input has been copied into
the captured input buffer: the output must equal the eager output bit for bit.
Covered: svdq_forward (NVFP4 with a static and with a per-call activation scale,
INT4), svdq_mlp_forward (the fused MLP pair), the awq_w4a16 GEMV and the W8A8
layer."""
import numpy as np
import pytest

import oracle
import workloads as wl
from svdq_cases import GpuLayer, oracle_layer

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


def _bf16(X):
    import torch

    return torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).view(torch.bfloat16).to("cuda:0")


def _inputs(X):
    """The layer's seeded input and a rescaled copy (a different replay input)."""
    return [X, wl.f32_to_bf16_bits(oracle.bf16_to_f32(X) * np.float32(0.37))]


def _check_graph(run, x_dev, y, Xs):
    import torch

    s = torch.cuda.Stream()
    eager = []
    for X in Xs:
        x_dev.copy_(_bf16(X))
        torch.cuda.synchronize()
        run(s)
        s.synchronize()
        eager.append(y.clone())
    x_dev.copy_(_bf16(Xs[0]))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(s)
    for X, ref in zip(Xs, eager):
        x_dev.copy_(_bf16(X))
        y.fill_(float("nan"))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    assert not torch.equal(eager[0].view(torch.int16), eager[1].view(torch.int16))  # the replays saw new inputs
    del g


@pytest.mark.parametrize("fmt,dynamic", [("nvfp4", False), ("nvfp4", True), ("int4", False)])
def test_forward_graph_replay(fmt, dynamic):
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    M, K, N, r = 300, 768, 400, 32
    X, W, b, prep = oracle_layer(wl.small_layer(M, K, N, r, fmt, layer_id=91))
    if dynamic:
        prep = dict(prep)
        prep["g_x"] = 0.0
    gl = GpuLayer(prep)
    x = torch.empty(M, K, dtype=torch.bfloat16, device="cuda:0")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda:0")
    ws = gl.lin.workspace(M)
    _check_graph(lambda s: svdq.svdq_forward(gl.lin.handle, x, M, y, ws, s), x, y, _inputs(X))
    assert gl.status(M) == 0


def test_mlp_forward_graph_replay():
    import torch

    import diffusion_transformer_w4a4_b200 as svdq
    from test_gpu_fused_mlp import _pair

    M, K, N, N2 = 300, 512, 768, 256
    X, p_up, p_dn = _pair(M, K, N, N2, 32, 32, lid=93)
    up, dn = GpuLayer(p_up), GpuLayer(p_dn)
    x = torch.empty(M, K, dtype=torch.bfloat16, device="cuda:0")
    y = torch.empty(M, N2, dtype=torch.bfloat16, device="cuda:0")
    wu, wd = up.lin.workspace(M), dn.lin.workspace(M)
    _check_graph(lambda s: svdq.svdq_mlp_forward(up.lin.handle, dn.lin.handle, x, M, y, wu, wd, s), x, y, _inputs(X))
    assert up.status(M) == 0 and dn.status(M) == 0


def test_awq_graph_replay():
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    M, K, N = 2, 768, 576
    X, W, b = wl.make_layer_inputs(wl.small_layer(M, K, N, 0, wl.AWQ, layer_id=95))
    lin = svdq.AwqLinear(svdq.svdq_awq_prepare(W, b, X), device="cuda:0")
    x = torch.empty(M, K, dtype=torch.bfloat16, device="cuda:0")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda:0")
    _check_graph(lambda s: svdq.svdq_awq_forward(lin.handle, x, M, y, s), x, y, _inputs(X))


def test_w8a8_graph_replay():
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    M, K, N = 300, 768, 400
    X, W, b = wl.make_layer_inputs(wl.small_layer(M, K, N, 0, "nvfp4", layer_id=97))
    prep = oracle.w8a8_prepare(W, b)
    lin = svdq.W8A8Linear(prep["wcodes"], float(prep["s_w"]), prep["bias"], device="cuda:0")
    x = torch.empty(M, K, dtype=torch.bfloat16, device="cuda:0")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda:0")
    ws = lin.workspace(M)
    _check_graph(lambda s: svdq.svdq_w8a8_forward(lin.handle, x, M, y, ws, s), x, y, _inputs(X))
