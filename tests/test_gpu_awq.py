"""GPU parity of the awq_w4a16 layer (4-bit weights, bf16 activations) against
the oracle, through the C ABI, on the FLUX modulation shapes and on small shapes
with ragged N, several passes over token rows, tiny K and M = 0.

Bar: bf16 Y within rel-L2 1e-3 and, elementwise, 2e-2 + one bf16 ulp of the
oracle value, the same gate as for svdq_w4a4.  On inputs scaled by 2^k away
from the calibration the output scales by 2^k, and so does the absolute part of
the gate (2e-2 * 2^k): the stated max-abs is read in the layer's own units.  The
forward error of binary32 accumulation (K 2^-22 times the sum of |x^| |w|) is
reported as a diagnostic only."""
import numpy as np
import pytest

import oracle
import workloads as wl
from svdq_cases import MAX_ABS, REL_L2, bf16_ulp

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


def _run(layer, x_scale=1.0):
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    X, W, b = wl.make_layer_inputs(layer)
    prep = oracle.awq_prepare(W, b, X)
    if x_scale != 1.0:  # run on inputs far from the calibration ones
        X = wl.f32_to_bf16_bits(oracle.bf16_to_f32(X) * np.float32(x_scale))
    lin = svdq.AwqLinear(dict(N=prep["N"], K=prep["K"], alpha=prep["alpha"], s=prep["s"], inv_s=prep["inv_s"],
                              wcodes=prep["wcodes"], wscales=prep["wscales"], bias=prep["bias"]), device="cuda:0")
    x = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).view(torch.bfloat16).to("cuda:0")
    y = lin.forward(x)
    torch.cuda.synchronize()
    assert lin.status() == 0
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    ref, yd = oracle.awq_forward(X, prep, want_f64=True)
    g, o = oracle.bf16_to_f32(got).astype(np.float64), oracle.bf16_to_f32(ref).astype(np.float64)
    xh = np.abs(oracle.smooth_act(X, prep["inv_s"]).astype(np.float64))
    wabs = np.abs(oracle.dequant(prep["wcodes"], prep["wscales"], oracle.INT4))
    fp32_bound = prep["K"] * 2.0 ** -22 * (xh @ wabs.T)
    bound = MAX_ABS * x_scale + bf16_ulp(o)
    d = np.abs(g - o)
    rel = float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30))
    assert np.all(np.isfinite(g))
    assert rel <= REL_L2, rel
    assert np.all(d <= bound), (int(np.sum(d > bound)), float(np.max(d - bound)))
    used = float(np.max(np.maximum(d - bf16_ulp(o), 0.0) / np.maximum(fp32_bound, 1e-300)))
    return dict(rel_l2=rel, max_abs=float(d.max()), n_flip=int(np.sum(got != ref)), alpha=prep["alpha"],
                max_err_over_fp32_bound=used)


@pytest.mark.parametrize("name", list(wl.AWQ_LAYERS))
def test_awq_flux_modulation(name):
    print(name, _run(wl.AWQ_LAYERS[name]))


@pytest.mark.parametrize("M,K,N", [(1, 64, 16), (3, 448, 130), (9, 1024, 72), (2, 12288, 40), (4, 3072, 517)])
def test_awq_small_shapes(M, K, N):
    print(M, K, N, _run(wl.small_layer(M, K, N, 0, wl.AWQ, layer_id=30 + M)))


def test_awq_empty_and_arguments():
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    layer = wl.small_layer(2, 256, 32, 0, wl.AWQ, layer_id=40)
    X, W, b = wl.make_layer_inputs(layer)
    lin = svdq.AwqLinear(svdq.svdq_awq_prepare(W, b, X), device="cuda:0")
    x = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda:0")
    assert lin.forward(x).shape == (0, 32)  # M = 0 is a no-op
    y = torch.empty(2, 32, dtype=torch.bfloat16, device="cuda:0")
    with pytest.raises(svdq.SvdqError) as e:
        svdq.svdq_awq_forward(lin.handle, None, 2, y)
    assert e.value.status == svdq.SVDQ_ERR_INVALID_ARG


@pytest.mark.parametrize("x_scale", [2.0 ** 60, 2.0 ** -60])
def test_awq_extreme_activation_magnitudes(x_scale):
    """Activations 2^60 above or below the calibration ones (far beyond any real
    layer, inside the kernel's |x^| < 2^113 domain for its pre-scaled decode)."""
    print(x_scale, _run(wl.small_layer(2, 1024, 136, 0, wl.AWQ, layer_id=17), x_scale))
