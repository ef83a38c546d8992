"""GPU parity of the INT8 tensorwise W8A8 layer through the C ABI.

Bar: the activation scale s_x and every int8 activation code bit-exact against
the oracle; bf16 Y within rel-L2 1e-3 and, elementwise, one bf16 ulp plus the
binary32 error of the epilogue (the int32 accumulator converted to binary32,
the product of the two scales and the fused multiply-add: 4 * 2^-24 of
|s_x s_w acc|).  Small shapes span several tiles and ragged tails; the FLUX MLP
shapes are checked on every code and on sampled output rows."""
import numpy as np
import pytest

import oracle
import workloads as wl
from svdq_cases import tile_rows

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


def _layer(M, K, N, layer_id):
    import diffusion_transformer_w4a4_b200 as svdq

    layer = wl.small_layer(M, K, N, 0, "nvfp4", layer_id=layer_id)
    X, W, b = wl.make_layer_inputs(layer)
    prep = oracle.w8a8_prepare(W, b)
    lin = svdq.W8A8Linear(prep["wcodes"], float(prep["s_w"]), prep["bias"], device="cuda:0")
    return X, prep, lin


def _run(lin, X):
    import torch

    x = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).view(torch.bfloat16).to("cuda:0")
    y = lin.forward(x)
    torch.cuda.synchronize()
    return y.view(torch.int16).cpu().numpy().view(np.uint16)


def _check_y(y, act, prep, rows=None):
    sub = act if rows is None else dict(codes=act["codes"][rows], s_x=act["s_x"])
    ref, yd = oracle.w8a8_forward_from_act(sub, prep, want_f64=True)
    g = oracle.bf16_to_f32(y if rows is None else y[rows]).astype(np.float64)
    o = oracle.bf16_to_f32(ref).astype(np.float64)
    acc = np.abs(sub["codes"].astype(np.int64) @ prep["wcodes"].astype(np.int64).T).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(o), 2.0 ** -133))) - 7)
    bound = ulp + 4 * 2.0 ** -24 * float(act["s_x"]) * float(prep["s_w"]) * acc
    d = np.abs(g - o)
    assert np.all(np.isfinite(g))
    rel = float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30))
    assert rel <= 1e-3, rel
    assert np.all(d <= bound), float(np.max(d - bound))
    return dict(rel_l2=rel, n_flip=int(np.sum((y if rows is None else y[rows]) != ref)))


@pytest.mark.parametrize("M,K,N", [(1, 128, 8), (37, 256, 264), (300, 768, 520), (128, 1024, 256),
                                   (513, 2048, 1032), (260, 384, 2048)])
def test_w8a8_parity(M, K, N):
    X, prep, lin = _layer(M, K, N, layer_id=5 * M + N)
    y = _run(lin, X)
    assert lin.status(M) == 0
    got = lin.read_act(M)
    ref = oracle.w8a8_quantize_act(X)
    assert got["s_x"] == ref["s_x"]
    np.testing.assert_array_equal(got["codes"], ref["codes"])
    print(M, K, N, _check_y(y, ref, prep))


@pytest.mark.parametrize("K,N", [(3072, 12288), (12288, 3072)])
def test_w8a8_flux_mlp_sampled_rows(K, N):
    M = 4608
    X, prep, lin = _layer(M, K, N, layer_id=K)
    y = _run(lin, X)
    assert lin.status(M) == 0
    got = lin.read_act(M)
    ref = oracle.w8a8_quantize_act(X)
    assert got["s_x"] == ref["s_x"]
    np.testing.assert_array_equal(got["codes"], ref["codes"])
    rows = tile_rows(M, 9)
    print(K, N, _check_y(y, ref, prep, rows))


def test_w8a8_zero_input_and_empty():
    import torch

    X, prep, lin = _layer(64, 256, 128, layer_id=1)
    y = _run(lin, np.zeros_like(X))
    assert lin.status(64) == 0
    np.testing.assert_array_equal(y, np.tile(prep["bias"], (64, 1)))
    x0 = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda:0")
    assert lin.forward(x0).shape == (0, 128)


def test_w8a8_wait_timeout_reports_status():
    """A one-cycle wait limit makes the GEMM give up on its first unsatisfied
    wait; it must report SVDQ_ERR_TIMEOUT and leave the context usable."""
    import diffusion_transformer_w4a4_b200 as svdq

    X, prep, lin = _layer(512, 1024, 768, layer_id=77)
    try:
        svdq.svdq_set_wait_limit(1)
        _run(lin, X)
        st = lin.status(512)
    finally:
        svdq.svdq_set_wait_limit(0)
    assert st == svdq.SVDQ_ERR_TIMEOUT
    y = _run(lin, X)  # the quantizer resets the status word
    assert lin.status(512) == 0
    _check_y(y, oracle.w8a8_quantize_act(X), prep)
