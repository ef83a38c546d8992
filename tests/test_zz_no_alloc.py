"""svdq_forward_noalloc: the forward for callers that cannot allocate device
memory (its scratch is a fixed library-owned device array).  Checked through
the C ABI against svdq_forward with a caller workspace, on two calls in a row:
the same kernels run on the same inputs, so the outputs must agree bit for bit.
Also covered: a dynamic-scale NVFP4 layer (g_x = 0, whose first pass leaves its
per-CTA maxima and g_x in the scratch's control block), the status word of the
scratch read through svdq_read_status with a null workspace, and a forced wait
timeout recorded there.  This file is collected last on purpose."""
import numpy as np
import pytest

import workloads as wl
from svdq_cases import GpuLayer, oracle_layer

pytestmark = pytest.mark.gpu


def _setup():
    import torch

    from diffusion_transformer_w4a4_b200 import build

    build.build()
    torch.cuda.set_device(0)


def _layer(fmt, dynamic=False):
    layer = wl.small_layer(300, 1024, 576, 32, fmt, layer_id=41)
    X, W, b, prep = oracle_layer(layer)
    if dynamic:
        prep = dict(prep)
        prep["g_x"] = 0.0
        X = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(X) * np.float32(3.7))  # away from the calibration
    return X, GpuLayer(prep)


@pytest.mark.parametrize("fmt,dynamic", [("nvfp4", False), ("int4", False), ("nvfp4", True)],
                         ids=["nvfp4", "int4", "nvfp4_dynamic"])
def test_forward_noalloc_matches_forward(fmt, dynamic):
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    _setup()
    X, gl = _layer(fmt, dynamic)
    y_ref = gl.forward(X)  # svdq_forward with a caller-owned workspace
    assert gl.status(300) == 0
    x = gl.x_dev(X)
    for _ in range(2):
        y = torch.full((300, 576), float("nan"), dtype=torch.bfloat16, device="cuda:0")
        svdq.svdq_forward_noalloc(gl.lin.handle, x, 300, y)
        torch.cuda.synchronize()
        assert svdq.svdq_read_status(gl.lin.handle, 300, None) == 0
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, y_ref)
    # beyond the fixed scratch: a clear argument error, nothing launched
    for big in (1 << 20, (1 << 30) + 1, 1 << 40):
        with pytest.raises(svdq.SvdqError) as e:
            svdq.svdq_forward_noalloc(gl.lin.handle, x, big, y)
        assert e.value.status == svdq.SVDQ_ERR_INVALID_ARG


def test_forward_noalloc_reports_a_timeout():
    """A one-cycle wait limit makes the kernels give up; the timeout lands in the
    scratch's status word, readable with a null workspace, and the next call
    (which zeroes the control block) is correct again."""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    _setup()
    X, gl = _layer("nvfp4")
    y_ref = gl.forward(X)
    x = gl.x_dev(X)
    y = torch.empty(300, 576, dtype=torch.bfloat16, device="cuda:0")
    try:
        svdq.svdq_set_wait_limit(1)
        svdq.svdq_forward_noalloc(gl.lin.handle, x, 300, y)
        torch.cuda.synchronize()
        st = svdq.svdq_read_status(gl.lin.handle, 300, None)
    finally:
        svdq.svdq_set_wait_limit(0)
    assert st == svdq.SVDQ_ERR_TIMEOUT
    svdq.svdq_forward_noalloc(gl.lin.handle, x, 300, y)
    torch.cuda.synchronize()
    assert svdq.svdq_read_status(gl.lin.handle, 300, None) == 0
    np.testing.assert_array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), y_ref)
