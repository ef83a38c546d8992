"""svdq_forward_noalloc: the forward for callers that cannot allocate device
memory (its scratch is a fixed library-owned device array).  Checked through
the C ABI against svdq_forward with a caller workspace, on two calls in a row.
This file is collected last on purpose."""
import numpy as np
import pytest

import oracle
import workloads as wl
from svdq_cases import GpuLayer, assert_y_close, oracle_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_forward_noalloc_matches_forward(fmt):
    import torch

    import diffusion_transformer_w4a4_b200 as svdq
    from diffusion_transformer_w4a4_b200 import build

    build.build()
    torch.cuda.set_device(0)
    layer = wl.small_layer(300, 1024, 576, 32, fmt, layer_id=41)
    X, W, b, prep = oracle_layer(layer)
    gl = GpuLayer(prep)
    y_ref = gl.forward(X)  # svdq_forward with a caller-owned workspace
    x = gl.x_dev(X)
    for _ in range(2):
        y = torch.full((300, 576), float("nan"), dtype=torch.bfloat16, device="cuda:0")
        svdq.svdq_forward_noalloc(gl.lin.handle, x, 300, y)
        torch.cuda.synchronize()
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        assert_y_close(got, y_ref)
    # beyond the fixed scratch: a clear argument error, nothing launched
    big = 1 << 20
    with pytest.raises(svdq.SvdqError) as e:
        svdq.svdq_forward_noalloc(gl.lin.handle, x, big, y)
    assert e.value.status == svdq.SVDQ_ERR_INVALID_ARG
