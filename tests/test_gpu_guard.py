"""Guard bands around every buffer the kernels write: the output Y and the
caller workspace are carved out of larger device buffers whose margins hold a
known byte pattern; after a forward at ragged token / feature counts (partial
128-row tiles, partial 192- and 128-column tiles) the margins must be
untouched and Y must equal the forward into an ordinary buffer bit for bit."""
import numpy as np
import pytest

import workloads as wl
from svdq_cases import GpuLayer, oracle_layer

pytestmark = pytest.mark.gpu

PAD = 4096  # bytes on each side (a multiple of 256, so alignment is kept)
PATTERN = 0xA5


def _guarded(torch, nbytes):
    buf = torch.full((nbytes + 2 * PAD,), PATTERN, dtype=torch.uint8, device="cuda:0")
    return buf, buf[PAD:PAD + nbytes]


def _margins_intact(buf, nbytes):
    m = buf.cpu().numpy()
    return bool((m[:PAD] == PATTERN).all() and (m[PAD + nbytes:] == PATTERN).all())


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
@pytest.mark.parametrize("M,K,N,rank", [(300, 512, 400, 32), (129, 768, 208, 16), (513, 256, 592, 48)])
def test_outputs_stay_inside_their_buffers(fmt, M, K, N, rank):
    import torch

    import diffusion_transformer_w4a4_b200 as svdq
    from diffusion_transformer_w4a4_b200 import build

    build.build()
    torch.cuda.set_device(0)
    X, W, b, prep = oracle_layer(wl.small_layer(M, K, N, rank, fmt, layer_id=M + N))
    gl = GpuLayer(prep)
    y_ref = gl.forward(X)
    x = gl.x_dev(X)
    ws_bytes = svdq.svdq_workspace_size(gl.lin.handle, M)
    wbuf, ws = _guarded(torch, ws_bytes)
    svdq.svdq_workspace_init(gl.lin.handle, M, ws)
    ybytes = M * N * 2
    ybuf, yraw = _guarded(torch, ybytes)
    y = yraw.view(torch.bfloat16).view(M, N)
    svdq.svdq_forward(gl.lin.handle, x, M, y, ws)
    torch.cuda.synchronize()
    assert svdq.svdq_read_status(gl.lin.handle, M, ws) == 0
    assert _margins_intact(ybuf, ybytes), "a kernel wrote outside Y"
    assert _margins_intact(wbuf, ws_bytes), "a kernel wrote outside its workspace"
    np.testing.assert_array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), y_ref)
