"""A packed checkpoint from the compression tool, loaded onto the device: every
svdq_w4a4 and awq_w4a16 layer it creates gives the same output, bit for bit, as
a layer built directly from the canonical arrays the tool prepared, on the
layer's own calibration input, and reports no device error."""
import numpy as np
import pytest

from diffusion_transformer_w4a4_b200 import compress as cp

pytestmark = pytest.mark.gpu


def test_load_packed_synthetic_block(tmp_path):
    import torch

    import diffusion_transformer_w4a4_b200 as svdq
    from diffusion_transformer_w4a4_b200 import build

    build.build()
    torch.cuda.set_device(0)
    layers, inputs = cp.synthetic_flux_block(tokens=300, width=512)
    path = str(tmp_path / "block.svdq")
    plans, canon = cp.compress(layers, inputs, path, rank=32, fmt="nvfp4")
    loaded = cp.load(path, device="cuda:0")
    for p in plans:
        x = torch.from_numpy(np.ascontiguousarray(inputs[p.name]).view(np.int16)).view(torch.bfloat16).to("cuda:0")
        if p.kind == cp.SVDQ:
            ref = svdq.SvdqLinear(canon[p.name], device="cuda:0")
        elif p.kind == cp.AWQ:
            ref = svdq.AwqLinear(canon[p.name], device="cuda:0")
        else:
            assert loaded[p.name] is None
            continue
        y = loaded[p.name](x)
        y_ref = ref(x)
        torch.cuda.synchronize()
        M = x.shape[0]
        assert (loaded[p.name].status(M) if p.kind == cp.SVDQ else loaded[p.name].status()) == 0
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), p.name
        assert torch.isfinite(y.float()).all()
