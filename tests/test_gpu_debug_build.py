"""The bounds-checked debug variant on the GPU: run in a child process with
SVDQ_LIBRARY=debug, the NVFP4 (one and several 128-row tiles), INT4 and
fused-MLP forwards at ragged shapes report no bounds error (status 0) and give
outputs bit-identical to the release library's."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys, numpy as np, torch
sys.path.insert(0, ROOT); sys.path.insert(0, os.path.join(ROOT, "tests"))
import workloads as wl
import diffusion_transformer_w4a4_b200 as svdq
from svdq_cases import GpuLayer, oracle_layer
torch.cuda.set_device(0)
out = {"debug": svdq.svdq_debug_build()}
for name, (M, K, N, r, fmt) in {"nvfp4_small": (100, 512, 400, 32, "nvfp4"), "nvfp4_multi": (300, 1024, 576, 48, "nvfp4"),
                                "int4": (300, 512, 400, 32, "int4")}.items():
    X, W, b, prep = oracle_layer(wl.small_layer(M, K, N, r, fmt, layer_id=M + K))
    gl = GpuLayer(prep)
    out[name] = gl.forward(X)
    out[name + "_status"] = gl.status(M)
X, W, b, p_up = oracle_layer(wl.small_layer(300, 512, 768, 32, "nvfp4", layer_id=61))
_, W2, b2, p_dn = oracle_layer(wl.small_layer(300, 768, 256, 32, "nvfp4", layer_id=62, gelu=True))
up, dn = GpuLayer(p_up), GpuLayer(p_dn)
y = torch.empty(300, 256, dtype=torch.bfloat16, device="cuda:0")
svdq.svdq_mlp_forward(up.lin.handle, dn.lin.handle, up.x_dev(X), 300, y, up.lin.workspace(300), dn.lin.workspace(300))
torch.cuda.synchronize()
out["fused"] = y.view(torch.int16).cpu().numpy().view(np.uint16)
out["fused_status"] = up.status(300) | dn.status(300)
np.savez(sys.argv[1], **out)
'''


def _run(tmp_path, variant):
    path = str(tmp_path / f"{variant}.npz")
    env = dict(os.environ, SVDQ_LIBRARY=variant)
    r = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT)), path], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    return dict(np.load(path))


def test_debug_variant_matches_release(tmp_path):
    from diffusion_transformer_w4a4_b200 import build

    build.build()
    build.build(debug=True)
    rel = _run(tmp_path, "release")
    dbg = _run(tmp_path, "debug")
    assert int(rel["debug"]) == 0 and int(dbg["debug"]) == 1
    for k in ("nvfp4_small", "nvfp4_multi", "int4", "fused"):
        assert int(dbg[k + "_status"]) == 0, (k, int(dbg[k + "_status"]))
        assert int(rel[k + "_status"]) == 0, k
        np.testing.assert_array_equal(dbg[k], rel[k], err_msg=k)
