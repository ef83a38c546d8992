"""GPU parity of the fused MLP pair (up-projection GEMM whose epilogue applies
GELU and quantizes the result as the down-projection's input), through the C ABI.

The fused kernel exports x' = bf16(GELU(bf16(y_up))) on request, so the down
layer is checked teacher-forced on the GPU's own x':
  * x' within one bf16 ulp of the oracle's binary64 GELU of the up layer's
    output as the unfused GPU path computes it (same GEMM arithmetic; GELU in
    binary32 on the GPU, so a rounding boundary may fall either way),
  * the down layer's activation codes and block scales bit-exact against the
    oracle quantizer on x', t' within its summation bound,
  * the down output within rel-L2 1e-3 and |dy| <= 2e-2 + 1 bf16 ulp given the
    GPU's t' (as in svdq_cases.check_layer_output), and within rel-L2 1e-3 of the
    fully independent oracle output,
  * svdq_mlp_forward (no export) bit-identical to the same steps.
Both layers are oracle-prepared; the down layer is calibrated on the dense
bf16 chain's GELU output, as the block tests do."""
import numpy as np
import pytest

import oracle
import workloads as wl
from svdq_cases import GpuLayer, assert_t_close, assert_y_close, bf16_ulp, tile_rows, y_stats

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


def _dense(x_bits, w_bits, b_bits):
    y = oracle.bf16_to_f32(x_bits) @ oracle.bf16_to_f32(w_bits).T + oracle.bf16_to_f32(b_bits)[None, :]
    return oracle.f32_to_bf16(np.ascontiguousarray(y, np.float32))


def _pair(M, K, N, N2, r_up, r_dn, lid, dyn_up=False):
    up = wl.Layer(f"mlp_up_{M}x{K}x{N}", M, K, N, r_up, wl.NVFP4, 0.005, 50.0, False, lid)
    dn = wl.Layer(f"mlp_dn_{M}x{N}x{N2}", M, N, N2, r_dn, wl.NVFP4, 0.0, 1.0, True, lid + 1)
    X, W1, b1 = wl.make_layer_inputs(up)
    W2, b2 = wl.make_w(dn), wl.make_bias(dn)
    p_up = oracle.prepare(W1, b1, oracle.calib_absmax(X), 0.5, r_up, "nvfp4")
    if dyn_up:  # the up layer's activation scale taken per call (g_x = 0), on an input away from calibration
        p_up = dict(p_up)
        p_up["g_x"] = 0.0
        X = wl.f32_to_bf16_bits(oracle.bf16_to_f32(X) * np.float32(3.7))
    h_cal = oracle.gelu_bf16(_dense(X, W1, b1))
    p_dn = oracle.prepare(W2, b2, oracle.calib_absmax(h_cal), 0.5, r_dn, "nvfp4")
    return X, p_up, p_dn


def _run(M, K, N, N2, r_up, r_dn, lid, rows=None, dyn_up=False):
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    X, p_up, p_dn = _pair(M, K, N, N2, r_up, r_dn, lid, dyn_up)
    g_up, g_dn = GpuLayer(p_up), GpuLayer(p_dn)
    assert svdq.svdq_mlp_fusable(g_up.lin.handle, g_dn.lin.handle) == svdq.SVDQ_OK
    x = g_up.x_dev(X)
    ws_up, ws_dn = g_up.lin.workspace(M), g_dn.lin.workspace(M)
    H = torch.empty(M, N, dtype=torch.bfloat16, device="cuda:0")
    y = torch.empty(M, N2, dtype=torch.bfloat16, device="cuda:0")
    svdq.svdq_quantize_act(g_up.lin.handle, x, M, ws_up)
    svdq.svdq_gemm_gelu_quantize(g_up.lin.handle, g_dn.lin.handle, M, ws_up, ws_dn, H)
    svdq.svdq_gemm(g_dn.lin.handle, M, y, ws_dn)
    torch.cuda.synchronize()
    assert g_up.status(M) == 0 and g_dn.status(M) == 0
    act_gpu = g_dn.read_act(M)
    Hb = H.view(torch.int16).cpu().numpy().view(np.uint16)
    y_gpu = y.view(torch.int16).cpu().numpy().view(np.uint16)

    # x' against the binary64 GELU of the unfused GPU path's up output (same GEMM
    # arithmetic; GELU in binary32 on the GPU, so a rounding boundary may fall
    # either way): within one ulp of the larger of the two
    y_up = g_up.forward(X)
    ref_h = oracle.gelu_bf16(y_up)
    hg, hr = oracle.bf16_to_f32(Hb).astype(np.float64), oracle.bf16_to_f32(ref_h).astype(np.float64)
    lim = np.maximum(bf16_ulp(hg), bf16_ulp(hr))
    bad = ~(np.abs(hg - hr) <= lim)
    if bad.any():
        i = np.argwhere(bad)[:5]
        ex = [(float(oracle.bf16_to_f32(y_up[a, b])), float(hg[a, b]), float(hr[a, b])) for a, b in i]
        raise AssertionError(f"{int(bad.sum())} x' elements beyond one ulp; (h, gpu, ref): {ex}")
    n_h_flip = int(np.sum(Hb != ref_h))

    # the down layer, teacher-forced on the GPU's x'
    ref = oracle.quantize_act(Hb, p_dn)
    np.testing.assert_array_equal(act_gpu["codes"], ref["codes"])
    np.testing.assert_array_equal(act_gpu["scales"], ref["scales"])
    st = assert_t_close(act_gpu["t"], ref["t"], ref, p_dn) if r_dn else {}
    rows = np.arange(M) if rows is None else rows
    sub = {k: (v[rows] if np.ndim(v) else v) for k, v in ref.items()}
    taught = dict(sub, t=act_gpu["t"][rows])  # the down layer's low-rank input teacher-forced too
    sy = assert_y_close(y_gpu[rows], oracle.forward_from_act(taught, p_dn), taught, p_dn)
    ind = y_stats(y_gpu[rows], oracle.forward_from_act(sub, p_dn))
    assert ind["rel_l2"] <= 1e-3, ind

    # the one-call form gives the same output bit for bit
    y2 = torch.full((M, N2), float("nan"), dtype=torch.bfloat16, device="cuda:0")
    svdq.svdq_mlp_forward(g_up.lin.handle, g_dn.lin.handle, x, M, y2, ws_up, ws_dn)
    torch.cuda.synchronize()
    assert g_up.status(M) == 0 and g_dn.status(M) == 0
    np.testing.assert_array_equal(y2.view(torch.int16).cpu().numpy().view(np.uint16), y_gpu)
    return dict(sy, h_flips=n_h_flip, **st)


# the up layer's N is the down layer's K: a multiple of 192 (fused tile) and of 256 (K stage)
@pytest.mark.parametrize("M,K,N,N2,r_up,r_dn", [(300, 512, 768, 256, 32, 32), (129, 256, 768, 208, 16, 16),
                                               (513, 768, 1536, 400, 48, 0), (1, 256, 768, 64, 0, 32),
                                               (600, 1024, 1536, 512, 32, 32)])
def test_fused_mlp_small(M, K, N, N2, r_up, r_dn):
    print(M, K, N, N2, r_up, r_dn, _run(M, K, N, N2, r_up, r_dn, lid=M + N))


def test_fused_mlp_dynamic_up_scale():
    """The up layer with a per-call activation scale (its first pass over X, the
    scale read by the fused kernel from the workspace); X scaled by 3.7 away from
    the calibration so the per-call scale differs from a static one."""
    print("dynamic up", _run(300, 512, 768, 256, 32, 32, lid=77, dyn_up=True))


def test_fused_mlp_flux_shape_sampled_rows():
    M = 4608
    print("flux mlp", _run(M, 3072, 12288, 3072, 32, 32, lid=50, rows=tile_rows(M, 5)))


def test_fused_mlp_rejects_unfusable_pairs():
    import diffusion_transformer_w4a4_b200 as svdq

    X, p_up, p_dn = _pair(128, 256, 768, 256, 16, 16, lid=70)
    g_up, g_dn = GpuLayer(p_up), GpuLayer(p_dn)
    assert svdq.svdq_mlp_fusable(g_dn.lin.handle, g_up.lin.handle) == svdq.SVDQ_ERR_INVALID_ARG  # widths differ
    dyn = dict(p_dn)
    dyn["g_x"] = 0.0
    assert svdq.svdq_mlp_fusable(g_up.lin.handle, GpuLayer(dyn).lin.handle) == svdq.SVDQ_ERR_INVALID_ARG
    # more tokens than the per-group counters cover: refused before anything is enqueued
    import torch

    dummy = torch.zeros(1024, dtype=torch.uint8, device="cuda:0")
    with pytest.raises(svdq.SvdqError) as e:
        svdq.svdq_mlp_forward(g_up.lin.handle, g_dn.lin.handle, dummy, 32 * 1024 + 1, dummy, dummy, dummy)
    assert e.value.status == svdq.SVDQ_ERR_INVALID_ARG
