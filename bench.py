"""Benchmark of the svdq_w4a4 linear layer on B200.

One step = one pass of the whole layer hot path (activation quantizer, then the
W4A4 GEMM with its low-rank/bias epilogue) over the FLUX 1024x1024 MLP pair at
4608 tokens: up-projection 3072 -> 12288 and down-projection 12288 -> 3072,
NVFP4, rank 32, through the C ABI.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU runs are independent replicas (the layer has no exchange step), one
process per GPU, timed on the device, max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "svdq_w4a4 linear TOPS (2*M*N*K per layer) at FLUX shapes"
UNIT = "TOPS"
WORKLOAD = "c4_mlp_4608x3072x12288_r32"
LAYERS = [l for l in wl.WORKLOADS[WORKLOAD] if l.fmt == wl.NVFP4]
FLUSH_BYTES = 256 << 20  # > 126 MB L2


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _traffic(kernel: str, source: str):
    """DRAM bytes per launch from a committed ncu capture, or None once the kernel
    source has changed since the counters were taken."""
    import hashlib

    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    src = os.path.join(ROOT, "diffusion_transformer_w4a4_b200", "csrc", source)
    if not rec or not os.path.exists(src):
        return None
    if hashlib.sha1(open(src, "rb").read()).hexdigest() != rec.get("kernel_source_sha1"):
        return None
    return rec["bytes_per_launch"]


def _layer_flops(l):
    return 2.0 * l.M * l.N * l.K


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        # NCCL between the GPUs; gloo where there is no GPU (the CPU tests of this path)
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def _max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ----------------------------------------------------------------------------- oracle timing
def oracle_sample(prepared, xs, rows: int):
    """Time the oracle (as it stands) on `rows` token rows of each layer."""
    import oracle

    t0 = time.perf_counter()
    flops = 0.0
    for l, prep, X in zip(LAYERS, prepared, xs):
        act = oracle.quantize_act(X[:rows], prep)
        oracle.forward_from_act(act, prep)
        flops += 2.0 * rows * l.N * l.K
    return flops, time.perf_counter() - t0


def _oracle_prep(canon):
    return dict(N=canon["N"], K=canon["K"], rank=canon["rank"], fmt=canon["fmt"], inv_lambda=canon["inv_lambda"],
                L1=canon["L1"], L2=canon["L2"], wcodes=canon["wcodes"], wscales=canon["wscales"],
                bias=canon["bias"], g_x=canon["g_x"], g_w=canon["g_w"])


def cpu_baseline(canons, xs, target_s=15.0):
    import oracle

    preps = [_oracle_prep(c) for c in canons]
    # the oracle has a fixed per-call cost (decoding all weight codes) plus a
    # per-row cost: size the sample from two probes
    _, t2 = oracle_sample(preps, xs, 2)
    _, t18 = oracle_sample(preps, xs, 18)
    per_row = max((t18 - t2) / 16.0, 1e-4)
    rows = int(max(2, min(2048, (target_s - (t2 - 2 * per_row)) / per_row)))
    flops, dt = oracle_sample(preps, xs, rows)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{rows} token rows of each MLP layer (up {LAYERS[0].K}->{LAYERS[0].N}, "
                      f"down {LAYERS[1].K}->{LAYERS[1].N}), NVFP4 r32, quantize + W4A4 product + output, "
                      f"{dt:.1f} s"}


# ----------------------------------------------------------------------------- setup
def _prepare_layers(seed=0):
    """Product-side preparation (C ABI svdq_prepare on the host) of both layers."""
    import diffusion_transformer_w4a4_b200 as svdq

    canons, xs = [], []
    for l in LAYERS:
        X, W, b = wl.make_layer_inputs(l, seed)
        amax = np.abs(wl.bf16_bits_to_f32(X)).max(axis=0).astype(np.float32)
        canons.append(svdq.svdq_prepare(W, b, amax, 0.5, l.rank, l.fmt))
        xs.append(X)
    return canons, xs


def _config(world):
    return {"workload": WORKLOAD + "_nvfp4", "layers": [f"{l.M}x{l.K}->{l.N}" for l in LAYERS],
            "rank": LAYERS[0].rank, "l2": "flushed between steps (256 MiB write)",
            "parallelism": f"replicas x{world}"}


def _oracle_prepare_layers(seed=0):
    """Oracle-side preparation (binary64 SVD, the oracle's own quantizers) of both
    layers, from the same seeded inputs as the product side."""
    import oracle

    preps, xs = [], []
    for l in LAYERS:
        X, W, b = wl.make_layer_inputs(l, seed)
        preps.append(oracle.prepare(W, b, oracle.calib_absmax(X), 0.5, l.rank, l.fmt))
        xs.append(X)
    return preps, xs


def run_reference(args, world, rank):
    """The oracle as it stands, on the host cores, on the bench's workload: each
    step quantizes and multiplies a sample of token rows of both layers, sized
    from two probes so that the oracle's fixed per-call cost (decoding every
    weight code) is amortized and the whole run takes about two minutes."""
    if rank != 0:
        return
    import oracle

    preps, xs = _oracle_prepare_layers()
    _, t2 = oracle_sample(preps, xs, 2)
    _, t34 = oracle_sample(preps, xs, 34)
    per_row = max((t34 - t2) / 32.0, 1e-4)
    fixed = max(t2 - 2 * per_row, 0.0)
    per_step = 120.0 / max(args.steps + args.warmup, 1)
    rows = int(max(32, min(LAYERS[0].M, (per_step - fixed) / per_row)))
    for _ in range(args.warmup):
        oracle_sample(preps, xs, rows)
    tot_f, tot_t = 0.0, 0.0
    for _ in range(args.steps):
        f, t = oracle_sample(preps, xs, rows)
        tot_f += f
        tot_t += t
    val = tot_f / tot_t / 1e12
    sample = (f"{rows} token rows of each MLP layer per step (full layer is {LAYERS[0].M} rows); "
              f"fixed per-call cost {fixed:.2f} s, {per_row * 1e3:.2f} ms per row pair")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(world),
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)


AWQ_LAYER = wl.AWQ_LAYERS["awq_flux_double_mod_2x3072x18432"]
AWQ_SET = 6  # distinct layers, 6 x 30 MB > L2: every launch streams its weights from HBM


def awq_measure(dev, hbm_peak):
    """awq_w4a16 layer at the FLUX double-block modulation shape (2 conditioning rows,
    3072 -> 18432): AWQ_SET distinct layers run back to back from one CUDA graph, so each
    launch reads its own weights from HBM and no host launch gaps enter the timing.
    The kernel's speed does not depend on the weight values, which are seeded random
    codes and scales here."""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    M, K, N = AWQ_LAYER.M, AWQ_LAYER.K, AWQ_LAYER.N
    rng = np.random.default_rng(1234)
    lins = []
    for _ in range(AWQ_SET):
        c = svdq._awq_arrays(N, K)
        c["inv_s"][:] = rng.uniform(0.5, 2.0, K).astype(np.float32)
        c["s"][:] = (1.0 / c["inv_s"].astype(np.float64)).astype(np.float32)
        c["wcodes"][:] = rng.integers(0, 256, c["wcodes"].shape)
        c["wscales"][:] = rng.integers(0x1000, 0x2400, c["wscales"].shape)
        c["bias"][:] = wl.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32) * 0.01)
        lins.append(svdq.AwqLinear(c, device=dev))
    x = torch.from_numpy(wl.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)).view(np.int16))
    x = x.view(torch.bfloat16).to(dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    for lin in lins:
        svdq.svdq_awq_forward(lin.handle, x, M, y)
    torch.cuda.synchronize()
    reps = 10
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):  # the C-ABI call itself is captured (the current stream is the capture stream)
        for _ in range(reps):
            for lin in lins:
                svdq.svdq_awq_forward(lin.handle, x, M, y)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(7):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3 / (reps * AWQ_SET))
    for lin in lins:
        assert lin.status() == 0, "awq kernel reported an error"
    us = statistics.median(ts)
    # algorithmic bytes of one launch: packed codes, fp16 group scales, 1/s, bias, x, y
    nbytes = N * K // 2 + N * (K // 64) * 2 + 4 * K + 4 * N + 2 * M * K + 2 * M * N
    gbs = nbytes / (us * 1e-6) / 1e9
    del graph, lins
    return {"workload": "awq_flux_double_mod_2x3072x18432", "us_per_launch": us, "bound": "hbm",
            "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak, "bytes_per_launch": nbytes,
            "kernel": "k_awq_gemv", "timing": f"CUDA graph of {reps} x {AWQ_SET} distinct layers (weights > L2)",
            "gpu_launches": reps * AWQ_SET}


def dynamic_measure(dev, canons, xs, steps=20):
    """The same two layers with the dynamic per-tensor activation scale (g_x = 0):
    per step, for each layer, the amax pass + quantizer and the GEMM, L2 flushed
    between steps like the main measurement.  The amax pass is HBM-bound (one read
    of X); its cost is the difference of the quantize times."""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    lins = []
    for c in canons:
        d = dict(c)
        d["g_x"] = 0.0
        lins.append(svdq.SvdqLinear(d, device=dev))
    xd = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in xs]
    ys = [torch.empty(l.M, l.N, dtype=torch.bfloat16, device=dev) for l in LAYERS]
    wss = [lin.workspace(l.M) for lin, l in zip(lins, LAYERS)]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps + 3)]
    for k in range(steps + 3):
        flush.zero_()
        for i, (lin, l) in enumerate(zip(lins, LAYERS)):
            evs[k][2 * i].record(stream)
            svdq.svdq_quantize_act(lin.handle, xd[i], l.M, wss[i], sp)
            evs[k][2 * i + 1].record(stream)
            svdq.svdq_gemm(lin.handle, l.M, ys[i], wss[i], sp)
        evs[k][4].record(stream)
    torch.cuda.synchronize()
    for lin, l in zip(lins, LAYERS):
        assert lin.status(l.M) == 0, "kernel reported an error (dynamic scale)"
    ev = evs[3:]
    step = statistics.median([e[0].elapsed_time(e[4]) for e in ev]) * 1e3
    q = statistics.median([e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in ev]) * 1e3
    amax_bytes = sum(2 * l.M * l.K + 4 * l.K for l in LAYERS)
    del lins
    return {"step_us": step, "quantize_with_amax_pass_us": q, "amax_pass_bytes_per_step": amax_bytes,
            "kernels": ["k_act_amax", "k_quantize", "k_gemm_nvfp4"],
            "note": "layers prepared like the main line, then g_x = 0 (per-call scale); "
                    "compare quantize_with_amax_pass_us with per_layer_us.quantize_both"}


def w8a8_measure(dev, xs, steps=20):
    """INT8 tensorwise W8A8 layers at the same FLUX MLP shapes (weights from the
    same seeded generator, prepared by the library): per step, for each layer,
    the max|x| pass + quantizer and the int8 tensor-core GEMM, L2 flushed between
    steps like the main measurement."""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    lins = []
    for l in LAYERS:
        _, W, b = wl.make_layer_inputs(l, 0)
        codes, s_w = svdq.svdq_w8a8_prepare(W)
        lins.append(svdq.W8A8Linear(codes, s_w, b, device=dev))
    xd = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in xs]
    ys = [torch.empty(l.M, l.N, dtype=torch.bfloat16, device=dev) for l in LAYERS]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps + 3)]
    for k in range(steps + 3):
        flush.zero_()
        for i, (lin, l) in enumerate(zip(lins, LAYERS)):
            evs[k][2 * i].record(stream)
            lin.quantize_act(xd[i], l.M)
            evs[k][2 * i + 1].record(stream)
            lin.gemm(l.M, ys[i])
        evs[k][4].record(stream)
    torch.cuda.synchronize()
    for lin, l in zip(lins, LAYERS):
        assert lin.status(l.M) == 0, "w8a8 kernel reported an error"
    ev = evs[3:]
    step = statistics.median([e[0].elapsed_time(e[4]) for e in ev]) * 1e3
    q = statistics.median([e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in ev]) * 1e3
    g = statistics.median([e[1].elapsed_time(e[2]) + e[3].elapsed_time(e[4]) for e in ev]) * 1e3
    flops = sum(2.0 * l.M * l.N * l.K for l in LAYERS)
    _, bf16, _, src = _peaks()
    i8_peak = 2.0 * bf16  # measured bf16 dense x nominal int8:bf16 ratio (4.5 / 2.25)
    gemm_tops = flops / (g * 1e-6) / 1e12
    del lins
    return {"metric": "W8A8 linear TOPS (2*M*N*K per layer)", "value": flops / (step * 1e-6) / 1e12, "unit": "TOPS",
            "step_us": step, "quantize_us": q, "gemm_us": g,
            "gemm_roofline": {"bound": "tensor", "achieved": gemm_tops, "peak": i8_peak, "unit": "TOPS",
                              "frac": gemm_tops / i8_peak, "kernel": "k_gemm_w8a8",
                              "peak_source": f"{src} bf16 {bf16} TFLOP/s (burst) x 2 (nominal int8/bf16)"},
            "gpu_launches": 6 * steps}


def library_fp4_ceiling(dev, ours_us):
    """Context for the GEMM roofline: a black-box library NVFP4 GEMM (cuBLASLt
    through torch._scaled_mm: E2M1 operands with E4M3 block-16 scales, bf16
    output) at the two MLP shapes, seeded random codes, L2 flushed, CUDA events.
    It is not on the product path; `ours_over_library` compares its time with the
    k_gemm_nvfp4 medians of the main line."""
    import torch

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    out = {"library": "cuBLASLt NVFP4 via torch._scaled_mm", "codes": "seeded random"}
    try:
        for key, l in zip(("up", "down"), LAYERS):
            ru = lambda x, m: (x + m - 1) // m * m
            a = torch.randint(0, 256, (l.M, l.K // 2), dtype=torch.uint8, device=dev, generator=g)
            b = torch.randint(0, 256, (l.N, l.K // 2), dtype=torch.uint8, device=dev, generator=g)
            sa = torch.randint(0x30, 0x40, (ru(l.M, 128) * ru(l.K // 16, 4),), dtype=torch.uint8, device=dev,
                               generator=g).view(torch.float8_e4m3fn)
            sb = torch.randint(0x30, 0x40, (ru(l.N, 128) * ru(l.K // 16, 4),), dtype=torch.uint8, device=dev,
                               generator=g).view(torch.float8_e4m3fn)
            af, bf = a.view(torch.float4_e2m1fn_x2), b.view(torch.float4_e2m1fn_x2)
            fn = lambda: torch._scaled_mm(af, bf.t(), sa, sb, out_dtype=torch.bfloat16)
            fn()
            torch.cuda.synchronize()
            ts = []
            for i in range(23):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                if i >= 3:
                    ts.append(e0.elapsed_time(e1) * 1e3)
            us = statistics.median(ts)
            out[key] = {"us": us, "tflops": _layer_flops(l) / (us * 1e-6) / 1e12, "ours_us": ours_us[key],
                        "ours_over_library": us / ours_us[key]}
    except Exception as e:  # the library or its fp4 types missing: context only
        out["unavailable"] = repr(e)[:200]
    del flush
    return out


def fused_mlp_measure(dev, lins, xs, steps=20):
    """The same MLP pair with cross-layer fusion: per step the up layer's
    quantizer, the up GEMM whose epilogue applies GELU and writes the down layer's
    quantized input (codes, scales, t') instead of y_up, and the down GEMM; L2
    flushed between steps like the main line.  (The unfused line's down input is
    its own seeded tensor, so the two lines time the same kernels' work except
    that the fused one also computes the GELU.)"""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    up, dn = lins
    if svdq.svdq_mlp_fusable(up.handle, dn.handle) != svdq.SVDQ_OK:
        return {"unavailable": "layer pair not fusable"}
    l_up, l_dn = LAYERS
    M = l_up.M
    x = torch.from_numpy(xs[0].view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.empty(M, l_dn.N, dtype=torch.bfloat16, device=dev)
    ws_up, ws_dn = up.workspace(M), dn.workspace(M)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps + 3)]
    for e in evs:
        flush.zero_()
        e[0].record(stream)
        svdq.svdq_quantize_act(up.handle, x, M, ws_up, sp)
        e[1].record(stream)
        svdq.svdq_gemm_gelu_quantize(up.handle, dn.handle, M, ws_up, ws_dn, None, sp)
        e[2].record(stream)
        svdq.svdq_gemm(dn.handle, M, y, ws_dn, sp)
        e[3].record(stream)
    torch.cuda.synchronize()
    assert up.status(M) == 0 and dn.status(M) == 0, "kernel reported an error (fused MLP)"
    ev = evs[3:]
    med = lambda a, b: statistics.median([e[a].elapsed_time(e[b]) for e in ev]) * 1e3
    step = med(0, 3)
    flops = sum(_layer_flops(l) for l in LAYERS)
    return {"step_us": step, "quantize_up_us": med(0, 1), "fused_gemm_gelu_quantize_us": med(1, 2),
            "gemm_down_us": med(2, 3), "tops": flops / (step * 1e-6) / 1e12,
            "kernels": ["k_quantize", "k_gemm_gelu_quant", "k_gemm_nvfp4"], "gpu_launches": 3 * steps,
            "note": "compare step_us with ms_per_step of the main line (unfused: two quantizers, two GEMMs)"}


def _random_canonical(N, K, r, fmt, rng):
    """Valid prepared weights with seeded random codes and scales.  The kernels'
    run time does not depend on the weight values, so the per-config timings use
    these instead of a host SVD of every shape (the main line above uses the
    product's own preparation of the seeded FLUX weights)."""
    import diffusion_transformer_w4a4_b200 as svdq

    c = svdq._canonical_arrays(N, K, r, fmt)
    c["inv_lambda"][:] = rng.uniform(0.5, 2.0, K).astype(np.float32)
    c["lambda_"][:] = (1.0 / c["inv_lambda"].astype(np.float64)).astype(np.float32)
    c["L1"][:] = wl.f32_to_bf16_bits(rng.standard_normal((K, r)).astype(np.float32) * 0.05)
    c["L2"][:] = wl.f32_to_bf16_bits(rng.standard_normal((r, N)).astype(np.float32) * 0.05)
    c["wcodes"][:] = rng.integers(0, 256, c["wcodes"].shape)
    if fmt == wl.NVFP4:
        c["wscales"][:] = rng.integers(0x20, 0x60, c["wscales"].shape)
        c["g_x"], c["g_w"] = 2.0 ** -6, 2.0 ** -12
    else:
        c["wscales"][:] = rng.integers(0x1000, 0x2400, c["wscales"].shape)
    c["bias"][:] = wl.f32_to_bf16_bits(rng.standard_normal(N).astype(np.float32) * 0.01)
    return c


def _peak_for(fmt):
    _, bf16, _, src = _peaks()
    if fmt == wl.NVFP4:
        return 4.0 * bf16, f"{src} bf16 {bf16} TFLOP/s (burst) x 4 (nominal fp4/bf16)"
    return 2.0 * bf16, f"{src} bf16 {bf16} TFLOP/s (burst) x 2 (nominal int8/bf16; INT4 runs on 8-bit tensor cores)"


def _time_layer(lin, x, y, M, flush, reps=20):
    """Median quantize / GEMM / layer times (us) with L2 flushed before every rep."""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    ws = lin.workspace(M)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps + 3)]
    for ev in evs:
        flush.zero_()
        ev[0].record(stream)
        svdq.svdq_quantize_act(lin.handle, x, M, ws, sp)
        ev[1].record(stream)
        svdq.svdq_gemm(lin.handle, M, y, ws, sp)
        ev[2].record(stream)
    torch.cuda.synchronize()
    assert lin.status(M) == 0, "kernel reported an error"
    ev = evs[3:]
    q = statistics.median([e[0].elapsed_time(e[1]) for e in ev]) * 1e3
    g = statistics.median([e[1].elapsed_time(e[2]) for e in ev]) * 1e3
    t = statistics.median([e[0].elapsed_time(e[2]) for e in ev]) * 1e3
    return q, g, t


def _graph_times(lin, x, y, M, flush, n=40):
    """us per forward from CUDA graphs: back to back with the weights warm in L2,
    and with an L2 flush before each forward (a graph of flushes alone subtracted)."""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    ws = lin.workspace(M)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graphs = {}
    with torch.cuda.stream(side):
        for kind in ("warm", "cold", "flush"):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                for _ in range(n):
                    if kind != "warm":
                        flush.zero_()
                    if kind != "flush":
                        svdq.svdq_forward(lin.handle, x, M, y, ws, side.cuda_stream)
            graphs[kind] = g
    torch.cuda.current_stream().wait_stream(side)
    out = {}
    for kind, g in graphs.items():
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3 / n)
        out[kind] = statistics.median(ts)
    assert lin.status(M) == 0, "kernel reported an error (graph)"
    del graphs
    return {"graph_warm_l2_us": out["warm"], "graph_cold_l2_us": max(out["cold"] - out["flush"], 0.0)}


def configs_measure(dev):
    """Every other configuration of the workload list, one entry each: the
    128-token INT4 layer and the 1024-token NVFP4 layer (eager with L2 flushed,
    and from CUDA graphs), the FLUX QKV projection and MLP pair in both formats,
    and the batch-2 block's four linears at ranks 16/32/64/128 (NVFP4)."""
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    rng = np.random.default_rng(4321)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    xcache = {}

    def xdev(M, K):
        if (M, K) not in xcache:
            xcache[(M, K)] = torch.randn(M, K, device=dev).to(torch.bfloat16)
        return xcache[(M, K)]

    def one(M, K, N, r, fmt, graphs=False):
        lin = svdq.SvdqLinear(_random_canonical(N, K, r, fmt, rng), device=dev)
        x = xdev(M, K)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        q, g, t = _time_layer(lin, x, y, M, flush)
        peak, src = _peak_for(fmt)
        flops = 2.0 * M * N * K
        e = {"shape": f"{M}x{K}->{N}", "rank": r, "fmt": fmt, "quantize_us": q, "gemm_us": g, "layer_us": t,
             "layer_tops": flops / (t * 1e-6) / 1e12,
             "gemm_roofline": {"bound": "tensor", "achieved": flops / (g * 1e-6) / 1e12, "peak": peak,
                               "unit": "TFLOP/s" if fmt == wl.NVFP4 else "TOPS",
                               "frac": flops / (g * 1e-6) / 1e12 / peak, "peak_source": src}}
        if graphs:
            e.update(_graph_times(lin, x, y, M, flush))
        del lin
        return e

    out = {"timing": "CUDA events, median of 20 with L2 flushed before each; weights are seeded random valid "
                     "codes and scales (run time does not depend on their values); X ~ N(0,1) bf16"}
    out["c1_int4_128x1024x1024_r32"] = one(128, 1024, 1024, 32, wl.INT4, graphs=True)
    out["c2_nvfp4_1024x3072x3072_r32"] = one(1024, 3072, 3072, 32, wl.NVFP4, graphs=True)
    for fmt in (wl.NVFP4, wl.INT4):
        out[f"c3_qkv_4608x3072x9216_r32_{fmt}"] = one(4608, 3072, 9216, 32, fmt)
    up, dn = one(4608, 3072, 12288, 32, wl.INT4), one(4608, 12288, 3072, 32, wl.INT4)
    flops = 2 * 2.0 * 4608 * 3072 * 12288
    peak, src = _peak_for(wl.INT4)
    gsum = up["gemm_us"] + dn["gemm_us"]
    out["c4_mlp_4608x3072x12288_r32_int4"] = {
        "up": up, "down": dn, "step_us": up["layer_us"] + dn["layer_us"],
        "tops": flops / ((up["layer_us"] + dn["layer_us"]) * 1e-6) / 1e12,
        "gemm_roofline": {"bound": "tensor", "achieved": flops / (gsum * 1e-6) / 1e12, "peak": peak, "unit": "TOPS",
                          "frac": flops / (gsum * 1e-6) / 1e12 / peak, "peak_source": src}}
    xcache.clear()
    M = wl.BLOCK_M
    peak, src = _peak_for(wl.NVFP4)
    for r in wl.BLOCK_RANKS:
        lay = {}
        for name, (K, N) in (("qkv", (3072, 9216)), ("out", (3072, 3072)), ("up", (3072, 12288)),
                             ("down", (12288, 3072))):
            lay[name] = one(M, K, N, r, wl.NVFP4)
        tot = sum(v["layer_us"] for v in lay.values())
        gsum = sum(v["gemm_us"] for v in lay.values())
        flops = sum(2.0 * M * int(v["shape"].split("x")[1].split("->")[0]) * int(v["shape"].split("->")[1])
                    for v in lay.values())
        out[f"c5_block_9216_nvfp4_r{r}"] = {
            "linears": lay, "block_us": tot, "tops": flops / (tot * 1e-6) / 1e12,
            "gemm_roofline": {"bound": "tensor", "achieved": flops / (gsum * 1e-6) / 1e12, "peak": peak,
                              "unit": "TFLOP/s", "frac": flops / (gsum * 1e-6) / 1e12 / peak, "peak_source": src}}
        xcache.clear()
    del flush
    return out


def run_ours(args, world, rank, local):
    import torch

    import diffusion_transformer_w4a4_b200 as svdq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    st = svdq.svdq_device_check(local)
    if st != svdq.SVDQ_OK:
        raise SystemExit(svdq.svdq_status_string(st))
    canons, xs = _prepare_layers()
    lins = [svdq.SvdqLinear(c, device=dev) for c in canons]
    xd = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev) for x in xs]
    ys = [torch.empty(l.M, l.N, dtype=torch.bfloat16, device=dev) for l in LAYERS]
    wss = [lin.workspace(l.M) for lin, l in zip(lins, LAYERS)]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    def step(ev=None):
        for i, (lin, l) in enumerate(zip(lins, LAYERS)):
            if ev is not None:
                ev[2 * i].record(stream)
            svdq.svdq_quantize_act(lin.handle, xd[i], l.M, wss[i], sp)
            if ev is not None:
                ev[2 * i + 1].record(stream)
            svdq.svdq_gemm(lin.handle, l.M, ys[i], wss[i], sp)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    for lin, l in zip(lins, LAYERS):
        assert lin.status(l.M) == 0, "kernel reported an error during warm-up"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for k in range(args.steps):
            flush.zero_()  # L2 flush between timed steps (outside the events)
            step(evs[k])
        torch.cuda.synchronize()
    _barrier(world)
    step_ms = [e[0].elapsed_time(e[4]) for e in evs]
    q_ms = [e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in evs]
    g_ms = [e[1].elapsed_time(e[2]) + e[3].elapsed_time(e[4]) for e in evs]
    g_up = [e[1].elapsed_time(e[2]) for e in evs]
    g_dn = [e[3].elapsed_time(e[4]) for e in evs]
    total_ms = _max_over_ranks(sum(step_ms), world)
    for lin, l in zip(lins, LAYERS):
        assert lin.status(l.M) == 0, "kernel reported an error during timing"

    flops_step = sum(_layer_flops(l) for l in LAYERS)
    value = world * flops_step * args.steps / (total_ms * 1e-3) / 1e12

    # roofline of the dominant kernel (the NVFP4 GEMM), tensor-bound
    hbm, bf16, bf16_sus, src = _peaks()
    fp4_peak = bf16 * 4.0  # measured bf16 dense x nominal fp4:bf16 ratio (9 / 2.25)
    g_avg_ms = statistics.mean(g_ms) / 2
    achieved = flops_step / 2 / (g_avg_ms * 1e-3) / 1e12
    traffic = _traffic("gemm_nvfp4", "gemm_nvfp4.cu")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": achieved / fp4_peak, "traffic": traffic,
                "peak_source": f"{src} bf16 {bf16} TFLOP/s (burst) x 4 (nominal fp4/bf16)",
                "kernel": "k_gemm_nvfp4", "flops_per_launch": flops_step / 2,
                "traffic_note": "DRAM bytes of the up-projection launch (ncu); achieved averages both launches"}
    # the activation quantizer is HBM-bound: algorithmic bytes per launch
    qbytes = 0.0
    for l in LAYERS:
        qbytes += 2 * l.M * l.K + l.M * l.K / 2 + l.M * l.K / 16 + 2 * l.M * l.rank + 2 * l.K * l.rank + 4 * l.K
    q_avg_ms = statistics.mean(q_ms)
    quant = {"bound": "hbm", "achieved": qbytes / (q_avg_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
             "frac": qbytes / (q_avg_ms * 1e-3) / 1e9 / hbm, "bytes_per_step": qbytes, "kernel": "k_quantize"}

    # end to end through the C ABI with host buffers: H2D of X, forward, D2H of Y.
    # The copies run on their own streams and the device buffers alternate
    # between steps, so step k's upload, step k-1's forward and step k-2's
    # download overlap (both PCIe directions at once), as a serving loop would.
    xh = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in xs]
    yh = [[torch.empty(l.M, l.N, dtype=torch.bfloat16).pin_memory() for l in LAYERS] for _ in range(2)]
    xdb = [xd, [torch.empty_like(t) for t in xd]]
    ysb = [ys, [torch.empty_like(t) for t in ys]]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_run(n):
        done_fwd = [[None] * len(LAYERS) for _ in range(2)]  # forward that last read buffer b
        done_out = [[None] * len(LAYERS) for _ in range(2)]  # download that last read buffer b
        for k in range(n):
            b = k % 2
            for i, (lin, l) in enumerate(zip(lins, LAYERS)):
                with torch.cuda.stream(s_in):
                    if done_fwd[b][i] is not None:
                        s_in.wait_event(done_fwd[b][i])
                    xdb[b][i].copy_(xh[i], non_blocking=True)
                    ready = torch.cuda.Event()
                    ready.record(s_in)
                stream.wait_event(ready)
                if done_out[b][i] is not None:
                    stream.wait_event(done_out[b][i])
                svdq.svdq_forward(lin.handle, xdb[b][i], l.M, ysb[b][i], wss[i], sp)
                fwd = torch.cuda.Event()
                fwd.record(stream)
                done_fwd[b][i] = fwd
                with torch.cuda.stream(s_out):
                    s_out.wait_event(fwd)
                    yh[b][i].copy_(ysb[b][i], non_blocking=True)
                    out = torch.cuda.Event()
                    out.record(s_out)
                done_out[b][i] = out
        return [e for row in done_out for e in row if e is not None]

    for e in e2e_run(2):
        e.synchronize()
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for e in e2e_run(e2e_steps):
        stream.wait_event(e)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), world)
    h2d = sum(2 * l.M * l.K for l in LAYERS)
    d2h = sum(2 * l.M * l.N for l in LAYERS)
    e2e = {"value": world * flops_step * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales) + bf16 low-rank, f32 accumulate", "data": "synthetic",
        "config": _config(world),
        "roofline": roofline, "quantize_roofline": quant,
        "per_layer_us": {"gemm_up": statistics.median(g_up) * 1e3, "gemm_down": statistics.median(g_dn) * 1e3,
                         "quantize_both": statistics.median(q_ms) * 1e3,
                         "step_p10_p50_p90": [float(np.percentile(step_ms, p)) * 1e3 for p in (10, 50, 90)]},
        "e2e": e2e, "gpu_launches": 4 * args.steps, "clocks": clk.summary(),
    }
    out["awq_w4a16"] = awq_measure(dev, hbm)
    out["dynamic_act_scale"] = dynamic_measure(dev, canons, xs)
    out["w8a8"] = w8a8_measure(dev, xs)
    out["fused_mlp"] = fused_mlp_measure(dev, lins, xs)
    out["library_fp4_ceiling"] = library_fp4_ceiling(
        dev, {"up": statistics.median(g_up) * 1e3, "down": statistics.median(g_dn) * 1e3})
    if not args.no_configs:
        out["configs"] = configs_measure(dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(canons, xs)
    if rank == 0:
        print(json.dumps(out), flush=True)
    del lins


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config timings")
    args = ap.parse_args()
    world, rank, local = _dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
