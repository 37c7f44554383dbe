#!/usr/bin/env python3
"""Benchmark of the fused SVDQuant W4A4 + low-rank linear layer on B200.

One step = the hot path over one FLUX.1 double-block's linears (M = 4608
tokens: attn-out 3072->3072, fused qkv 3072->9216, MLP-up 3072->12288,
MLP-down 12288->3072; rank 32), each layer = activation kernel + GEMM kernel.
The metric is whole-job FP4 GEMM throughput 2*M*N*K / time (TFLOP/s), plus
us per layer.  With torchrun every rank runs its own replica of the step on
its own batch (weak scaling; the layer needs no collective), and the time is
the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

``--impl reference`` times the CPU oracle on a bounded row sample of the
same workload on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import config_cases, make_layer_inputs  # noqa: E402

METRIC = "fused W4A4+low-rank linear TFLOPS & % of FP4 roofline; us/layer on FLUX shapes"
WORKLOAD = "FLUX.1 double-block linears (attn_out, qkv, mlp_up, mlp_down), M=4608, rank 32, NVFP4 g16"
NOMINAL_FP4_OVER_BF16 = 4.0      # dense FP4 : dense BF16 tensor rate (9 : 2.25 PFLOP/s)
FALLBACK_BF16_SUSTAINED = 1400.0
FALLBACK_BF16_BURST = 1590.0
FALLBACK_HBM = 6650.0

SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "hbm": d["hbm_gbs"], "source": "measured"}
    except Exception:
        return {"bf16": FALLBACK_BF16_BURST, "bf16_sustained": FALLBACK_BF16_SUSTAINED,
                "hbm": FALLBACK_HBM, "source": "fallback"}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# step's GEMM (gemm_w4a4_kernel for K = 3072, the CTA-pair gemm_w4a4_pair_kernel
# for K = 12288) on this workload, from one ncu capture, with the SHA-256 of the
# kernel source the counters were taken on; counters of another source are stale
# and not reported.
K2_TRAFFIC = {
    "source_sha256": "9482a6cdf741aef42773aed4d9c3fa2f865809d300b8ffab3cc1fa8a2e20917c",
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum: read + write per launch
    "bytes_per_launch": {"attn_out": 14127616 + 17152, "qkv": 25167872 + 32066816,
                         "mlp_up": 30682624 + 59291392, "mlp_down": 55654144 + 6521344},
}


def k2_traffic_per_launch(names):
    import hashlib
    src = os.path.join(ROOT, "rank_outlier_gemm_b200", "csrc", "gemm_w4a4.cu")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    per = K2_TRAFFIC["bytes_per_launch"]
    if K2_TRAFFIC["source_sha256"] != sha or not all(n in per for n in names):
        return None, "no ncu counters for the current kernel source"
    return (sum(per[n] for n in names) / len(names),
            "mean over the step's launches of dram read+write bytes from one ncu capture")


LAYER_FILTER = None


def flux_cases():
    cs = config_cases("flux")
    if LAYER_FILTER:
        cs = [c for c in cs if c.name in LAYER_FILTER]
    return cs


def layer_bytes(c) -> float:
    """Minimum HBM bytes of one layer: X read, weight codes+scales, Y write."""
    return 2 * c.M * c.K + c.N * c.K * (0.5 + 1 / 16) + 2 * c.M * c.N


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None
        self.gpu = gpu_index

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={SMI_FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        time.sleep(0.15)
        return self

    def __exit__(self, *a):
        if self.p:
            time.sleep(0.15)
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()

    def summary(self):
        try:
            rows = [l.strip().split(",") for l in open(self.f.name) if l.strip()]
            os.unlink(self.f.name)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if len(r) >= 9]
        mx = [float(r[2]) for r in rows if len(r) >= 9]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows if len(r) >= 9 for i in range(4)
                          if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sm)}


# ------------------------------------------------------------------ ranks
def dist_env():
    """(world size, rank, local rank) as a torchrun launch sets them; 1, 0, 0 alone."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (each rank's own device time of the same
    timed region; the slowest rank sets the job's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank_step: float, ms_step: float, world: int) -> float:
    """Whole-job TFLOP/s of independent replicas: every rank's work over the
    slowest rank's step time (weak scaling)."""
    return world * flops_per_rank_step / (ms_step * 1e-3) / 1e12


# ------------------------------------------------------------------ extras
def _time_ms(torch, stream, fn, reps):
    for _ in range(3):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def unfused_overhead(L, torch, layers, stream, ms0, reps):
    """The low-rank branch run unfused (SVDQuant §4.3, Fig. 6: the naive
    implementation): both kernels at rank 0, then T = X L1' and Y += T L2 as two
    separate cuBLAS bf16 GEMMs that re-read X and re-write Y.  Returns its step
    time over the rank-0 step's, minus one."""
    extra = []
    for l in layers:
        ex = L.svdq_weights_export(l["w"])
        dev = l["X"].device
        L1p = torch.from_numpy(ex["L1p"].view(np.int16).copy()).view(torch.bfloat16).to(dev)
        L2 = torch.from_numpy(ex["L2"].view(np.int16).copy()).view(torch.bfloat16).to(dev)
        extra.append((L1p, L2))

    def step_unfused():
        for l, (L1p, L2) in zip(layers, extra):
            xq, xsf, _ = l["bufs"]
            L.svdq_quantize_act_lowrank_down(l["w0"], l["X"], xq, xsf, None)
            L.svdq_linear_w4a4(l["w0"], xq, xsf, None, l["case"].M, l["Y"])
            T = l["X"] @ L1p
            l["Y"].addmm_(T, L2)

    return _time_ms(torch, stream, step_unfused, reps) / ms0 - 1.0


def rank_sweep(L, torch, layers, dev, stream, reps=50):
    """Layer time (both kernels) of the largest step layer at ranks 0, 16, 32,
    32 + a rank-16 LoRA attached without re-quantization, and 64; the
    per-rank overhead is relative to rank 0 (SVDQuant App. E.5 trade-off)."""
    l = max(layers, key=lambda z: z["case"].flops)
    c = l["case"]
    t = make_layer_inputs(c)
    out = {"layer": f"{c.label} M={c.M} K={c.K} N={c.N}", "us": {}, "overhead_vs_rank0": {}}
    handles = {"0": l["w0"], "32": l["w"]}
    for r in (16, 64):
        handles[str(r)] = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=r)
    wl = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=32)
    g = np.random.default_rng(7)
    A = (g.standard_normal((c.K, 16)) * 0.01).astype(np.float32)
    B = (g.standard_normal((16, c.N)) * 0.01).astype(np.float32)
    to_bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    L.svdq_attach_lora(wl, to_bits(A), to_bits(B), 1.0)
    handles["32+lora16"] = wl
    for key, w in handles.items():
        xq, xsf, T = L.act_buffers(w, c.M, dev)

        def one():
            L.svdq_quantize_act_lowrank_down(w, l["X"], xq, xsf, T)
            L.svdq_linear_w4a4(w, xq, xsf, T, c.M, l["Y"])

        out["us"][key] = 1e3 * _time_ms(torch, stream, one, reps)
    for key, us in out["us"].items():
        out["overhead_vs_rank0"][key] = us / out["us"]["0"] - 1.0
    return out


def _graph_us(torch, fn, inner=10, reps=20):
    """Device time of one fn() call, replayed from a CUDA graph of `inner`
    calls (so the host's per-call launch cost is not part of it)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(inner):
            fn()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    return 1e3 * a.elapsed_time(b) / (reps * inner)


def small_m(L, torch, dev, stream, reps=100):
    """The small-M + LoRA configuration (K = 3072, N in {3072, 12288}, M in {1, 16,
    256}, rank 32 + a rank-16 LoRA): layer time (both kernels) and the fraction of
    its HBM floor (weight codes + scales + low-rank factors + X + Y at the measured
    copy bandwidth).  `us` is device time from CUDA-graph replay; `us_eager` is
    back-to-back eager calls from Python, where the host's launch cost shows."""
    hbm = peaks()["hbm"] * 1e9
    out = {}
    for c in config_cases("small_m_lora"):
        t = make_layer_inputs(c)
        w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=c.rank)
        L.svdq_attach_lora(w, t.lora_A_bits, t.lora_B_bits, 1.0)
        X = torch.from_numpy(t.X_bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
        xq, xsf, T = L.act_buffers(w, c.M, dev)

        def one():
            L.svdq_quantize_act_lowrank_down(w, X, xq, xsf, T)
            L.svdq_linear_w4a4(w, xq, xsf, T, c.M, Y)

        us_eager = 1e3 * _time_ms(torch, stream, one, reps)
        us = _graph_us(torch, one)
        r = c.rank + c.lora_rank
        floor = (c.N * c.K * (0.5 + 1 / 16) + 2 * r * (c.K + c.N) + 2 * c.M * (c.K + c.N)) / hbm * 1e6
        out[c.name] = {"us": us, "us_eager": us_eager, "hbm_floor_us": floor, "frac": floor / us}
    return out


def model_layers(L, torch, dev, reps=20):
    """The PixArt-Sigma and SDXL layers at full M (SVDQuant App. B: the evaluated
    models besides FLUX.1), rank 32, library-prepared weights: per layer the
    time of both kernels and of each alone (CUDA-graph replay, so the host's
    launch cost is not part of it), TFLOP/s (2MNK / t), the layer roofline
    max(2MNK / FP4 peak, B_min / HBM) and its fraction, and the low-rank
    overhead against the same kernels at rank 0.  These shapes have short K
    (640-1280 on the input side), so they are HBM-bound."""
    pk = peaks()
    fp4 = pk["bf16"] * NOMINAL_FP4_OVER_BF16
    out = {"fp4_peak_tflops": fp4, "hbm_gbs": pk["hbm"], "layers": {}}
    for cfg in ("pixart", "sdxl"):
        for c in config_cases(cfg):
            t = make_layer_inputs(c)
            X = torch.from_numpy(t.X_bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
            Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
            res = {}
            for r in (c.rank, 0):
                w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=r)
                xq, xsf, T = L.act_buffers(w, c.M, dev)

                def layer():
                    L.svdq_quantize_act_lowrank_down(w, X, xq, xsf, T)
                    L.svdq_linear_w4a4(w, xq, xsf, T, c.M, Y)

                res[r] = _graph_us(torch, layer, inner=10, reps=reps)
                if r == c.rank:
                    res["act"] = _graph_us(torch, lambda: L.svdq_quantize_act_lowrank_down(w, X, xq, xsf, T),
                                           inner=10, reps=reps)
                    res["gemm"] = _graph_us(torch, lambda: L.svdq_linear_w4a4(w, xq, xsf, T, c.M, Y),
                                            inner=10, reps=reps)
                del w, xq, xsf, T
            roof = max(c.flops / (fp4 * 1e12), layer_bytes(c) / (pk["hbm"] * 1e9)) * 1e6
            us = res[c.rank]
            out["layers"][c.label] = {
                "M": c.M, "K": c.K, "N": c.N, "us": us, "us_act_kernel": res["act"], "us_gemm_kernel": res["gemm"],
                "tflops": c.flops / (us * 1e-6) / 1e12, "roofline_us": roof, "frac_of_layer_roofline": roof / us,
                "bound": "tensor" if c.flops / (fp4 * 1e12) > layer_bytes(c) / (pk["hbm"] * 1e9) else "hbm",
                "us_rank0": res[0], "lowrank_overhead_vs_rank0": us / res[0] - 1.0}
            del X, Y
            torch.cuda.empty_cache()
    return out


def refinement(L, iters=4):
    """NEXT-2 (SVDQuant §4.2, iterative refinement of the split): residual
    quantization error of each split tried and the host preparation time,
    plain vs refined, on one SDXL attention layer."""
    c = config_cases("sdxl")[0]
    t = make_layer_inputs(c)
    out = {"layer": f"{c.label} N={c.N} K={c.K} rank={c.rank}"}
    for it in (1, iters):
        t0 = time.time()
        w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=c.rank, refine_iters=it)
        out[f"iters{it}"] = {"errors": L.svdq_weights_refine_errors(w), "prepare_s": time.time() - t0}
    e1, e4 = out["iters1"]["errors"][0], min(out[f"iters{iters}"]["errors"])
    out["error_reduction"] = 1.0 - e4 / e1
    return out


def int4_layers(L, torch, layers, dev, stream, reps=30):
    """NEXT-4, the INT4 variant (App. D: groups of 64, 16-bit scales) on the step's
    layers: library-prepared INT4 weights (rank 32), layer time (both kernels)
    and GEMM time, the GEMM's rate against the measured dense bf16 peak (its
    contraction runs on fp16 tiles dequantized on chip), and the NVFP4 layer
    time for comparison."""
    pk = peaks()
    out = {"peak_bf16_tflops": pk["bf16"], "layers": {}}
    for l in layers:
        c = l["case"]
        t = make_layer_inputs(c)
        w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=c.rank, fmt="int4")
        xq, xsf, T = L.act_buffers(w, c.M, dev)

        def layer():
            L.svdq_quantize_act_lowrank_down(w, l["X"], xq, xsf, T)
            L.svdq_linear_w4a4(w, xq, xsf, T, c.M, l["Y"])

        def gemm():
            L.svdq_linear_w4a4(w, xq, xsf, T, c.M, l["Y"])

        us = 1e3 * _time_ms(torch, stream, layer, reps)
        us_g = 1e3 * _time_ms(torch, stream, gemm, reps)
        tf = c.flops / (us_g * 1e-6) / 1e12
        out["layers"][c.name] = {"us": us, "gemm_us": us_g, "gemm_tflops": tf, "frac_of_bf16_peak": tf / pk["bf16"]}
    return out


def norm_fusion(L, torch, layers, dev, stream, reps=30, eps=1e-6):
    """NEXT-3, the activation kernel fused with the adaLN front end (LayerNorm
    over K, then a = 1 + scale, c = shift per channel): per step layer, the
    fused path (row statistics + fused activation kernel + GEMM) against the
    unfused one (a PyTorch LayerNorm and modulation writing bf16 X, then the
    layer), and the layer alone on a ready X for reference."""
    out = {}
    g = torch.Generator(device="cpu").manual_seed(5)
    for l in layers:
        c, w = l["case"], l["w"]
        Z = (torch.randn(c.M, c.K, generator=g) * 2 + 1).to(torch.bfloat16).to(dev)
        a = (1 + 0.1 * torch.randn(c.K, generator=g)).to(dev)
        sh = (0.1 * torch.randn(c.K, generator=g)).to(dev)
        ws = torch.empty(L.svdq_forward_norm_workspace_bytes(w, c.M), dtype=torch.uint8, device=dev)
        Y = l["Y"]

        def fused():
            L.svdq_forward_norm(w, Z, a, sh, eps, Y, ws)

        def unfused():
            X = (torch.nn.functional.layer_norm(Z.float(), (c.K,), eps=eps) * a + sh).to(torch.bfloat16)
            L.svdq_forward(w, X, Y, ws)

        def layer_only():
            L.svdq_forward(w, l["X"], Y, ws)

        out[c.name] = {"fused_us": 1e3 * _time_ms(torch, stream, fused, reps),
                       "unfused_us": 1e3 * _time_ms(torch, stream, unfused, reps),
                       "layer_only_us": 1e3 * _time_ms(torch, stream, layer_only, reps)}
    return out


def _cublaslt_fp4_us(torch, M, K, N, dev, stream, reps):
    """cuBLASLt's NVFP4 GEMM (torch._scaled_mm on float4_e2m1fn_x2 with E4M3 block
    scales in the 128 x 4 atom layout, bf16 out, no low-rank branch): a plain
    library GEMM timed only as a measured FP4 reference; None when this torch
    build has no such path."""
    if not hasattr(torch, "float4_e2m1fn_x2"):
        return None
    g = torch.Generator(device=dev).manual_seed(0)

    def atoms(rows):
        kb = K // 16
        return torch.full((((rows + 127) // 128 * 128) * kb,), 0x30, dtype=torch.uint8,
                          device=dev).view(torch.float8_e4m3fn)  # 0x30 = 0.5, every block

    a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g).view(torch.float4_e2m1fn_x2)
    b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g).view(torch.float4_e2m1fn_x2)
    sa, sb = atoms(M), atoms(N)
    try:
        return 1e3 * _time_ms(torch, stream, lambda: torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16),
                              reps)
    except (RuntimeError, TypeError) as ex:  # this torch has no NVFP4 kernel
        print(f"cuBLASLt NVFP4 GEMM unavailable: {str(ex)[:200]}", file=sys.stderr)
        return None


def fp4_reference(L, torch, dev, stream, reps=20):
    """A measured FP4 rate beside the nominal one: this library's GEMM (rank 0,
    unit smoothing, random weights and activations) and cuBLASLt's NVFP4 GEMM on
    a large square problem and on the step's largest layer shape, as TFLOP/s."""
    out = {}
    for name, (M, K, N) in {"square_8192": (8192, 8192, 8192), "flux_mlp_up": (4608, 3072, 12288)}.items():
        rng = np.random.default_rng(M + K + N)
        R = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
        w = L.svdq_weights_from_factors(N, K, 0, np.ones(K, np.float32), None, None, R)
        del R
        X = torch.randn((M, K), generator=torch.Generator(device=dev).manual_seed(1), device=dev).to(torch.bfloat16)
        xq, xsf, _ = L.act_buffers(w, M, dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        L.svdq_quantize_act_lowrank_down(w, X, xq, xsf, None)
        us = 1e3 * _time_ms(torch, stream, lambda: L.svdq_linear_w4a4(w, xq, xsf, None, M, Y), reps)
        del X
        cub = _cublaslt_fp4_us(torch, M, K, N, dev, stream, reps)
        fl = 2.0 * M * N * K
        out[name] = {"M": M, "K": K, "N": N, "ours_us": us, "ours_tflops": fl / (us * 1e-6) / 1e12,
                     "cublaslt_us": cub, "cublaslt_tflops": fl / (cub * 1e-6) / 1e12 if cub else None}
        del w, xq, xsf, Y
        torch.cuda.empty_cache()
    return out


def alpha_search(L, rows=256):
    """NEXT-3 (App. D migration strength): relative output error per candidate
    alpha on a calibration batch of one FLUX layer, through the library's own
    preparation and kernels, and the search's wall time."""
    c = [x for x in config_cases("flux") if x.name == "attn_out"][0]
    t = make_layer_inputs(c)
    alphas = (0.3, 0.4, 0.5, 0.6, 0.7, 0.8, 0.9)
    t0 = time.time()
    errs, best = L.svdq_search_alpha(t.W_bits, t.X_bits[:rows], t.bias_bits, alphas, rank=c.rank)
    return {"layer": f"{c.label} N={c.N} K={c.K} rank={c.rank}, calibration rows {rows}",
            "rel_err": dict(zip([str(a) for a in alphas], errs)), "best_alpha": alphas[best],
            "gain_vs_0.5": 1.0 - errs[best] / errs[alphas.index(0.5)], "search_s": time.time() - t0}


# ------------------------------------------------------------------ ours
def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local))
    import rank_outlier_gemm_b200 as L

    dev = torch.device("cuda", local)
    cases = flux_cases()
    layers = []
    for c in cases:
        t = make_layer_inputs(c)
        w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=c.rank, fmt=args.format)
        w0 = (L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=0, fmt=args.format)
              if args.extras else None)
        X = torch.from_numpy(t.X_bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        bufs = L.act_buffers(w, c.M, dev)
        Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
        layers.append(dict(case=c, w=w, w0=w0, X=X, bufs=bufs, Y=Y, X_bits=t.X_bits))
    stream = torch.cuda.current_stream()

    def step(evs=None):
        for i, l in enumerate(layers):
            xq, xsf, T = l["bufs"]
            if evs is not None:
                evs[i][0].record(stream)
            L.svdq_quantize_act_lowrank_down(l["w"], l["X"], xq, xsf, T)
            if evs is not None:
                evs[i][1].record(stream)
            L.svdq_linear_w4a4(l["w"], xq, xsf, T, l["case"].M, l["Y"])
            if evs is not None:
                evs[i][2].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def slowest(x: float) -> float:
        return max_over_ranks(x, world, dev)

    for _ in range(args.warmup):
        step()
    assert L.svdq_check_device_errors() == 0
    nl = len(layers)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nl)]
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(local) as cs:
        # headline: K steps with events only around them, so that each GEMM
        # launch can overlap the tail of the activation kernel ahead of it
        t0.record(stream)
        for s in range(args.steps):
            step()
        t1.record(stream)
        barrier()
        # per-kernel breakdown: the same K steps with events between the
        # kernels (which serialise each GEMM behind its activation kernel)
        for s in range(args.steps):
            step(evs[s])
        barrier()
    assert L.svdq_check_device_errors() == 0
    ms = slowest(t0.elapsed_time(t1))
    ms_step = ms / args.steps
    k1 = [statistics.mean(evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(args.steps)) for i in range(nl)]
    k2 = [statistics.mean(evs[s][i][1].elapsed_time(evs[s][i][2]) for s in range(args.steps)) for i in range(nl)]
    flops_step = sum(l["case"].flops for l in layers)
    value = job_throughput(flops_step, ms_step, world)

    pk = peaks()
    # The burst cuBLAS figure applies while the SM clock holds its maximum; a run that
    # the power cap pulled down is compared with the sustained one.
    cl = cs.summary()
    capped = bool(cl) and ("sw_power_cap" in cl["reasons"] or
                           (cl["sm_mhz"] or 0) < 0.95 * (cl["sm_max_mhz"] or 1))
    bf16_peak = pk["bf16_sustained"] if capped else pk["bf16"]
    if args.format == "int4":  # the INT4 GEMM contracts fp16 tiles dequantized on chip
        fp4_peak = bf16_peak
        peak_src = f"{pk['source']} bf16 {'sustained' if capped else 'burst'} {bf16_peak} (fp16 contraction)"
        traffic, traffic_note = None, "no ncu counters kept for the INT4 GEMM in bench.py"
    else:
        fp4_peak = bf16_peak * NOMINAL_FP4_OVER_BF16
        peak_src = (f"{pk['source']} bf16 {'sustained' if capped else 'burst'} {bf16_peak} x "
                    f"{NOMINAL_FP4_OVER_BF16} (nominal FP4:BF16)")
        traffic, traffic_note = k2_traffic_per_launch([l["case"].name for l in layers])
    k2_flops = flops_step
    k2_ms = sum(k2)
    achieved = k2_flops / (k2_ms * 1e-3) / 1e12
    roof_us = {l["case"].name: max(l["case"].flops / (fp4_peak * 1e12), layer_bytes(l["case"]) / (pk["hbm"] * 1e9)) * 1e6
               for l in layers}

    # low-rank overhead: the same kernels at rank 0, timed in alternating blocks
    # of rank-32 and rank-0 steps so that clock drift hits both alike; the
    # median of the per-round ratios is reported
    overhead = overhead_rounds = None
    unfused = sweep = small = refine = asearch = int4 = normf = fp4ref = models = None
    if args.extras:
        def step0():
            for l in layers:
                xq, xsf, _ = l["bufs"]
                L.svdq_quantize_act_lowrank_down(l["w0"], l["X"], xq, xsf, None)
                L.svdq_linear_w4a4(l["w0"], xq, xsf, None, l["case"].M, l["Y"])
        n0 = max(10, args.steps // 4)
        for _ in range(3):
            step0()
        ratios, ms0s = [], []
        for _ in range(7):
            t32 = _time_ms(torch, stream, step, n0)
            t00 = _time_ms(torch, stream, step0, n0)
            ratios.append(t32 / t00 - 1.0)
            ms0s.append(t00)
        overhead = statistics.median(ratios)
        overhead_rounds = ratios
        ms0 = statistics.median(ms0s)
        if rank == 0:
            unfused = unfused_overhead(L, torch, layers, stream, ms0, n0)
            sweep = rank_sweep(L, torch, layers, dev, stream)
            small = small_m(L, torch, dev, stream)
            models = model_layers(L, torch, dev)
            refine = refinement(L)
            asearch = alpha_search(L)
            int4 = int4_layers(L, torch, layers, dev, stream) if args.format == "nvfp4" else None
            normf = norm_fusion(L, torch, layers, dev, stream)
            fp4ref = fp4_reference(L, torch, dev, stream) if args.format == "nvfp4" else None

    # end to end through the public host-buffer call: H2D of X, both kernels, D2H of Y
    e2e = None
    if args.e2e_steps > 0:
        host = []
        for l in layers:
            c = l["case"]
            Xh = torch.from_numpy(l["X_bits"].view(np.int16).copy()).view(torch.bfloat16).pin_memory()
            Yh = torch.empty((c.M, c.N), dtype=torch.bfloat16).pin_memory()
            ws = torch.empty(L.svdq_forward_host_workspace_bytes(l["w"], c.M), dtype=torch.uint8, device=dev)
            host.append((Xh, Yh, ws))

        def step_e2e():
            for l, (Xh, Yh, ws) in zip(layers, host):
                L.svdq_forward_host(l["w"], Xh, Yh, ws)

        step_e2e()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            step_e2e()
        b.record(stream)
        barrier()
        ems = slowest(a.elapsed_time(b)) / args.e2e_steps
        h2d = sum(l["case"].M * l["case"].K * 2 for l in layers)
        d2h = sum(l["case"].M * l["case"].N * 2 for l in layers)
        e2e = {"value": job_throughput(flops_step, ems, world), "unit": "TFLOP/s", "ms_per_step": ems,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}

    if rank == 0:
        us_layer = {l["case"].name: 1e3 * (k1[i] + k2[i]) for i, l in enumerate(layers)}
        # the extras go on a line of their own, before the headline line
        extras = {
            "extras_of": METRIC,
            "breakdown_note": ("us_per_layer / us_act_kernel / us_gemm_kernel come from a second pass of the "
                               "same steps with events between the kernels, which serialise each GEMM "
                               "behind its activation kernel; the headline step time lets them overlap"),
            "roofline_us_per_layer": roof_us,
            "lowrank_overhead_rounds": overhead_rounds,
            "unfused_lowrank_overhead_vs_rank0": unfused,
            "rank_sweep": sweep,
            "small_m_lora": small,
            "model_layers": models,
            "refinement": refine,
            "alpha_search": asearch,
            "int4": int4,
            "norm_fusion": normf,
            "fp4_reference": fp4ref,
        }
        if args.extras:
            print(json.dumps(extras))
        out = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": args.format, "data": "synthetic (seeded; FLUX.1 shapes, random weights)",
            "config": {"workload": WORKLOAD, "format": args.format, "M": cases[0].M,
                       "layers": [[c.K, c.N] for c in cases],
                       "rank": cases[0].rank, "parallelism": f"replicas x{world}",
                       "l2": "step footprint ~0.5 GB > 126 MB L2; no flush"},
            "us_per_layer": us_layer,
            "us_act_kernel": {l["case"].name: 1e3 * k1[i] for i, l in enumerate(layers)},
            "us_gemm_kernel": {l["case"].name: 1e3 * k2[i] for i, l in enumerate(layers)},
            "frac_of_layer_roofline": sum(roof_us.values()) / (1e3 * (sum(k1) + sum(k2))),
            "lowrank_overhead_vs_rank0": overhead,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": achieved / fp4_peak, "traffic": traffic, "traffic_note": traffic_note,
                         "kernel": "gemm_int4_kernel" if args.format == "int4" else
                         "gemm_w4a4_kernel (K = 3072 layers), gemm_w4a4_pair_kernel (K = 12288)",
                         "peak_source": peak_src,
                         "frac_of_datasheet_9pf": achieved / 9000.0},
            "gpu_launches": 2 * nl * args.steps,
            "e2e": e2e,
        }
        if cl:
            out["clocks"] = cl
        if args.cpu_baseline and world == 1:
            out["cpu_baseline"] = cpu_baseline(args.cpu_rows, reps=1)
        print(json.dumps(out))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ oracle
def _oracle_layers():
    from oracle import svdquant as OS
    preps = []
    for c in flux_cases():
        t = make_layer_inputs(c)
        preps.append((c, t, OS.prepare(t.W, t.act_absmax, t.bias, c.rank)))
    return preps


def cpu_baseline(rows: int, reps: int = 1, preps=None):
    """The oracle's runtime step (activation codec, fp64 dequantized GEMM,
    low-rank branch) on `rows` rows of every layer; weight preparation untimed."""
    from oracle import svdquant as OS
    preps = preps or _oracle_layers()
    sample = np.arange(rows)
    flops = sum(2 * rows * c.N * c.K for c, _, _ in preps)

    def timed():
        t = time.perf_counter()
        for _ in range(reps):
            for c, inp, prep in preps:
                OS.linear(prep, inp.X, rows=sample)
        return (time.perf_counter() - t) / reps

    dt = timed()
    out = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
           "sample": f"first {rows} of 4608 rows of each FLUX layer per step (weights full size)",
           "seconds_per_step": dt}
    try:  # the same sample on one thread (BLAS limited to one thread)
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            dt1 = timed()
        out["single_thread"] = {"value": flops / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                                "seconds_per_step": dt1}
    except ImportError:
        pass
    return out


def _threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    """The oracle as the reference arm: each step computes a bounded sample of
    the step's outputs (args.ref_rows rows x args.ref_cols output columns of
    every layer) on the host cores; flops count only the sampled outputs."""
    world, rank, _ = dist_env()
    if rank != 0:  # the host-side reference runs once per job, on rank 0
        return
    from oracle import svdquant as OS
    preps = _oracle_layers()
    rows = np.arange(args.ref_rows)

    def one_step(s):
        for c, inp, prep in preps:
            cols = (np.arange(args.ref_cols) * 7919 + s * 131) % c.N
            OS.linear(prep, inp.X, rows=rows, cols=cols)

    for s in range(args.warmup):
        one_step(s)
    t = time.perf_counter()
    for s in range(args.steps):
        one_step(s)
    dt = (time.perf_counter() - t) / args.steps
    flops = sum(2 * args.ref_rows * args.ref_cols * c.K for c, _, _ in preps)
    v = flops / dt / 1e12
    sample = (f"{args.ref_rows} rows x {args.ref_cols} output columns of each of the 4 FLUX layers "
              f"per step (weights prepared untimed)")
    out = {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; FLUX.1 shapes, random weights)",
           "config": {"workload": WORKLOAD, "M": 4608, "layers": [[c.K, c.N] for c, _, _ in preps],
                      "rank": 32, "parallelism": "host cores"},
           "impl": "reference",
           "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out))


def run_layer_only(args):
    """Profiling mode: one configured layer (``cfg/name`` or ``cfg/name:M``),
    library-prepared weights (LoRA attached where the configuration has one),
    ``--warmup`` + ``--steps`` launches of the activation kernel and the GEMM
    (``--kernel act|gemm|both``: the GEMM-only mode runs the activation kernel
    once first), and one JSON line with the mean device time per launch pair.
    For ncu captures of a single kernel on a chosen shape."""
    import torch
    import rank_outlier_gemm_b200 as L

    lab, _, m = args.layer_only.partition(":")
    cfg, name = lab.split("/")
    c = [x for x in config_cases(cfg) if x.name == name][0]
    M = int(m) if m else c.M
    t = make_layer_inputs(c, M=M)
    w = L.svdq_prepare_weights(t.W_bits, t.act_absmax, t.bias_bits, rank=c.rank, fmt=args.format)
    if c.lora_rank:
        L.svdq_attach_lora(w, t.lora_A_bits, t.lora_B_bits, t.lora_scale)
    X = torch.from_numpy(t.X_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    xq, xsf, T = L.act_buffers(w, M)
    Y = torch.empty((M, c.N), dtype=torch.bfloat16, device="cuda")

    def one():
        if args.kernel in ("act", "both"):
            L.svdq_quantize_act_lowrank_down(w, X, xq, xsf, T)
        if args.kernel in ("gemm", "both"):
            L.svdq_linear_w4a4(w, xq, xsf, T, M, Y)

    if args.kernel == "gemm":
        L.svdq_quantize_act_lowrank_down(w, X, xq, xsf, T)
    for _ in range(args.warmup):
        one()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(args.steps):
        one()
    b.record()
    torch.cuda.synchronize()
    assert L.svdq_check_device_errors() == 0
    print(json.dumps({"layer": f"{lab} M={M} K={c.K} N={c.N}", "kernel": args.kernel,
                      "us_per_launch": 1e3 * a.elapsed_time(b) / args.steps}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-rows", type=int, default=16)
    ap.add_argument("--ref-rows", type=int, default=2)
    ap.add_argument("--ref-cols", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-extras", dest="extras", action="store_false")
    ap.add_argument("--layers", default="", help="comma-separated subset of the FLUX layers (profiling)")
    ap.add_argument("--format", choices=["nvfp4", "int4"], default="nvfp4",
                    help="4-bit format of the timed step (INT4: the variant with group-64 bf16 scales)")
    ap.add_argument("--layer-only", default="",
                    help="profiling: time one configured layer, cfg/name[:M] (e.g. small_m_lora/M16_N12288:16)")
    ap.add_argument("--kernel", choices=["act", "gemm", "both"], default="both",
                    help="with --layer-only: which kernel(s) to launch")
    args = ap.parse_args()
    if args.layer_only:
        if args.warmup < 3:
            ap.error("--warmup must be >= 3")
        run_layer_only(args)
        return
    global LAYER_FILTER
    LAYER_FILTER = [x for x in args.layers.split(",") if x] or None
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
