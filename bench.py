#!/usr/bin/env python
"""Benchmark of the DiT-block denoising path on B200; prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config dit512] [--impl reference]

A step is one complete denoise of the workload: every Euler step of the configured sigma
grid, each running every active DiT block over the joint video+audio token stream (the
whole hot path: AdaLN LN, QKV+RoPE, attention, out-proj+gated residual, LN, FC1+GELU,
FC2+gated residual, final AdaLN + Euler).  Inputs are synthetic (seeded, random-init
weights of the stated architecture).  The metric is DiT block tokens per second: tokens
processed by each executed block, summed over blocks and Euler steps, per second of
device time; TFLOPS counts 24 N d^2 + 4 N^2 d per block.

Multi-GPU (one process per GPU): every rank denoises its own latent with the same weights
(independent replicas, no data-path collective); value = all ranks' tokens / the slowest
rank's device time.  Under torchrun the ranks come from the environment; `--gpus N` with
N > 1 and no WORLD_SIZE set re-launches this script under torch.distributed.run with N
processes (127.0.0.1 rendezvous), so N GPUs really run.

--impl reference runs the CPU oracle (the plain float64 definition of the same block) on
a bounded sample of the workload: one block over the full token count per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DiT block tokens/sec and achieved bf16 TFLOPS vs tensor peak, 1xB200"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# dram bytes per launch from an ncu capture, keyed by kernel; only used while the kernel
# source still hashes to the value recorded with it.
NCU_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch on the dit512 shape after 3
    # warm-ups (`bench.py --kernel <name> --reps 3`, ncu --metrics dram__bytes_read.sum,
    # dram__bytes_write.sum; profiles/), valid while the kernel's source file hashes to src_sha
    "gemm_fc1_gelu": {"bytes": 85670144 + 18355200, "src": "gemm_tc.cu",
                      "src_sha": "af9960a45b179aa3"},
    "gemm_fc2_gate": {"bytes": 137548544 + 17156096, "src": "gemm_tc.cu",
                      "src_sha": "af9960a45b179aa3"},
    "gemm_qkv_rope": {"bytes": 67616512 + 9027072, "src": "gemm_tc.cu",
                      "src_sha": "af9960a45b179aa3"},
    "gemm_out_gate": {"bytes": 38624512 + 1132032, "src": "gemm_tc.cu",
                      "src_sha": "af9960a45b179aa3"},
    "attention": {"bytes": 29571328 + 206848, "src": "attention_tc.cu",
                  "src_sha": "83cba2667860a7ac"},
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="dit512")
    ap.add_argument("--impl", default="h3b", choices=["h3b", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--kernel", default=None,
                    help="time one kernel of the block alone on the workload shapes, or the "
                         "fc2_int8_row / token_pairing / grouped_fc2_int8 workload (for ncu)")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--no-also", action="store_true",
                    help="skip the secondary measurements of the other workloads")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel from the host instead of replaying a CUDA graph")
    ap.add_argument("--attn-variant", type=int, default=0,
                    help="attention form: 0 automatic, 1 one query tile per CTA, 2 two tiles")
    ap.add_argument("--replica-check", action="store_true",
                    help="CPU only: run the replica plumbing (gloo barrier, max over ranks, "
                         "job rate) through the same launcher and print what every rank saw")
    return ap.parse_args(argv)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        peaks = dict(FALLBACK_PEAKS)
        peaks.update({k: float(d[k]) for k in FALLBACK_PEAKS if k in d})
        peaks["source"] = "MEASURED_PEAKS.json"
        return peaks, "measured"
    peaks = dict(FALLBACK_PEAKS)
    peaks["source"] = "the fallback figures (MEASURED_PEAKS.json absent)"
    return peaks, "fallback"


def block_flops(n, d, f):
    return 2 * n * d * 3 * d + 2 * n * d * d + 4 * n * d * f + 4 * n * n * d


def workload_counts(cfg, active):
    """Per complete denoise: block-tokens, FLOPs and launches of each block kernel."""
    order = [b for b in range(cfg.n_blocks) if active is None or active[b]]
    n_full, n_red = cfg.n_tokens, cfg.n_video_reduced + cfg.n_audio
    tokens = flops = 0
    for k, _ in enumerate(order):
        n = n_red if (cfg.reduce_after > 0 and k >= cfg.reduce_after) else n_full
        tokens += n
        flops += block_flops(n, cfg.d, cfg.d_ff)
    per_step = {"tokens": tokens, "flops": flops, "blocks": len(order)}
    return {k: v * cfg.run_steps for k, v in per_step.items()}, len(order)


def src_hash(name):
    with open(os.path.join(ROOT, "video_diffusion_transformer_03_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.path = tempfile.mktemp(prefix="h3b_clocks_", suffix=".csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", gpu_id, "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 9:
                        continue
                    try:
                        sm.append(float(parts[1]))
                        smax.append(float(parts[2]))
                    except ValueError:
                        continue
                    for name, val in zip(self.NAMES, parts[5:9]):
                        if val.lower() == "active":
                            reasons.add(name)
            os.unlink(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------ CPU oracle
def oracle_sample(cfg, min_seconds=10.0, max_blocks=8):
    """Time the oracle (float64 numpy, as it stands) on full-size blocks of the workload."""
    import numpy as np
    from oracle import workloads
    from video_diffusion_transformer_03_b200 import synth
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        cores = os.cpu_count()
    f64 = lambda t: t.float().numpy().astype(np.float64)
    p = {k: f64(v) for k, v in synth.block_params(cfg, 0).items()}
    c = f64(synth.conditioning(cfg))
    x = f64(synth.latent_noise(cfg).to(__import__("torch").bfloat16))
    done, t0 = 0, time.perf_counter()
    while done < max_blocks:
        x, _ = workloads.block(cfg, p, c, x)
        done += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": cfg.n_tokens * done / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{done} full block forward(s) of {cfg.name} ({cfg.n_tokens} tokens, "
                      f"d={cfg.d}) in float64 numpy, {dt:.1f} s"}


def run_reference(args):
    from video_diffusion_transformer_03_b200 import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    from oracle import workloads
    cfg = synth.CONFIGS[args.config]
    f64 = lambda t: t.float().numpy().astype(np.float64)
    p = {k: f64(v) for k, v in synth.block_params(cfg, 0).items()}
    c = f64(synth.conditioning(cfg))
    x0 = f64(synth.latent_noise(cfg).to(__import__("torch").bfloat16))
    for _ in range(args.warmup):
        workloads.block(cfg, p, c, x0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        workloads.block(cfg, p, c, x0)
    dt = time.perf_counter() - t0
    value = cfg.n_tokens * args.steps / dt
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        cores = os.cpu_count()
    flops = block_flops(cfg.n_tokens, cfg.d, cfg.d_ff)
    # one process (rank 0) ran the CPU oracle on the host cores; no GPU was used
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "processes": 1, "ranks_launched": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": workload_name(cfg), "sample": "one full block forward per step"},
            "tflops": flops * args.steps / dt / 1e12,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"one full block forward of {cfg.name} per step "
                                       f"({cfg.n_tokens} tokens), float64 numpy"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_name(cfg):
    t, h, w = cfg.grid
    s = (f"{cfg.name}: {cfg.n_blocks} DiT blocks d={cfg.d} {cfg.n_heads}x{cfg.head_dim} heads "
         f"MLP {cfg.d_ff}, video grid t{t}xh{h}xw{w}={cfg.n_video} + {cfg.n_audio} audio tokens, "
         f"{cfg.run_steps} Euler steps")
    if cfg.reduce_after > 0:
        s += f", token pairing after block {cfg.reduce_after}"
    if cfg.active_count < cfg.n_blocks:
        s += f", {cfg.active_count} of {cfg.n_blocks} blocks active"
    return s


# ------------------------------------------------------------------------------ GPU arm
def time_kernels(model, cfg, peaks, counts_per_step, reps=20, only=None, warm=3):
    """Time each kernel of the block alone (CUDA events around a CUDA-graph replay of
    `reps` launches, as the denoise runs them), with the weights rotated over all blocks
    so that they stream from HBM as in the step."""
    import torch
    from video_diffusion_transformer_03_b200 import h3b
    dev = model.device
    n, d, f, hd, H = cfg.n_tokens, cfg.d, cfg.d_ff, cfg.head_dim, cfg.n_heads
    g = torch.Generator(device=dev).manual_seed(7)
    rnd = lambda *s: torch.randn(*s, generator=g, device=dev).to(torch.bfloat16)
    h = rnd(n, d)
    qkv = rnd(n, 3 * d)
    attn = torch.empty(n, d, dtype=torch.bfloat16, device=dev)
    gbuf = rnd(n, f)
    x = rnd(n, d)
    xs = torch.randn(n, d, device=dev)
    cs = torch.empty((n, hd // 2, 2), dtype=torch.float32, device=dev)
    h3b.rope_table(model.dims, model.grid, False, cs)
    mod = model.mods[0]
    P = model.params
    nb = len(P)
    ws = torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=dev)
    st = torch.empty((n, d // 256, 2), dtype=torch.float32, device=dev)
    h3b.row_stats(x, st)
    if model.fold:
        # the kernels of the folded block: projections that read the raw residual and its
        # row statistics, gated-residual epilogues that write the statistics
        gemms = {
            "gemm_qkv_rope": (lambda i: h3b.gemm_bf16_ln(
                x, P[i % nb]["w_qkv_fold"], h3b.EPI_LN_ROPE, qkv, fold_c=P[i % nb]["c_qkv"],
                fold_dv=P[i % nb]["d_qkv"], stats_in=st, ln_eps=cfg.ln_eps, rope_cs=cs,
                rope_cols=2 * d, head_dim=hd, ws=ws), "tensor", 2 * n * d * 3 * d),
            "gemm_out_gate": (lambda i: h3b.gemm_bf16_ln(
                attn, P[i % nb]["w_o"], h3b.EPI_GATE_RESID, x, bias=P[i % nb]["b_o"],
                gate=mod[2], stats_out=st, ws=ws), "tensor", 2 * n * d * d),
            "gemm_fc1_gelu": (lambda i: h3b.gemm_bf16_ln(
                x, P[i % nb]["w_fc1_fold"], h3b.EPI_LN_GELU, gbuf, fold_c=P[i % nb]["c_fc1"],
                fold_dv=P[i % nb]["d_fc1"], stats_in=st, ln_eps=cfg.ln_eps, ws=ws),
                "tensor", 2 * n * d * f),
            "gemm_fc2_gate": (lambda i: h3b.gemm_bf16_ln(
                gbuf, P[i % nb]["w_fc2"], h3b.EPI_GATE_RESID, x, bias=P[i % nb]["b_fc2"],
                gate=mod[5], stats_out=st, ws=ws), "tensor", 2 * n * f * d),
        }
    else:
        gemms = {
            "gemm_qkv_rope": (lambda i: h3b.gemm_bf16(h, P[i % nb]["w_qkv"], h3b.EPI_BIAS_ROPE,
                                                      P[i % nb]["b_qkv"], qkv, rope_cs=cs,
                                                      rope_cols=2 * d, head_dim=hd, ws=ws),
                              "tensor", 2 * n * d * 3 * d),
            "gemm_out_gate": (lambda i: h3b.gemm_bf16(attn, P[i % nb]["w_o"], h3b.EPI_GATE_RESID,
                                                      P[i % nb]["b_o"], x, gate=mod[2], ws=ws),
                              "tensor", 2 * n * d * d),
            "gemm_fc1_gelu": (lambda i: h3b.gemm_bf16(h, P[i % nb]["w_fc1"], h3b.EPI_BIAS_GELU,
                                                      P[i % nb]["b_fc1"], gbuf, ws=ws),
                              "tensor", 2 * n * d * f),
            "gemm_fc2_gate": (lambda i: h3b.gemm_bf16(gbuf, P[i % nb]["w_fc2"], h3b.EPI_GATE_RESID,
                                                      P[i % nb]["b_fc2"], x, gate=mod[5], ws=ws),
                              "tensor", 2 * n * f * d),
        }
    kinds = {
        "gemm_qkv_rope": gemms["gemm_qkv_rope"],
        "attention": (lambda i: h3b.attention(qkv, H, hd, attn, ws=ws), "tensor", 4 * n * n * d),
        "gemm_out_gate": gemms["gemm_out_gate"],
        "gemm_fc1_gelu": gemms["gemm_fc1_gelu"],
        "gemm_fc2_gate": gemms["gemm_fc2_gate"],
        "final_euler": (lambda i: h3b.final_euler(x, cfg.n_video, cfg.ln_eps, model.final_mod,
                                                  1.0, 0.75, xs), "hbm", 10 * n * d),
    }
    if not model.fold:
        kinds["ln_modulate"] = (lambda i: h3b.ln_modulate(x, cfg.ln_eps, mod[0], mod[1], h),
                                "hbm", 4 * n * d)
    blocks = counts_per_step["blocks"]
    launches = {"gemm_qkv_rope": blocks, "attention": blocks, "gemm_out_gate": blocks,
                "gemm_fc1_gelu": blocks, "gemm_fc2_gate": blocks, "ln_modulate": 2 * blocks,
                "final_euler": cfg.run_steps}
    out = {}
    for name, (fn, bound, work) in kinds.items():
        if only is not None and name != only:
            continue
        for i in range(warm):
            fn(i)
        torch.cuda.synchronize(dev)
        # the reps are captured as one CUDA graph and replayed, so the device time is not
        # bounded by the host's per-call cost (short kernels would otherwise measure it)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(reps):
                fn(i)
        graph.replay()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        stream = torch.cuda.current_stream(dev)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        del graph
        h3b.sync_status()
        ms = e0.elapsed_time(e1) / reps
        if bound == "tensor":
            achieved, peak, unit = work / (ms * 1e-3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        else:
            achieved, peak, unit = work / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
        out[name] = {"bound": bound, "ms": ms, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "work_per_launch": work,
                     "launches_per_step": launches[name],
                     "ms_per_step": ms * launches[name]}
        if bound == "hbm":
            # the same launch with the L2 flushed before each one (its inputs come from HBM)
            cold = time_cold(lambda: fn(0), dev)
            out[name]["cold_ms"] = cold
            out[name]["cold_frac"] = work / (cold * 1e-3) / 1e9 / peaks["hbm_gbs"]
    return out


_FLUSH = {}


def flush_l2(dev):
    """Overwrite a buffer twice the size of the 126 MB L2."""
    import torch
    buf = _FLUSH.get(dev)
    if buf is None:
        buf = _FLUSH[dev] = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    buf.zero_()


def time_cold(fn, dev, reps=10):
    """Average device time of single launches, each after an L2 flush (CUDA events around
    the launch only)."""
    import torch
    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    fn()
    for a, b in ev:
        flush_l2(dev)
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize(dev)
    return sum(a.elapsed_time(b) for a, b in ev) / reps


def time_gemm_widths(dev, peaks, reps=10):
    """bf16 GEMMs at the model widths the pages name (5376, 7168), M = 1600 and 2048 rows:
    out = A[M, d] W[d, d]^T + bias (an out-projection shape) and the QKV shape N = 3 d."""
    import torch
    from video_diffusion_transformer_03_b200 import h3b
    g = torch.Generator(device=dev).manual_seed(11)
    ws = torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=dev)
    res = []
    for d in (5376, 7168):
        for M in (1600, 2048):
            for N in (d, 3 * d):
                A = (torch.randn(M, d, generator=g, device=dev) * 0.5).to(torch.bfloat16)
                W = (torch.randn(N, d, generator=g, device=dev) * 0.02).to(torch.bfloat16)
                b = torch.zeros(N, dtype=torch.bfloat16, device=dev)
                out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
                f = lambda: h3b.gemm_bf16(A, W, h3b.EPI_BIAS, b, out, ws=ws)
                for _ in range(3):
                    f()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize(dev)
                e0.record()
                for _ in range(reps):
                    f()
                e1.record()
                torch.cuda.synchronize(dev)
                ms = e0.elapsed_time(e1) / reps
                tf = 2 * M * N * d / (ms * 1e-3) / 1e12
                res.append({"M": M, "N": N, "K": d, "ms": ms, "tflops": tf,
                            "frac": tf / peaks["bf16_tflops"]})
                del A, W, out
    h3b.sync_status()
    torch.cuda.empty_cache()
    return res


def time_library_same_shapes(model, cfg, dev, reps=20):
    """Context for the breakdown: the vendor libraries on the block's shapes, timed the same
    way (CUDA events around a CUDA-graph replay of `reps` launches, weights rotated over the
    blocks).  cuBLAS through torch's bf16 linear (no epilogue: no bias, LayerNorm fold, RoPE,
    GELU or gate), and torch's scaled-dot-product attention on its cuDNN backend where it
    is available (else torch's own choice, named)."""
    import torch
    import torch.nn.functional as F
    n, d, f, hd, H = cfg.n_tokens, cfg.d, cfg.d_ff, cfg.head_dim, cfg.n_heads
    P = model.params
    nb = len(P)
    g = torch.Generator(device=dev).manual_seed(9)
    rnd = lambda *s: torch.randn(*s, generator=g, device=dev).to(torch.bfloat16)
    x, gbuf = rnd(n, d), rnd(n, f)
    gemms = {"gemm_qkv_rope": (x, "w_qkv", 2 * n * d * 3 * d),
             "gemm_out_gate": (x, "w_o", 2 * n * d * d),
             "gemm_fc1_gelu": (x, "w_fc1", 2 * n * d * f),
             "gemm_fc2_gate": (gbuf, "w_fc2", 2 * n * f * d)}

    def graph_ms(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(reps):
                fn(i)
        graph.replay()
        stream = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        del graph
        return e0.elapsed_time(e1) / reps

    out = {}
    for name, (a, w, flops) in gemms.items():
        ms = graph_ms(lambda i: F.linear(a, P[i % nb][w]))
        out[name] = {"library": "cuBLAS (torch bf16 linear, no epilogue)", "ms": ms,
                     "tflops": flops / (ms * 1e-3) / 1e12}
    q, k, v = (rnd(1, H, n, hd) for _ in range(3))
    backend = "torch default"
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
            F.scaled_dot_product_attention(q, k, v)
            torch.cuda.synchronize(dev)
        backend = "cuDNN"
    except Exception:  # noqa: BLE001  (backend unavailable on this build)
        pass

    def sdpa(i):
        if backend == "cuDNN":
            with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
                return F.scaled_dot_product_attention(q, k, v)
        return F.scaled_dot_product_attention(q, k, v)
    ms = graph_ms(sdpa)
    out["attention"] = {"library": f"torch scaled_dot_product_attention ({backend})", "ms": ms,
                        "tflops": 4 * n * n * d / (ms * 1e-3) / 1e12}
    del x, gbuf, q, k, v
    torch.cuda.empty_cache()
    return out


def time_reuse(cfg_name, dev, reps=10):
    """Whole denoises under the reuse policies (host loop over the C ABI captured as one
    CUDA graph): ms per denoise and fresh model evaluations, for whole-velocity and
    core-residual reuse with period 2 and 3."""
    import torch
    from video_diffusion_transformer_03_b200 import h3b, synth
    from video_diffusion_transformer_03_b200.pipeline import DiTDenoiser
    cfg = synth.CONFIGS[cfg_name]
    model = DiTDenoiser(cfg, device=str(dev), gen_device=str(dev))
    x = synth.latent_noise(cfg, device=str(dev))
    res = {}
    for mode in ("velocity", "core"):
        for every in (2, 3):
            fresh = model.run_reuse(x, every, mode)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                model.run_reuse(x, every, mode)
            graph.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record()
            for _ in range(reps):
                graph.replay()
            e1.record()
            torch.cuda.synchronize(dev)
            del graph
            res[f"{mode}{every}"] = {"ms_per_denoise": e0.elapsed_time(e1) / reps,
                                     "fresh_evaluations": fresh, "steps": cfg.steps}
    h3b.sync_status()
    del model
    torch.cuda.empty_cache()
    return res


def time_int8_block(dev, peaks, reps=20):
    """One DiT block of the 512x512 workload on the int8 path (h3b_block_forward_int8)
    against the bf16 block (h3b_block_forward): CUDA graphs of `reps` blocks, the median of
    three alternating replays each."""
    import torch
    from video_diffusion_transformer_03_b200 import h3b, synth
    from video_diffusion_transformer_03_b200.pipeline import dims_of, grid_of
    cfg = synth.CONFIGS["dit512"]
    dims, grid = dims_of(cfg), grid_of(cfg)
    n = cfg.n_tokens
    p = {k: v.to(dev) for k, v in synth.block_params(cfg, 0, device=str(dev)).items()}
    mod = torch.empty((6, cfg.d), dtype=torch.float32, device=dev)
    h3b.adaln_modulation(p.pop("w_ada"), p.pop("b_ada"), synth.conditioning(cfg, str(dev)), mod)
    tq, wq = h3b.quantize_block_int8(p)
    w = h3b.make_block_weights(p)
    cs = torch.empty((n, cfg.head_dim // 2, 2), dtype=torch.float32, device=dev)
    h3b.rope_table(dims, grid, False, cs)
    x = synth.latent_noise(cfg, device=str(dev)).to(torch.bfloat16)
    h = torch.empty_like(x)
    ws8 = h3b.workspace(h3b.workspace_size_int8(dims, n), dev)
    ws = h3b.workspace(h3b.workspace_size(dims, n), dev)
    forms = {"int8": lambda: h3b.block_forward_int8(dims, w, wq, mod, cs, x, ws8),
             "bf16": lambda: h3b.block_forward(dims, w, mod, mod, cs, x, h, ws, True)}
    graphs = {}
    for name, fn in forms.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(reps):
                fn()
        graph.replay()
        graphs[name] = graph
    # the two forms' replays alternate, three each, and the median counts: single replays
    # of either differ by up to 20% with the clock under the power cap
    times = {name: [] for name in forms}
    for _ in range(3):
        for name, graph in graphs.items():
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize(dev)
            times[name].append(e0.elapsed_time(e1) / reps * 1e3)
    del graphs
    res = {name + "_block_us": sorted(t)[1] for name, t in times.items()}
    res.update({name + "_block_us_replays": [round(v, 1) for v in t] for name, t in times.items()})
    h3b.sync_status()
    del p, tq, x, ws8, ws
    torch.cuda.empty_cache()
    return res


def time_attention_forms(dev, peaks, reps=10):
    """Attention alone at the 512x512 (1,600 tokens) and 768x1344 (11,344 tokens) shapes,
    24 heads x 128, split schedule, in both kernel forms (one or two query tiles per CTA);
    CUDA-graph replays of `reps` launches."""
    import torch
    from video_diffusion_transformer_03_b200 import h3b
    g = torch.Generator(device=dev).manual_seed(5)
    ws = torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=dev)
    res = {}
    for n in (1600, 11344):
        d = 24 * 128
        qkv = torch.randn(n, 3 * d, generator=g, device=dev).to(torch.bfloat16)
        out = torch.empty(n, d, dtype=torch.bfloat16, device=dev)
        for name, v in (("two_tile", h3b.ATTN_TWO_TILES), ("one_tile", h3b.ATTN_ONE_TILE),
                        ("two_tile_poly", h3b.ATTN_TWO_TILES_POLY)):
            with h3b.attention_variant(v):
                for _ in range(3):
                    h3b.attention(qkv, 24, 128, out, ws=ws)
                torch.cuda.synchronize(dev)
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    for _ in range(reps):
                        h3b.attention(qkv, 24, 128, out, ws=ws)
            graph.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize(dev)
            del graph
            ms = e0.elapsed_time(e1) / reps
            tf = 4 * n * n * d / (ms * 1e-3) / 1e12
            res[f"{name}_{n}"] = {"us": ms * 1e3, "tflops": tf, "frac": tf / peaks["bf16_tflops"]}
        del qkv, out
    h3b.sync_status()
    torch.cuda.empty_cache()
    return res


def time_denoise(cfg_name, dev, reps, warm=1):
    """Device time of complete denoises of another workload (graph replays)."""
    import torch
    from video_diffusion_transformer_03_b200 import h3b, synth
    from video_diffusion_transformer_03_b200.pipeline import DiTDenoiser
    cfg = synth.CONFIGS[cfg_name]
    model = DiTDenoiser(cfg, device=str(dev), gen_device=str(dev))
    counts, _ = workload_counts(cfg, model.active)
    x = (synth.latent_state(cfg, device=str(dev)) if cfg.latent_channels
         else synth.latent_noise(cfg, device=str(dev)))
    for _ in range(warm):
        model.run(x)
    graph = model.capture(x)
    graph.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    h3b.sync_status()
    ms = e0.elapsed_time(e1) / reps
    del graph, model
    torch.cuda.empty_cache()
    return {"workload": workload_name(cfg), "ms_per_denoise": ms,
            "tokens_per_s": counts["tokens"] / (ms * 1e-3),
            "tflops": counts["flops"] / (ms * 1e-3) / 1e12, "denoises_timed": reps}


def time_int8_fc2(dev, peaks, reps=10):
    """The int8 row-scaled FC2 workload: quantise 8192 x 12288 activations, int8 GEMM
    against 3072 x 12288 int8 weights, dequantise + gated residual."""
    import torch
    from video_diffusion_transformer_03_b200 import h3b, synth
    c = synth.INT8_CONFIG
    inp = synth.int8_fc2_inputs(c, device=str(dev))
    M, K, N = c.M, c.K, c.n_out
    wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    wsc = torch.empty((N,), dtype=torch.float32, device=dev)
    h3b.quantize_rows(inp["w"], wq, wsc)
    aq = torch.empty((M, K), dtype=torch.int8, device=dev)
    rs = torch.empty((M,), dtype=torch.float32, device=dev)
    resid = inp["resid"]
    ws = torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=dev)
    run = lambda: h3b.fc2_int8_row(inp["act"], wq, wsc, None, inp["gate"], resid, aq, rs, None, ws=ws)
    q_only = lambda: h3b.quantize_rows(inp["act"], aq, rs)
    out = {}
    for name, fn in (("fc2_int8_row", run), ("quantize_rows", q_only)):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        out[name] = e0.elapsed_time(e1) / reps
    q_cold = time_cold(q_only, dev)
    h3b.sync_status()
    q_bytes = 3 * M * K + 4 * M
    int8_peak = 2 * peaks["bf16_tflops"]
    gemm_ms = max(out["fc2_int8_row"] - out["quantize_rows"], 1e-6)
    res = {"workload": f"fc2_int8_row M={M} K={K} N={N}", "ms": out["fc2_int8_row"],
           "tops_whole_call": 2 * M * N * K / (out["fc2_int8_row"] * 1e-3) / 1e12,
           "quantize_ms": out["quantize_rows"],
           "quantize_gbs": q_bytes / (out["quantize_rows"] * 1e-3) / 1e9,
           "quantize_hbm_frac": q_bytes / (out["quantize_rows"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
           "quantize_cold_ms": q_cold,
           "quantize_cold_hbm_frac": q_bytes / (q_cold * 1e-3) / 1e9 / peaks["hbm_gbs"],
           "int8_gemm_tops": 2 * M * N * K / (gemm_ms * 1e-3) / 1e12,
           "int8_gemm_frac": 2 * M * N * K / (gemm_ms * 1e-3) / 1e12 / int8_peak,
           "int8_peak_tops": int8_peak,
           "int8_peak_note": "bf16 burst peak x 2 (nominal ratio); bf16 peak from "
                             + peaks.get("source", "MEASURED_PEAKS.json or the fallback")}
    del inp, wq, aq, resid
    torch.cuda.empty_cache()
    return res


def time_grouped_fc2(dev, peaks, reps=20):
    """The int8 MLP's FC2 at the 512x512 shape (M = 1600 tokens, K = 12288, N = 3072): the
    grouped int8 GEMM alone (h3b_gemm_i8_grouped with the kernel scratch, as the int8 block
    runs it; activations quantised per row and 1024 channels, weights per output channel)
    with the gated-residual epilogue, CUDA events around `reps` launches."""
    import torch
    from video_diffusion_transformer_03_b200 import h3b
    M, K, N = 1600, 12288, 3072
    g = torch.Generator(device=dev).manual_seed(5)
    a = torch.nn.functional.gelu(torch.randn(M, K, generator=g, device=dev),
                                 approximate="tanh").to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    aq = torch.empty((M, K), dtype=torch.int8, device=dev)
    asc = torch.empty((M, K // 1024), dtype=torch.float32, device=dev)
    h3b.quantize_groups(a, aq, asc)
    wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    wsc = torch.empty((N,), dtype=torch.float32, device=dev)
    h3b.quantize_rows(w, wq, wsc)
    bias = torch.zeros(N, dtype=torch.bfloat16, device=dev)
    gate = torch.ones(N, device=dev)
    resid = torch.randn(M, N, generator=g, device=dev).to(torch.bfloat16)
    scratch = torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=dev)
    run = lambda: h3b.gemm_i8_grouped(aq, asc, wq, wsc, bias, gate, resid, ws=scratch)
    for _ in range(3):
        run()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize(dev)
    h3b.sync_status()
    ms = e0.elapsed_time(e1) / reps
    tops = 2 * M * N * K / (ms * 1e-3) / 1e12
    res = {"workload": f"grouped int8 FC2 M={M} K={K} N={N}", "us": ms * 1e3, "tops": tops,
           "frac_int8": tops / (2 * peaks["bf16_tflops"])}
    del a, w, aq, wq, resid
    torch.cuda.empty_cache()
    return res


def time_token_pairing(dev, peaks, reps=20):
    import torch
    from video_diffusion_transformer_03_b200 import h3b, synth
    cfg = synth.CONFIGS["dit768x1344"]
    t, h, w = cfg.grid
    n, nr, d = cfg.n_tokens, cfg.n_video_reduced + cfg.n_audio, cfg.d
    x = torch.randn(n, d, device=dev).to(torch.bfloat16)
    red = torch.empty(nr, d, dtype=torch.bfloat16, device=dev)
    back = torch.empty_like(x)
    res = {}
    for name, fn, nbytes in (
            ("pair", lambda: h3b.token_reduce(h3b.PAIR, x, red, None, t, h, w, cfg.n_audio),
             2 * (n * d + nr * d)),
            ("unpair_bypass", lambda: h3b.token_reduce(h3b.UNPAIR, red, back, x, t, h, w, cfg.n_audio),
             2 * (nr * d + 2 * n * d))):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / reps
        cold = time_cold(fn, dev)
        res[name] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                     "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "cold_ms": cold,
                     "cold_hbm_frac": nbytes / (cold * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    h3b.sync_status()
    res["shape"] = f"{cfg.name} stream: {n} tokens x {d} bf16 -> {nr} tokens"
    return res


class Replicas:
    """The N-GPU run: one process per GPU (torchrun sets RANK / WORLD_SIZE), each an
    independent replica of the whole denoise; nothing crosses GPUs on the data path.  The
    only collectives are the timing barrier and the max of the device times over ranks."""

    def __init__(self, backend="nccl", device=None, timeout_s=300):
        import datetime
        import torch.distributed as dist
        self.dist = dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.backend = backend
        self.device = device
        if self.world > 1:
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            if self.backend == "nccl":
                self.dist.barrier(device_ids=[self.device.index])
            else:
                self.dist.barrier()

    def max(self, v):
        """Max of a per-rank float over all ranks (the slowest replica sets the time)."""
        if self.world == 1:
            return float(v)
        import torch
        t = torch.tensor([float(v)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def throughput(self, units_per_step, steps, ms_max):
        """Whole-job rate: every rank processed units_per_step per step."""
        return units_per_step * steps * self.world / (ms_max * 1e-3)

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def run_gpu(args):
    import torch
    from video_diffusion_transformer_03_b200 import h3b, synth
    from video_diffusion_transformer_03_b200.pipeline import DiTDenoiser

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    replicas = Replicas("nccl", dev)
    world, rank = replicas.world, replicas.rank
    barrier, max_over_ranks = replicas.barrier, replicas.max

    peaks, peak_src = load_peaks()
    if args.attn_variant:
        h3b.set_attention_variant(args.attn_variant)
    if args.kernel in ("fc2_int8_row", "token_pairing", "grouped_fc2_int8"):  # outside the block
        res = {"fc2_int8_row": time_int8_fc2, "token_pairing": time_token_pairing,
               "grouped_fc2_int8": time_grouped_fc2}[args.kernel](dev, peaks, reps=args.reps)
        if rank == 0:
            print(json.dumps({"kernel_only": args.kernel, **res}), flush=True)
        return
    cfg = synth.CONFIGS[args.config]
    model = DiTDenoiser(cfg, device=str(dev), gen_device=str(dev))
    counts, n_active = workload_counts(cfg, model.active)
    if args.kernel:
        res = time_kernels(model, cfg, peaks, {"blocks": n_active * cfg.run_steps},
                           reps=args.reps, only=args.kernel)
        if rank == 0:
            print(json.dumps({"kernel_only": args.kernel, "config": cfg.name, **res}), flush=True)
        return
    x0 = synth.latent_noise(cfg, device=str(dev))
    x = x0.clone()
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        model.run(x)
    h3b.sync_status()
    graph = None
    launches_per_denoise = None
    if not args.no_graph:
        c0 = h3b.launch_count()
        graph = model.capture(x)
        launches_per_denoise = h3b.launch_count() - c0
        for _ in range(2):
            graph.replay()
        h3b.sync_status()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)

    # ---- timed region: K complete denoises, device time
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(gpu_id)
    launches0 = h3b.launch_count()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            model.run(x)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    launches = h3b.launch_count() - launches0
    if graph is not None:  # graph replays launch the captured kernels without host calls
        launches = launches_per_denoise * args.steps
    clk = clocks.stop()
    barrier()
    h3b.sync_status()
    ms = max_over_ranks(e0.elapsed_time(e1))
    ms_step = ms / args.steps
    value = replicas.throughput(counts["tokens"], args.steps, ms)
    tflops = counts["flops"] * args.steps * world / (ms * 1e-3) / 1e12

    # ---- end to end through the host-buffer entry point (copies inside the timed region):
    # batches of requests, each uploaded from pinned host memory and its result downloaded,
    # the copies overlapped with the neighbouring requests' compute
    e2e_steps = max(1, args.steps // 2)
    batch = min(10, e2e_steps)
    n_batches = (e2e_steps + batch - 1) // batch
    e2e_steps = n_batches * batch
    host_in = torch.stack([synth.latent_noise(cfg)] * batch).pin_memory()
    host_out = torch.empty_like(host_in).pin_memory()
    state2 = torch.empty((2,) + tuple(x0.shape), dtype=torch.float32, device=dev)
    model.run_host_pipelined(host_in[:2], host_out[:2], state2)
    barrier()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e2.record(stream)
    for _ in range(n_batches):
        model.run_host_pipelined(host_in, host_out, state2)
    e3.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e2.elapsed_time(e3))
    nbytes = host_in[0].numel() * host_in.element_size()
    e2e = {"value": replicas.throughput(counts["tokens"], e2e_steps, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
           "ms_per_step": e2e_ms / e2e_steps,
           "api": f"h3b_denoise_host_pipelined, {batch} requests per call"}

    breakdown = None
    roofline = None
    if not args.no_breakdown:
        breakdown = time_kernels(model, cfg, peaks, {"blocks": n_active * cfg.run_steps})
        dom = max(breakdown, key=lambda k: breakdown[k]["ms_per_step"])
        b = breakdown[dom]
        tr = NCU_TRAFFIC.get(dom)
        traffic = tr["bytes"] if tr and tr.get("src_sha") == src_hash(tr["src"]) else None
        roofline = {"kernel": dom, "bound": b["bound"], "achieved": b["achieved"],
                    "peak": b["peak"], "unit": b["unit"], "frac": b["frac"], "traffic": traffic,
                    "peak_source": f"{peak_src} burst"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random-init weights and latent noise)",
            "config": {"workload": workload_name(cfg), "tokens": cfg.n_tokens,
                       "blocks_executed_per_denoise": counts["blocks"],
                       "block_tokens_per_step": counts["tokens"],
                       "flops_per_step": counts["flops"],
                       "l2": "no flush: each pass streams "
                             f"{sum(p['w_qkv'].numel() + p['w_o'].numel() + p['w_fc1'].numel() + p['w_fc2'].numel() for p in model.params) * 2 / 1e9:.2f}"
                             " GB of weights, more than the 126 MB L2",
                       "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                       "launch": "CUDA graph of one complete denoise, replayed" if graph
                                 is not None else "host launches"},
            "tflops": tflops,
            "tensor_frac": tflops / world / peaks["bf16_tflops_sustained"],
            "tensor_frac_peak": f"{peak_src} sustained bf16 {peaks['bf16_tflops_sustained']} TFLOP/s",
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches, "clocks": clk}
    if breakdown:
        line["kernels"] = {k: {kk: (round(vv, 5) if isinstance(vv, float) else vv)
                               for kk, vv in v.items()} for k, v in breakdown.items()}
    if rank == 0 and world == 1 and not args.no_also:
        del graph
        graph = None
        also = {}
        for name, reps in (("dit512_tokred", 20), ("dit768x1344", 2), ("dit512_latent", 20),
                           ("dit512_qknorm", 20)):
            if name != args.config:
                also[name] = time_denoise(name, dev, reps)
        also["reuse_dit512"] = time_reuse("dit512", dev)
        also["int8_block_dit512"] = time_int8_block(dev, peaks)
        also["attention_forms"] = time_attention_forms(dev, peaks)
        also["fc2_int8_row"] = time_int8_fc2(dev, peaks)
        also["grouped_fc2_int8"] = time_grouped_fc2(dev, peaks)
        also["token_pairing"] = time_token_pairing(dev, peaks)
        also["gemm_widths"] = time_gemm_widths(dev, peaks)
        try:  # context only: a library that cannot run here must not cost the bench line
            also["libraries_same_shapes"] = time_library_same_shapes(model, cfg, dev)
        except Exception as exc:  # noqa: BLE001
            also["libraries_same_shapes"] = {"error": f"{type(exc).__name__}: {exc}"}
        line["also"] = also
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(cfg)
    del graph
    replicas.close()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_command(n: int, argv, port: int):
    """The torch.distributed.run command that starts this script as n local ranks."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__)] + list(argv)


def relaunch_as_ranks(n: int, argv, timeout_s: float = 3600.0) -> int:
    """Run this script as n ranks (one process per GPU) and return the launcher's status.
    The ranks' process group has its own short timeout; this bound sits well above it."""
    cmd = launch_command(n, argv, _free_port())
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    try:
        return subprocess.run(cmd, env=env, timeout=timeout_s).returncode
    except subprocess.TimeoutExpired:
        return 124


def run_replica_check(args):
    """The N-rank plumbing on CPU (gloo): barrier, max of a per-rank time, job rate; rank 0
    prints one line with what every rank saw."""
    import torch
    reps = Replicas("gloo", torch.device("cpu"), timeout_s=60)
    reps.barrier()
    ms = reps.max(10.0 + 5.0 * reps.rank)
    value = reps.throughput(1000, 4, ms)
    seen = {"rank": reps.rank, "world": reps.world, "max_ms": ms, "value": value}
    views = [seen]
    if reps.world > 1:
        views = [None] * reps.world
        reps.dist.all_gather_object(views, seen)
    reps.barrier()
    reps.close()
    if reps.rank == 0:
        print(json.dumps({"replica_check": True, "ranks": views}), flush=True)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl != "reference":
        sys.exit(relaunch_as_ranks(args.gpus, argv))
    if args.replica_check:
        run_replica_check(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
