"""Write the oracle's reference trajectories for the 512x512-shaped denoising workloads.

    python tests/golden/make_golden.py [name ...]

Calls only oracle/ (float64) and the seeded input generators; no CUDA code is involved.
For each workload it stores, for a fixed sample of token rows, the state after the first
Euler step and after the last one, plus the oracle's layer-thinning mask.  The parity
tests recompute the same rows on the GPU from the same seeded inputs.  The reuse entries
("<workload>_reuse_<velocity|core><period>") store the final state of a whole denoise
under that reuse policy.
"""
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import workloads  # noqa: E402
from video_diffusion_transformer_03_b200 import synth  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))
NAMES = ("dit512", "dit512_tokred", "dit256_halved", "dit512_qknorm", "dit512_latent")
REUSE = {"dit512_reuse_velocity2": ("dit512", "velocity", 2),
         "dit512_reuse_core3": ("dit512", "core", 3)}


def sample_rows(cfg) -> np.ndarray:
    nv, n = cfg.n_video, cfg.n_tokens
    rows = np.concatenate([np.arange(0, 4), np.linspace(4, nv - 3, 32).astype(int),
                           np.arange(nv - 2, nv + 2), np.linspace(nv + 2, n - 1, 8).astype(int)])
    return np.unique(rows)


def path(name: str) -> str:
    return os.path.join(HERE, f"{name}_oracle.npz")


def make(name: str) -> None:
    cfg = synth.CONFIGS[name]
    f32 = lambda t: t.float().numpy()
    blocks = [{k: f32(v) for k, v in synth.block_params(cfg, b).items()}
              for b in range(cfg.n_blocks)]
    final = {k: f32(v) for k, v in synth.final_params(cfg).items()}
    c = f32(synth.conditioning(cfg)).astype(np.float64)
    x0 = f32(synth.latent_noise(cfg)).astype(np.float64)
    t0 = time.time()
    trace = []
    if cfg.latent_channels:
        heads = {k: f32(v).astype(np.float64) for k, v in synth.head_params(cfg).items()}
        x0 = f32(synth.latent_state(cfg)).astype(np.float64)
        workloads.denoise_latent(cfg, blocks, final, heads, c, x0, trace=trace)
    else:
        workloads.denoise(cfg, blocks, final, c, x0, trace=trace)
    mods = workloads.modulation_vectors(cfg, blocks, c)
    mask = workloads.active_mask(cfg, mods)
    rows = sample_rows(cfg)
    np.savez_compressed(path(name), rows=rows, step1=trace[0][rows].astype(np.float32),
                        final=trace[-1][rows].astype(np.float32),
                        active=np.ones(cfg.n_blocks, bool) if mask is None else mask)
    print(f"{name}: {len(trace)} steps, {time.time() - t0:.1f} s -> {path(name)}")


def make_reuse(name: str) -> None:
    base, mode, every = REUSE[name]
    cfg = synth.CONFIGS[base]
    f32 = lambda t: t.float().numpy()
    blocks = [{k: f32(v) for k, v in synth.block_params(cfg, b).items()}
              for b in range(cfg.n_blocks)]
    final = {k: f32(v) for k, v in synth.final_params(cfg).items()}
    c = f32(synth.conditioning(cfg)).astype(np.float64)
    x0 = f32(synth.latent_noise(cfg)).astype(np.float64)
    t0 = time.time()
    out = workloads.denoise_reuse(cfg, blocks, final, c, x0, every, mode)
    rows = sample_rows(cfg)
    np.savez_compressed(path(name), rows=rows, final=out[rows].astype(np.float32))
    print(f"{name}: {time.time() - t0:.1f} s -> {path(name)}")


if __name__ == "__main__":
    for n in (sys.argv[1:] or NAMES + tuple(REUSE)):
        make_reuse(n) if n in REUSE else make(n)
