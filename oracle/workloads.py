"""Oracle runs of whole workloads from plain numpy inputs (test infrastructure only).

Takes the seeded parameters as numpy arrays (bf16 values upcast), computes the oracle's
own AdaLN vectors, layer mask and positions, and runs the oracle denoising loop or one
block.  ``cfg`` is any object with the workload fields (d, n_heads, head_dim, rope_split,
rope_theta, ln_eps, grid, n_audio, steps, run_steps, reduce_after, active_count,
n_blocks, rope_halved, unpair_bypass).
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np

from . import oracle as O


def modulation_vectors(cfg, blocks: List[Dict[str, np.ndarray]], c: np.ndarray):
    return np.stack([O.adaln_modulation(b["w_ada"], b["b_ada"], c, cfg.d) for b in blocks])


def final_vectors(cfg, final: Dict[str, np.ndarray], c: np.ndarray):
    return O.final_modulation(final["w_fin"], final["b_fin"], c, cfg.d)


def active_mask(cfg, mods) -> Optional[np.ndarray]:
    if cfg.active_count >= cfg.n_blocks:
        return None
    return O.layer_mask(mods, cfg.active_count)


def denoise(cfg, blocks, final, c, x0, run_steps: Optional[int] = None, dt=np.float64,
            trace: Optional[list] = None) -> np.ndarray:
    mods = modulation_vectors(cfg, blocks, c)
    fm = final_vectors(cfg, final, c)
    return O.denoise(x0, blocks, mods, fm, cfg.grid, cfg.n_audio, cfg.n_heads, cfg.rope_split,
                     cfg.rope_theta, cfg.ln_eps, cfg.steps,
                     cfg.run_steps if run_steps is None else run_steps,
                     active=active_mask(cfg, mods), reduce_after=cfg.reduce_after,
                     halved=cfg.rope_halved, unpair_bypass=cfg.unpair_bypass, dt=dt, trace=trace)


def block(cfg, params, c, x, next_params=None, rows=None, dt=np.float64):
    """One block on x [N, d] with its own modulation vectors; h_next uses next_params'."""
    mod = O.adaln_modulation(params["w_ada"], params["b_ada"], c, cfg.d)
    mod_next = None
    if next_params is not None:
        mod_next = O.adaln_modulation(next_params["w_ada"], next_params["b_ada"], c, cfg.d)
    pos = O.rope_positions(cfg.grid, cfg.n_audio, halved=cfg.rope_halved)
    return O.block_forward(x, params, mod, pos, cfg.n_heads, cfg.rope_split, cfg.rope_theta,
                           cfg.ln_eps, mod_next=mod_next, rows=rows, dt=dt)


def denoise_reuse(cfg, blocks, final, c, x0, every: int, mode: str, dt=np.float64) -> np.ndarray:
    """A whole denoise of cfg.steps Euler steps under whole-velocity ("velocity") or
    core-residual ("core") reuse with the given period."""
    mods = modulation_vectors(cfg, blocks, c)
    fm = final_vectors(cfg, final, c)
    fn = O.denoise_velocity_reuse if mode == "velocity" else O.denoise_core_reuse
    return fn(x0, blocks, mods, fm, cfg.grid, cfg.n_audio, cfg.n_heads, cfg.rope_split,
              cfg.rope_theta, cfg.ln_eps, cfg.steps, every, active=active_mask(cfg, mods),
              reduce_after=cfg.reduce_after, halved=cfg.rope_halved,
              unpair_bypass=cfg.unpair_bypass, dt=dt)


def denoise_latent(cfg, blocks, final, heads, c, lat0, run_steps: Optional[int] = None,
                   dt=np.float64, trace: Optional[list] = None) -> np.ndarray:
    """The Euler loop on the per-token latent (patch embedding, blocks, final heads)."""
    mods = modulation_vectors(cfg, blocks, c)
    fm = final_vectors(cfg, final, c)
    steps = cfg.run_steps if run_steps is None else run_steps
    lat = lat0
    for i in range(steps):
        lat = O.denoise_latent(lat, blocks, mods, fm, heads, cfg.grid, cfg.n_audio,
                               cfg.n_heads, cfg.rope_split, cfg.rope_theta, cfg.ln_eps,
                               cfg.steps, 1, active=active_mask(cfg, mods),
                               reduce_after=cfg.reduce_after, halved=cfg.rope_halved,
                               unpair_bypass=cfg.unpair_bypass, dt=dt, first_step=i)
        if trace is not None:
            trace.append(lat.copy())
    return lat
