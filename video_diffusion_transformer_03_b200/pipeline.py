"""Device-resident synthetic DiT denoiser driven through the C ABI.

Holds a workload's bf16 block weights, the AdaLN modulation vectors (computed on the GPU
by h3b_adaln_modulation), the layer-thinning mask and the step workspace, and runs Euler
steps with h3b_denoise_step / h3b_denoise_host.  No arithmetic of the method happens in
Python.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import h3b, synth
from .synth import DiTConfig


def dims_of(cfg: DiTConfig) -> h3b.Dims:
    return h3b.make_dims(cfg.d, cfg.n_heads, cfg.head_dim, cfg.d_ff, cfg.c_dim, cfg.rope_split,
                         cfg.rope_theta, cfg.ln_eps)


def grid_of(cfg: DiTConfig) -> h3b.Grid:
    t, h, w = cfg.grid
    return h3b.make_grid(t, h, w, cfg.n_audio, cfg.rope_halved)


class DiTDenoiser:
    """fold=True (default) folds each block's two AdaLN modulations into its QKV and FC1
    weights once (h3b_fold_adaln), so the step runs without LayerNorm passes; fold=False
    keeps the LayerNorm + AdaLN kernel between the projections."""

    def __init__(self, cfg: DiTConfig, device: str = "cuda", gen_device: str = "cpu",
                 keep_host_params: bool = False, fold: bool = True):
        self.cfg = cfg
        self.fold = fold
        self.device = torch.device(device)
        self.dims = dims_of(cfg)
        self.grid = grid_of(cfg)
        self.host_params = [] if keep_host_params else None
        self.params = []
        self.mods = torch.empty((cfg.n_blocks, 6, cfg.d), dtype=torch.float32, device=self.device)
        self.c = synth.conditioning(cfg, gen_device).to(self.device)
        for b in range(cfg.n_blocks):
            p = synth.block_params(cfg, b, device=gen_device)
            if keep_host_params:
                self.host_params.append({k: v.cpu() for k, v in p.items()})
            pd = {k: v.to(self.device) for k, v in p.items()}
            del p
            h3b.adaln_modulation(pd.pop("w_ada"), pd.pop("b_ada"), self.c, self.mods[b])
            if fold:
                pd.update(h3b.fold_block(pd, self.mods[b]))
            self.params.append(pd)
        self.weights = [h3b.make_block_weights(p) for p in self.params]
        fin = synth.final_params(cfg, gen_device)
        self.host_final = {k: v.cpu() for k, v in fin.items()} if keep_host_params else None
        self.final_mod = torch.empty((2, 2, cfg.d), dtype=torch.float32, device=self.device)
        for s in range(2):
            h3b.adaln_modulation(fin["w_fin"][s].contiguous().to(self.device),
                                 fin["b_fin"][s].contiguous().to(self.device), self.c,
                                 self.final_mod[s])
        self.active: Optional[list] = None
        if cfg.active_count < cfg.n_blocks:
            mask = h3b.layer_mask(self.mods.cpu().numpy(), cfg.active_count)
            self.active = [bool(m) for m in mask]
        self.reduce = cfg.reduce_after > 0
        self.latent = cfg.latent_channels > 0
        if self.latent:
            # patch embedding and heads per stream; each head gets its stream's final AdaLN
            # folded in (the blocks must be folded too)
            if not fold:
                raise ValueError("the latent step runs the folded block form")
            hp = {k: v.to(self.device) for k, v in synth.head_params(cfg, gen_device).items()}
            self.host_heads = {k: v.cpu() for k, v in hp.items()} if keep_host_params else None
            self.heads_t = {"w_patch": [hp["w_patch"][s].contiguous() for s in range(2)],
                            "b_patch": [hp["b_patch"][s].contiguous() for s in range(2)],
                            "w_head_fold": [], "c_head": [], "dv_head": []}
            for st in range(2):
                w, b = hp["w_head"][st].contiguous(), hp["b_head"][st].contiguous()
                wo = torch.empty_like(w)
                c = torch.empty(w.shape[0], dtype=torch.float32, device=self.device)
                dv = torch.empty_like(c)
                h3b.fold_adaln(w, b, self.final_mod[st, 0].contiguous(),
                               self.final_mod[st, 1].contiguous(), wo, c, dv)
                self.heads_t["w_head_fold"].append(wo)
                self.heads_t["c_head"].append(c)
                self.heads_t["dv_head"].append(dv)
            self.heads = h3b.make_latent_heads(cfg.latent_channels, self.heads_t)
            nbytes = h3b.denoise_latent_workspace_size(self.dims, self.grid, self.reduce,
                                                       cfg.latent_channels)
        else:
            nbytes = h3b.denoise_workspace_size(self.dims, self.grid, self.reduce)
        self.ws = h3b.workspace(nbytes, self.device)

    @property
    def n_tokens(self) -> int:
        return self.cfg.n_tokens

    def sigmas(self, i: int):
        s = self.cfg.steps
        return 1.0 - i / s, 1.0 - (i + 1) / s

    def step(self, x_state: torch.Tensor, i: int, stream=None) -> None:
        """One Euler step on x_state: [N, d] model-space state, or the [N, C] latent for a
        latent workload."""
        sg, sn = self.sigmas(i)
        if self.latent:
            h3b.denoise_step_latent(self.dims, self.grid, self.weights, self.active, self.mods,
                                    self.heads, self.cfg.reduce_after, self.cfg.unpair_bypass,
                                    sg, sn, x_state, self.ws, stream)
            return
        h3b.denoise_step(self.dims, self.grid, self.weights, self.active, self.mods,
                         self.final_mod, self.cfg.reduce_after, self.cfg.unpair_bypass, sg, sn,
                         x_state, self.ws, stream)

    def run(self, x_state: torch.Tensor, n_run: Optional[int] = None, stream=None) -> None:
        for i in range(self.cfg.run_steps if n_run is None else n_run):
            self.step(x_state, i, stream)

    def run_reuse(self, x_state: torch.Tensor, every: int, mode: str = "velocity",
                  stream=None) -> int:
        """A whole denoise under a reuse policy (host policy over the C ABI): the steps
        h3b_reuse_schedule marks fresh run the model and keep its velocity ("velocity") or
        its core residual ("core"); the others reuse it.  Returns the fresh step count."""
        if mode not in ("velocity", "core"):
            raise ValueError(mode)
        steps = self.cfg.steps
        fresh = h3b.reuse_schedule(steps, every)
        held = getattr(self, "_reuse_buf", None)
        if held is None or held.shape != x_state.shape:
            held = self._reuse_buf = torch.empty_like(x_state)
        for i in range(steps):
            sg, sn = self.sigmas(i)
            if fresh[i]:
                h3b.denoise_step_keep(self.dims, self.grid, self.weights, self.active, self.mods,
                                      self.final_mod, self.cfg.reduce_after,
                                      self.cfg.unpair_bypass, sg, sn, x_state,
                                      held if mode == "velocity" else None,
                                      held if mode == "core" else None, self.ws, stream)
            elif mode == "velocity":
                h3b.euler_velocity(held, sg, sn, x_state, stream)
            else:
                h3b.euler_core_reuse(held, self.cfg.n_video, self.cfg.ln_eps, self.final_mod,
                                     sg, sn, x_state, stream)
        return int(fresh.sum())

    def capture(self, x_state: torch.Tensor, n_run: Optional[int] = None) -> torch.cuda.CUDAGraph:
        """Record a whole denoise of x_state (in place) as one CUDA graph; replaying it
        relaunches every kernel of every Euler step without host work.  Call run() once
        first on this device (the library sets kernel attributes on first use)."""
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.run(x_state, n_run)
        return graph

    def run_host_pipelined(self, x_host_in: torch.Tensor, x_host_out: torch.Tensor,
                           x_state_dev2: torch.Tensor, n_run: Optional[int] = None,
                           stream=None) -> None:
        """Whole denoises of a batch of host latents [requests, n_tokens, d], copies
        overlapped with compute (h3b_denoise_host_pipelined)."""
        h3b.denoise_host_pipelined(self.dims, self.grid, self.weights, self.active, self.mods,
                                   self.final_mod, self.cfg.reduce_after,
                                   self.cfg.unpair_bypass, self.cfg.steps, 0,
                                   self.cfg.run_steps if n_run is None else n_run, x_host_in,
                                   x_host_out, x_state_dev2, self.ws, stream)

    def run_host(self, x_host_in: torch.Tensor, x_host_out: torch.Tensor,
                 x_state_dev: torch.Tensor, n_run: Optional[int] = None, stream=None) -> None:
        h3b.denoise_host(self.dims, self.grid, self.weights, self.active, self.mods,
                         self.final_mod, self.cfg.reduce_after, self.cfg.unpair_bypass,
                         self.cfg.steps, 0, self.cfg.run_steps if n_run is None else n_run,
                         x_host_in, x_host_out, x_state_dev, self.ws, stream)
