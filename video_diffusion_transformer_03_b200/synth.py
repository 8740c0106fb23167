"""Seeded synthetic inputs for the DiT-block denoising path.

This module only draws numbers: Gaussian parameters, conditioning vectors and latent
noise, rounded once to bf16.  It holds none of the method's arithmetic (no
normalisation, projection, rotation, attention, quantisation or update), so the CUDA
path and the CPU oracle can both consume its tensors without sharing any step of the
computation.

Draw recipe (the same on every machine for a given torch version):
  * every tensor has its own generator, seeded from (config seed, block index, tensor
    name), so any subset of blocks can be drawn without drawing the others;
  * parameters ~ N(0, 0.02), conditioning vector c ~ N(0, 1), tokens / latent noise
    ~ N(0, 1), all drawn in fp32 and rounded to bf16 (round-to-nearest-even);
  * the int8-FC2 activations are GELU(z) of z ~ N(0, 1) (torch's tanh-form GELU, used
    here only to shape the input distribution), rounded to bf16.

Workload shapes follow the pages' 512x512 / 22-frame and 768x1344 renders with a
32-pixel token pitch (a 256x256 render has an 8x8 spatial token grid: h3-metal README,
"Choose resolution and duration").
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import torch

__all__ = ["DiTConfig", "Int8Config", "CONFIGS", "INT8_CONFIG", "block_params",
           "final_params", "conditioning", "latent_noise", "int8_fc2_inputs",
           "BLOCK_TENSORS"]

PARAM_STD = 0.02

# Order of the per-block tensors; the index is part of each tensor's seed.
BLOCK_TENSORS = ("w_qkv", "b_qkv", "w_o", "b_o", "w_fc1", "b_fc1", "w_fc2", "b_fc2",
                 "w_ada", "b_ada", "q_norm", "k_norm")
QK_GAIN_STD = 0.1  # Q/K RMSNorm gains ~ 1 + N(0, 0.1)
_FINAL_TENSORS = ("w_fin", "b_fin")
_HEAD_TENSORS = ("w_patch", "b_patch", "w_head", "b_head")
_COND_IDX = 100
_NOISE_IDX = 101
_INT8_IDX = {"act": 200, "w": 201, "gate": 202, "resid": 203, "bias": 204}


@dataclass(frozen=True)
class DiTConfig:
    """Shape of one DiT denoising workload."""
    name: str
    d: int
    n_heads: int
    head_dim: int
    d_ff: int
    c_dim: int
    rope_split: Tuple[int, int, int]
    n_blocks: int
    grid: Tuple[int, int, int]          # video token grid (t, h, w)
    n_audio: int
    steps: int                          # intervals of the linear sigma grid
    run_steps: int                      # how many of those Euler steps are run
    seed: int
    rope_theta: float = 10000.0
    ln_eps: float = 1e-6
    reduce_after: int = -1              # pair tokens after this many executed blocks
    n_active: Optional[int] = None      # layer thinning: active blocks (None = all)
    rope_halved: bool = False           # spatial RoPE coordinates halved
    unpair_bypass: bool = True          # bypass restore (False: duplicate)
    qk_norm: bool = False               # per-head Q/K RMSNorm gains in every block
    latent_channels: int = 0            # > 0: the state is a per-token latent of this many
                                        # channels, with patch embedding and final heads

    @property
    def n_video(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def n_tokens(self) -> int:
        return self.n_video + self.n_audio

    @property
    def n_video_reduced(self) -> int:
        t, h, w = self.grid
        return t * h * (w // 2)

    @property
    def active_count(self) -> int:
        return self.n_blocks if self.n_active is None else self.n_active


@dataclass(frozen=True)
class Int8Config:
    name: str
    M: int
    K: int
    n_out: int
    seed: int
    with_bias: bool = False


def _c(name, **kw):
    return DiTConfig(name=name, **kw)


_BIG = dict(d=3072, n_heads=24, head_dim=128, d_ff=12288, c_dim=256, rope_split=(32, 48, 48))

CONFIGS: Dict[str, DiTConfig] = {
    # 1 block, d=256, 4 heads x 64, MLP 1024, grid 2x4x4 + 8 audio, one Euler step 1 -> 0.75
    "tiny": _c("tiny", d=256, n_heads=4, head_dim=64, d_ff=1024, c_dim=256,
               rope_split=(16, 24, 24), n_blocks=1, grid=(2, 4, 4), n_audio=8,
               steps=4, run_steps=1, seed=0),
    # 512x512, 22 frames: 6 latent frames of 16x16 tokens + 64 audio tokens, 8 blocks, 4 steps
    "dit512": _c("dit512", n_blocks=8, grid=(6, 16, 16), n_audio=64, steps=4, run_steps=4,
                 seed=1, **_BIG),
    # same with horizontal token pairing after the 3rd executed block, 6 of 8 blocks active
    "dit512_tokred": _c("dit512_tokred", n_blocks=8, grid=(6, 16, 16), n_audio=64, steps=4,
                        run_steps=4, seed=2, reduce_after=3, n_active=6, **_BIG),
    # small-grid variant of the above: 256x256-class grid with halved spatial RoPE
    # coordinates, token reduction off at this size (the pages keep it off at 256^2)
    "dit256_halved": _c("dit256_halved", n_blocks=8, grid=(6, 8, 8), n_audio=64, steps=4,
                        run_steps=4, seed=2, n_active=6, rope_halved=True, **_BIG),
    # 768x1344: 11 latent frames of 24x42 tokens + 256 audio tokens, 50 blocks, 4 steps
    "dit768x1344": _c("dit768x1344", n_blocks=50, grid=(11, 24, 42), n_audio=256, steps=4,
                      run_steps=4, seed=3, **_BIG),
    # the 512x512 workload with per-head Q/K RMSNorm before RoPE in every block (the
    # QKV-tile RMS normalisation of the pages' int8 path); same weights as dit512 otherwise
    "dit512_qknorm": _c("dit512_qknorm", n_blocks=8, grid=(6, 16, 16), n_audio=64, steps=4,
                        run_steps=4, seed=1, qk_norm=True, **_BIG),
    # the 512x512 workload on a 128-channel per-token latent: patch embedding and the
    # final heads (AdaLN folded into the head) around the same 8 blocks
    "dit512_latent": _c("dit512_latent", n_blocks=8, grid=(6, 16, 16), n_audio=64, steps=4,
                        run_steps=4, seed=1, latent_channels=128, **_BIG),
    "tiny_latent": _c("tiny_latent", d=256, n_heads=4, head_dim=64, d_ff=1024, c_dim=256,
                      rope_split=(16, 24, 24), n_blocks=1, grid=(2, 4, 4), n_audio=8,
                      steps=4, run_steps=2, seed=0, latent_channels=128),
    # the tiny workload with Q/K RMSNorm
    "tiny_qknorm": _c("tiny_qknorm", d=256, n_heads=4, head_dim=64, d_ff=1024, c_dim=256,
                      rope_split=(16, 24, 24), n_blocks=1, grid=(2, 4, 4), n_audio=8,
                      steps=4, run_steps=1, seed=0, qk_norm=True),
}

INT8_CONFIG = Int8Config(name="fc2_int8_row", M=8192, K=12288, n_out=3072, seed=4)


def _seed(seed: int, block: int, idx: int) -> int:
    return (seed * 1_000_003 + (block + 1) * 10_007 + idx * 101) & 0x7FFF_FFFF_FFFF


def _randn(shape, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _param(shape, seed, block, idx, device, std=PARAM_STD) -> torch.Tensor:
    return (_randn(shape, _seed(seed, block, idx), device) * std).to(torch.bfloat16)


def block_params(cfg: DiTConfig, block: int, device="cpu") -> Dict[str, torch.Tensor]:
    """Parameters of one block, weights as [out, in] row-major bf16; with cfg.qk_norm also
    the Q/K RMSNorm gains q_norm, k_norm [head_dim] (1 + N(0, 0.1), bf16-valued fp32)."""
    d, f, c = cfg.d, cfg.d_ff, cfg.c_dim
    shapes = {"w_qkv": (3 * d, d), "b_qkv": (3 * d,), "w_o": (d, d), "b_o": (d,),
              "w_fc1": (f, d), "b_fc1": (f,), "w_fc2": (d, f), "b_fc2": (d,),
              "w_ada": (6 * d, c), "b_ada": (6 * d,)}
    out = {name: _param(shapes[name], cfg.seed, block, i, device)
           for i, name in enumerate(BLOCK_TENSORS) if name in shapes}
    if cfg.qk_norm:
        for name in ("q_norm", "k_norm"):
            i = BLOCK_TENSORS.index(name)
            z = _randn((cfg.head_dim,), _seed(cfg.seed, block, i), device)
            out[name] = (1.0 + QK_GAIN_STD * z).to(torch.bfloat16).float()
    return out


def final_params(cfg: DiTConfig, device="cpu") -> Dict[str, torch.Tensor]:
    """Final AdaLN projections, one per stream (video, audio): w [2, 2d, c], b [2, 2d]."""
    d, c = cfg.d, cfg.c_dim
    return {"w_fin": _param((2, 2 * d, c), cfg.seed, -1, 0, device),
            "b_fin": _param((2, 2 * d), cfg.seed, -1, 1, device)}


def head_params(cfg: DiTConfig, device="cpu") -> Dict[str, torch.Tensor]:
    """Patch embedding and final heads of a latent workload, one per stream (video, audio):
    w_patch [2, d, C], b_patch [2, d], w_head [2, C, d], b_head [2, C], bf16 N(0, 0.02)."""
    d, C = cfg.d, cfg.latent_channels
    shapes = {"w_patch": (2, d, C), "b_patch": (2, d), "w_head": (2, C, d), "b_head": (2, C)}
    return {name: _param(shapes[name], cfg.seed, -2, i, device)
            for i, name in enumerate(_HEAD_TENSORS)}


def latent_state(cfg: DiTConfig, device="cpu") -> torch.Tensor:
    """Initial latent [N, C] ~ N(0, 1) as fp32 holding bf16-representable values."""
    x = _randn((cfg.n_tokens, cfg.latent_channels), _seed(cfg.seed, -2, _NOISE_IDX), device)
    return x.to(torch.bfloat16).float()


def conditioning(cfg: DiTConfig, device="cpu") -> torch.Tensor:
    """Conditioning vector c ~ N(0, 1), bf16 [c_dim]."""
    return _randn((cfg.c_dim,), _seed(cfg.seed, -1, _COND_IDX), device).to(torch.bfloat16)


def latent_noise(cfg: DiTConfig, device="cpu", n_tokens: Optional[int] = None) -> torch.Tensor:
    """Initial state x ~ N(0, 1) as fp32 [N, d] holding bf16-representable values."""
    n = cfg.n_tokens if n_tokens is None else n_tokens
    x = _randn((n, cfg.d), _seed(cfg.seed, -1, _NOISE_IDX), device).to(torch.bfloat16)
    return x.float()


def int8_fc2_inputs(cfg: Int8Config = INT8_CONFIG, device="cpu", M: Optional[int] = None,
                    K: Optional[int] = None, n_out: Optional[int] = None,
                    ) -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of the int8 row-scaled FC2: act bf16 [M, K] = GELU(z), weight bf16 [n_out, K]
    (output channel per row, K contiguous), gate fp32 [n_out] ~ N(0,1), residual bf16
    [M, n_out] ~ N(0,1), bias fp32 [n_out] or None."""
    M = cfg.M if M is None else M
    K = cfg.K if K is None else K
    n_out = cfg.n_out if n_out is None else n_out
    s = cfg.seed
    z = _randn((M, K), _seed(s, -1, _INT8_IDX["act"]), device)
    act = torch.nn.functional.gelu(z, approximate="tanh").to(torch.bfloat16)
    del z
    w = (_randn((n_out, K), _seed(s, -1, _INT8_IDX["w"]), device) * PARAM_STD).to(torch.bfloat16)
    gate = _randn((n_out,), _seed(s, -1, _INT8_IDX["gate"]), device)
    resid = _randn((M, n_out), _seed(s, -1, _INT8_IDX["resid"]), device).to(torch.bfloat16)
    bias = None
    if cfg.with_bias:
        bias = _randn((n_out,), _seed(s, -1, _INT8_IDX["bias"]), device) * PARAM_STD
    return {"act": act, "w": w, "gate": gate, "resid": resid, "bias": bias}
