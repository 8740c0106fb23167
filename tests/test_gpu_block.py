"""Block-level parity: h3b_block_forward against the oracle's block, per block, with the
oracle fed the GPU's bf16 block input (tolerance: rel-L2 <= 1e-2 per output tensor)."""
import numpy as np
import pytest
import torch

from oracle import workloads
from tests.helpers import np64, rel_l2

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("video_diffusion_transformer_03_b200.h3b")
from video_diffusion_transformer_03_b200 import synth  # noqa: E402
from video_diffusion_transformer_03_b200.pipeline import dims_of, grid_of  # noqa: E402

DEV = "cuda"
TOL_BLOCK = 1e-2


def gpu_block(cfg, params, next_params, c, x, compute_h=True, h_in=None):
    dims, grid = dims_of(cfg), grid_of(cfg)
    n = x.shape[0]
    dev = {k: v.to(DEV) for k, v in params.items()}
    cd = c.to(DEV)
    mod = torch.empty((6, cfg.d), dtype=torch.float32, device=DEV)
    h3b.adaln_modulation(dev["w_ada"], dev["b_ada"], cd, mod)
    mod_next = None
    if next_params is not None:
        mod_next = torch.empty((6, cfg.d), dtype=torch.float32, device=DEV)
        h3b.adaln_modulation(next_params["w_ada"].to(DEV), next_params["b_ada"].to(DEV), cd,
                             mod_next)
    cs = torch.empty((n, cfg.head_dim // 2, 2), dtype=torch.float32, device=DEV)
    h3b.rope_table(dims, grid, False, cs)
    ws = h3b.workspace(h3b.workspace_size(dims, n))
    xd = x.to(DEV)
    hd = torch.empty_like(xd) if h_in is None else h_in.to(DEV)
    h3b.block_forward(dims, h3b.make_block_weights(dev), mod, mod_next, cs, xd, hd, ws, compute_h)
    h3b.sync_status()
    return xd.cpu(), (hd.cpu() if next_params is not None else None)


def f64(t):
    return t.float().numpy().astype(np.float64)


def oracle_block(cfg, params, next_params, c, x, rows=None):
    p = {k: f64(v) for k, v in params.items()}
    nxt = None if next_params is None else {k: f64(v) for k, v in next_params.items()}
    return workloads.block(cfg, p, f64(c), f64(x), next_params=nxt, rows=rows)


def check(name, got, want, x_in=None, tol=TOL_BLOCK):
    e = rel_l2(got, want)
    msg = f"{name}: rel-L2 {e:.3e}"
    if x_in is not None:
        msg += f", update rel-L2 {rel_l2(got - x_in, want - x_in):.3e}"
    assert e <= tol, msg
    return e


def test_block_tiny_full():
    cfg = synth.CONFIGS["tiny"]
    params = synth.block_params(cfg, 0)
    nxt = synth.block_params(cfg, 1)
    c = synth.conditioning(cfg)
    x = synth.latent_noise(cfg).to(torch.bfloat16)
    xg, hg = gpu_block(cfg, params, nxt, c, x)
    xo, ho = oracle_block(cfg, params, nxt, c, x)
    check("x_out", np64(xg), xo, np64(x))
    check("h_next", np64(hg), ho)


def _rows(cfg, k=40):
    nv, n = cfg.n_video, cfg.n_tokens
    return np.unique(np.concatenate([np.arange(3), np.linspace(3, nv - 1, k).astype(int),
                                     np.arange(nv - 2, min(n, nv + 3)), [n - 1]]))


def test_block_512_chain_two_blocks():
    cfg = synth.CONFIGS["dit512"]
    p0, p1, p2 = (synth.block_params(cfg, b) for b in range(3))
    c = synth.conditioning(cfg)
    x0 = synth.latent_noise(cfg).to(torch.bfloat16)
    rows = _rows(cfg)
    x1, h1 = gpu_block(cfg, p0, p1, c, x0)
    xo, ho = oracle_block(cfg, p0, p1, c, x0, rows=rows)
    check("block0 x_out", np64(x1)[rows], xo, np64(x0)[rows])
    check("block0 h_next", np64(h1)[rows], ho)
    # block 1 consumes the h that block 0's epilogue chain produced
    x2, h2 = gpu_block(cfg, p1, p2, c, x1, compute_h=False, h_in=h1)
    xo2, ho2 = oracle_block(cfg, p1, p2, c, x1, rows=rows)
    check("block1 x_out", np64(x2)[rows], xo2, np64(x1)[rows])
    check("block1 h_next", np64(h2)[rows], ho2)


def test_block_768x1344_first_block():
    cfg = synth.CONFIGS["dit768x1344"]
    p0, p1 = synth.block_params(cfg, 0), synth.block_params(cfg, 1)
    c = synth.conditioning(cfg)
    x0 = synth.latent_noise(cfg).to(torch.bfloat16)
    rows = _rows(cfg, k=24)
    x1, h1 = gpu_block(cfg, p0, p1, c, x0)
    xo, ho = oracle_block(cfg, p0, p1, c, x0, rows=rows)
    check("x_out", np64(x1)[rows], xo, np64(x0)[rows])
    check("h_next", np64(h1)[rows], ho)
