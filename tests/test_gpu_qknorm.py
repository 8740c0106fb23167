"""Q/K RMSNorm fused with RoPE in the QKV projection's epilogue (dothoosh.com, "The
powerful int8 path": RMS normalisation and RoPE for Q/K inside the QKV tile), against the
oracle's rms_norm then rope_rotate: the GEMM alone (plain and LN-folded forms), one block
(both block forms) and whole denoises."""
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from oracle import workloads
from tests.helpers import max_block_rel_l2, np64, rel_l2, rnd

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("video_diffusion_transformer_03_b200.h3b")
from video_diffusion_transformer_03_b200 import synth  # noqa: E402
from video_diffusion_transformer_03_b200.pipeline import DiTDenoiser, dims_of, grid_of  # noqa: E402

DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _qk_want(pre, grid, n_audio, heads, hd, split, gq, gk):
    M, d = pre.shape[0], heads * hd
    pos = O.rope_positions(grid, n_audio)
    want = pre.copy()
    for part, g in ((0, gq), (1, gk)):
        blk = pre[:, part * d:(part + 1) * d].reshape(M, heads, hd)
        blk = O.rms_norm(blk, g, 1e-6)
        want[:, part * d:(part + 1) * d] = O.rope_rotate(blk, pos, split, 1e4).reshape(M, d)
    return want


@pytest.mark.parametrize("M,heads,hd", [(1600, 24, 128), (40, 4, 64), (1000, 8, 128)])
@pytest.mark.parametrize("folded", [False, True], ids=["bias", "ln-folded"])
def test_qkv_gemm_with_qk_rmsnorm(M, heads, hd, folded):
    d = heads * hd
    N = 3 * d
    split = (32, 48, 48) if hd == 128 else (16, 24, 24)
    grid, n_audio = (1, 1, min(M, 8)), M - min(M, 8)
    dims = h3b.make_dims(d, heads, hd, 4 * d, 256, split)
    cs = torch.empty((M, hd // 2, 2), dtype=torch.float32, device=DEV)
    h3b.rope_table(dims, h3b.make_grid(*grid, n_audio), False, cs)
    x = rnd((M, d), 1.0, seed=M + 1)
    w = rnd((N, d), 0.02, seed=M + 2)
    b = rnd((N,), 0.02, seed=M + 3)
    gq = (1 + 0.1 * rnd((hd,), 1.0, seed=M + 4, dtype=torch.float32))
    gk = (1 + 0.1 * rnd((hd,), 1.0, seed=M + 5, dtype=torch.float32))
    out = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=DEV)
    kw = dict(rope_cs=cs, rope_cols=2 * d, head_dim=hd, q_gain=gq.to(DEV), k_gain=gk.to(DEV),
              ws=ws)
    if folded:
        shift = rnd((d,), 0.3, seed=M + 6, dtype=torch.float32)
        scale = rnd((d,), 0.3, seed=M + 7, dtype=torch.float32)
        wo = torch.empty_like(w, device=DEV)
        c = torch.empty((N,), dtype=torch.float32, device=DEV)
        dv = torch.empty((N,), dtype=torch.float32, device=DEV)
        h3b.fold_adaln(w.to(DEV), b.to(DEV), shift.to(DEV), scale.to(DEV), wo, c, dv)
        st = torch.empty((M, d // 256, 2), dtype=torch.float32, device=DEV)
        xd = x.to(DEV)
        h3b.row_stats(xd, st)
        h3b.gemm_bf16_ln(xd, wo, h3b.EPI_LN_ROPE, out, fold_c=c, fold_dv=dv, stats_in=st, **kw)
        pre = (O.modulate(O.layer_norm(np64(x), 1e-6), np64(shift), np64(scale)) @ np64(w).T
               + np64(b))
    else:
        h3b.gemm_bf16_ln(x.to(DEV), w.to(DEV), h3b.EPI_BIAS_ROPE, out, bias=b.to(DEV), **kw)
        pre = np64(x) @ np64(w).T + np64(b)
    h3b.sync_status()
    want = _qk_want(pre, grid, n_audio, heads, hd, split, np64(gq), np64(gk))
    got = np64(out)
    assert rel_l2(got, want) < 6e-3
    assert max_block_rel_l2(got, want) < 1.2e-2
    # every q and k head of every row keeps the oracle's RMS (a wrong head boundary or a
    # missed head would move it by far more than bf16 rounding)
    rms = lambda a: np.sqrt((a[:, :2 * d].reshape(M, 2, heads, hd) ** 2).mean(-1))
    assert np.max(np.abs(rms(got) / rms(want) - 1)) < 1e-2


@pytest.mark.parametrize("name", ["tiny_qknorm", "dit512_qknorm"])
@pytest.mark.parametrize("folded", [False, True], ids=["layernorm-pass", "folded"])
def test_qknorm_block_vs_oracle(name, folded):
    cfg = synth.CONFIGS[name]
    dims, grid = dims_of(cfg), grid_of(cfg)
    n = cfg.n_tokens
    params = synth.block_params(cfg, 0)
    c = synth.conditioning(cfg)
    x = synth.latent_noise(cfg).to(torch.bfloat16)
    dev = {k: v.to(DEV) for k, v in params.items()}
    mod = torch.empty((6, cfg.d), dtype=torch.float32, device=DEV)
    h3b.adaln_modulation(dev.pop("w_ada"), dev.pop("b_ada"), c.to(DEV), mod)
    cs = torch.empty((n, cfg.head_dim // 2, 2), dtype=torch.float32, device=DEV)
    h3b.rope_table(dims, grid, False, cs)
    ws = h3b.workspace(h3b.workspace_size(dims, n))
    xd = x.to(DEV)
    if folded:
        dev.update(h3b.fold_block(dev, mod))
        st = torch.empty((n, cfg.d // 256, 2), dtype=torch.float32, device=DEV)
        h3b.row_stats(xd, st)
        h3b.block_forward_folded(dims, h3b.make_block_weights(dev), mod, cs, xd, st, ws)
    else:
        h = torch.empty_like(xd)
        h3b.block_forward(dims, h3b.make_block_weights(dev), mod, None, cs, xd, h, ws, True)
    h3b.sync_status()
    rows = None
    if name.startswith("dit512"):
        nv = cfg.n_video
        rows = np.unique(np.concatenate([np.arange(3), np.linspace(3, nv - 1, 40).astype(int),
                                         np.arange(nv - 2, n)]))
    p64 = {k: v.float().numpy().astype(np.float64) for k, v in params.items()}
    xo, _ = workloads.block(cfg, p64, np64(c), np64(x), rows=rows)
    got = np64(xd) if rows is None else np64(xd)[rows]
    xin = np64(x) if rows is None else np64(x)[rows]
    assert rel_l2(got, xo) <= 1e-2
    if rows is not None:       # the update is 2/3 of x here: hold it to the block bound too
        assert rel_l2(got - xin, xo - xin) <= 1.5e-2


@pytest.mark.parametrize("fold", [True, False], ids=["folded", "layernorm-pass"])
def test_qknorm_denoise_vs_oracle_tiny(fold):
    cfg = synth.CONFIGS["tiny_qknorm"]
    m = DiTDenoiser(cfg, keep_host_params=True, fold=fold)
    x0 = synth.latent_noise(cfg)
    x = x0.to(DEV)
    m.run(x)
    h3b.sync_status()
    blocks = [{k: v.float().numpy().astype(np.float64) for k, v in p.items()}
              for p in m.host_params]
    final = {k: v.float().numpy().astype(np.float64) for k, v in m.host_final.items()}
    want = workloads.denoise(cfg, blocks, final, np64(synth.conditioning(cfg)), np64(x0))
    got = x.cpu().numpy().astype(np.float64)
    assert rel_l2(got - np64(x0), want - np64(x0)) < 3e-2


def test_qknorm_denoise_vs_golden_512():
    ref = np.load(os.path.join(GOLDEN, "dit512_qknorm_oracle.npz"))
    cfg = synth.CONFIGS["dit512_qknorm"]
    m = DiTDenoiser(cfg)
    x0 = synth.latent_noise(cfg)
    x = x0.to(DEV)
    m.run(x)
    h3b.sync_status()
    rows = ref["rows"]
    got = x.cpu().numpy()[rows].astype(np.float64)
    base = np64(x0)[rows]
    want = ref["final"].astype(np.float64)
    assert rel_l2(got, want) < 3e-2 and rel_l2(got - base, want - base) < 3e-2
