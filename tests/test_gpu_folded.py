"""The AdaLN-folded block path (dothoosh.com, "DiT fusions and memory management": the
attention gate fused with the MLP AdaLN, the MLP gate producing the next block's AdaLN).

The folded projections read the raw bf16 residual and apply the LayerNorm + modulation in
their epilogue from row statistics that the previous gated-residual epilogue wrote, so no
LayerNorm pass runs.  Checked against the oracle's plain LN -> modulate -> matmul order:
the fold kernel's identity, the row statistics, one block at the tiny, 512x512 and
768x1344 shapes, and the denoise trajectories (tests/test_gpu_denoise.py runs both
forms)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from oracle import workloads
from tests.helpers import bf16_bits, np64, rel_l2, rnd

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("video_diffusion_transformer_03_b200.h3b")
from video_diffusion_transformer_03_b200 import synth  # noqa: E402
from video_diffusion_transformer_03_b200.pipeline import dims_of, grid_of  # noqa: E402

DEV = "cuda"
TOL_BLOCK = 1e-2


@pytest.mark.parametrize("n_out,d", [(384, 256), (9216, 3072), (1024, 512)])
def test_fold_adaln_identity(n_out, d):
    # y = (LN(x)(1 + scale) + shift) W^T + b, computed by the oracle's plain order, equals
    # rstd (x W'^T - mean c) + dv built from the kernel's W', c and dv
    w = rnd((n_out, d), 0.02, seed=1)
    b = rnd((n_out,), 0.02, seed=2)
    shift = rnd((d,), 0.3, seed=3, dtype=torch.float32)
    scale = rnd((d,), 0.3, seed=4, dtype=torch.float32)
    wo = torch.empty((n_out, d), dtype=torch.bfloat16, device=DEV)
    c = torch.empty((n_out,), dtype=torch.float32, device=DEV)
    dv = torch.empty((n_out,), dtype=torch.float32, device=DEV)
    h3b.fold_adaln(w.to(DEV), b.to(DEV), shift.to(DEV), scale.to(DEV), wo, c, dv)
    h3b.sync_status()
    wf = np64(wo)
    # W' is W (1 + scale) rounded once to bf16; c sums the stored W'; dv = W shift + b
    want_w = O.round_to_bf16(np64(w) * (1 + np64(scale))[None, :]).astype(np.float64)
    assert np.max(np.abs(wf - want_w)) <= np.max(np.abs(want_w)) * 2 ** -8
    assert rel_l2(np64(c), wf.sum(axis=1)) < 1e-5
    assert rel_l2(np64(dv), np64(w) @ np64(shift) + np64(b)) < 1e-5
    x = np64(rnd((37, d), 1.0, seed=5)) + 0.5
    mean = x.mean(axis=1, keepdims=True)
    rstd = 1 / np.sqrt(x.var(axis=1, keepdims=True) + 1e-6)
    got = rstd * (x @ wf.T - mean * np64(c)[None, :]) + np64(dv)[None, :]
    want = O.modulate(O.layer_norm(x, 1e-6), np64(shift), np64(scale)) @ np64(w).T + np64(b)
    assert rel_l2(got, want) < 4e-3


@pytest.mark.parametrize("n,d,offset", [(5, 256, 0.0), (1000, 3072, 0.0), (77, 3072, 100.0)])
def test_row_stats_groups(n, d, offset):
    x = (rnd((n, d), 1.0, seed=6).float() + offset).to(torch.bfloat16)
    st = torch.empty((n, d // 256, 2), dtype=torch.float32, device=DEV)
    h3b.row_stats(x.to(DEV), st)
    h3b.sync_status()
    g = np64(x).reshape(n, d // 256, 256)
    mean = g.mean(axis=2)
    m2 = ((g - mean[..., None]) ** 2).sum(axis=2)
    got = st.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got[..., 0] - mean)) < 1e-5 * (1 + abs(offset))
    assert rel_l2(got[..., 1], m2) < 1e-5


def _folded_block(cfg, params, c, x, stats_from_gpu=True):
    dims, grid = dims_of(cfg), grid_of(cfg)
    n = x.shape[0]
    dev = {k: v.to(DEV) for k, v in params.items()}
    mod = torch.empty((6, cfg.d), dtype=torch.float32, device=DEV)
    h3b.adaln_modulation(dev.pop("w_ada"), dev.pop("b_ada"), c.to(DEV), mod)
    dev.update(h3b.fold_block(dev, mod))
    cs = torch.empty((n, cfg.head_dim // 2, 2), dtype=torch.float32, device=DEV)
    h3b.rope_table(dims, grid, False, cs)
    ws = h3b.workspace(h3b.workspace_size(dims, n))
    xd = x.to(DEV)
    st = torch.empty((n, cfg.d // 256, 2), dtype=torch.float32, device=DEV)
    h3b.row_stats(xd, st)
    h3b.block_forward_folded(dims, h3b.make_block_weights(dev), mod, cs, xd, st, ws)
    st_ref = torch.empty_like(st)
    h3b.row_stats(xd, st_ref)
    h3b.sync_status()
    return xd.cpu(), st.cpu(), st_ref.cpu(), mod


def _rows(cfg, k):
    nv, n = cfg.n_video, cfg.n_tokens
    return np.unique(np.concatenate([np.arange(3), np.linspace(3, nv - 1, k).astype(int),
                                     np.arange(nv - 2, min(n, nv + 3)), [n - 1]]))


def _update_tol(cfg, p, c, x):
    from tests.test_gpu_block import update_tolerance
    return update_tolerance(cfg, p, c, x)


@pytest.mark.parametrize("name", ["tiny", "dit512", "dit768x1344"])
def test_folded_block_vs_oracle(name):
    cfg = synth.CONFIGS[name]
    params = synth.block_params(cfg, 0)
    c = synth.conditioning(cfg)
    x = synth.latent_noise(cfg).to(torch.bfloat16)
    xg, st, st_ref, _ = _folded_block(cfg, params, c, x)
    rows = None if name == "tiny" else _rows(cfg, 24 if name == "dit768x1344" else 40)
    p64 = {k: v.float().numpy().astype(np.float64) for k, v in params.items()}
    xo, _ = workloads.block(cfg, p64, np64(c), np64(x), rows=rows)
    got = np64(xg) if rows is None else np64(xg)[rows]
    xin = np64(x) if rows is None else np64(x)[rows]
    e = rel_l2(got, xo)
    assert e <= TOL_BLOCK, f"x_out rel-L2 {e:.3e}"
    if name == "tiny":
        tol = _update_tol(cfg, params, c, x)
        eu = rel_l2(got - xin, xo - xin)
        assert eu <= tol, f"update rel-L2 {eu:.3e} > {tol:.3e}"
    # the statistics the FC2 epilogue wrote describe the output before its bf16 rounding:
    # against those of the stored output they differ by the rounding only (each value moves
    # by at most 2^-9 of itself, averaging out over a 256-column group)
    s, r = st.numpy().astype(np.float64), st_ref.numpy().astype(np.float64)
    scale = np.sqrt(r[..., 1] / 256.0) + np.abs(r[..., 0])
    assert np.max(np.abs(s[..., 0] - r[..., 0]) / scale) < 2e-3
    assert rel_l2(s[..., 1], r[..., 1]) < 2e-3


def test_folded_block_close_to_unfolded_block():
    # same block through both GPU paths: they differ by the folded weights' rounding only
    cfg = synth.CONFIGS["dit512"]
    params = synth.block_params(cfg, 0)
    c = synth.conditioning(cfg)
    x = synth.latent_noise(cfg).to(torch.bfloat16)
    xf, _, _, mod = _folded_block(cfg, params, c, x)
    dims, grid = dims_of(cfg), grid_of(cfg)
    n = cfg.n_tokens
    dev = {k: v.to(DEV) for k, v in params.items() if k not in ("w_ada", "b_ada")}
    cs = torch.empty((n, cfg.head_dim // 2, 2), dtype=torch.float32, device=DEV)
    h3b.rope_table(dims, grid, False, cs)
    ws = h3b.workspace(h3b.workspace_size(dims, n))
    xu = x.to(DEV)
    h = torch.empty_like(xu)
    h3b.block_forward(dims, h3b.make_block_weights(dev), mod, None, cs, xu, h, ws, True)
    h3b.sync_status()
    d_f, d_u = np64(xf) - np64(x), np64(xu) - np64(x)
    assert rel_l2(d_f, d_u) < 1e-2


def test_folded_block_zero_gates_bit_exact():
    cfg = synth.CONFIGS["dit512"]
    params = dict(synth.block_params(cfg, 0))
    # zero gates through the AdaLN weights: rows 2d..3d and 5d..6d of w_ada / b_ada
    d = cfg.d
    w_ada, b_ada = params["w_ada"].clone(), params["b_ada"].clone()
    for g in (2, 5):
        w_ada[g * d:(g + 1) * d] = 0
        b_ada[g * d:(g + 1) * d] = 0
    params["w_ada"], params["b_ada"] = w_ada, b_ada
    c = synth.conditioning(cfg)
    x = synth.latent_noise(cfg).to(torch.bfloat16)
    xg, st, st_ref, _ = _folded_block(cfg, params, c, x)
    assert np.array_equal(bf16_bits(xg), bf16_bits(x))


# (M, d, N): the QKV shape of the 512x512 workload, a ragged tiny one, and an FC1 shape
LN_GEMM_SHAPES = [(1600, 3072, 9216), (40, 256, 768), (1000, 1024, 4096)]


def _ln_gemm_inputs(M, d, N, seed, offset=0.0):
    x = (rnd((M, d), 1.0, seed=seed).float() + offset).to(torch.bfloat16)
    w = rnd((N, d), 0.02, seed=seed + 1)
    b = rnd((N,), 0.02, seed=seed + 2)
    shift = rnd((d,), 0.3, seed=seed + 3, dtype=torch.float32)
    scale = rnd((d,), 0.3, seed=seed + 4, dtype=torch.float32)
    return x, w, b, shift, scale


def _fold_on_gpu(w, b, shift, scale):
    N, d = w.shape
    wo = torch.empty((N, d), dtype=torch.bfloat16, device=DEV)
    c = torch.empty((N,), dtype=torch.float32, device=DEV)
    dv = torch.empty((N,), dtype=torch.float32, device=DEV)
    h3b.fold_adaln(w.to(DEV), b.to(DEV), shift.to(DEV), scale.to(DEV), wo, c, dv)
    return wo, c, dv


@pytest.mark.parametrize("M,d,N", LN_GEMM_SHAPES)
@pytest.mark.parametrize("epi", [h3b.EPI_LN_GELU, h3b.EPI_LN_ROPE])
def test_ln_folded_gemm_vs_oracle(M, d, N, epi):
    x, w, b, shift, scale = _ln_gemm_inputs(M, d, N, seed=M + N)
    wo, c, dv = _fold_on_gpu(w, b, shift, scale)
    xd = x.to(DEV)
    st = torch.empty((M, d // 256, 2), dtype=torch.float32, device=DEV)
    h3b.row_stats(xd, st)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    h_o = O.modulate(O.layer_norm(np64(x), 1e-6), np64(shift), np64(scale))
    pre = h_o @ np64(w).T + np64(b)
    kw = {}
    if epi == h3b.EPI_LN_GELU:
        want = O.gelu_tanh(pre)
    else:
        hd = 128 if d % 128 == 0 and d >= 256 else 64
        heads = d // hd
        split = (32, 48, 48) if hd == 128 else (16, 24, 24)
        # a token grid of M tokens (one row of video tokens, the rest audio)
        grid, n_audio = (1, 1, min(M, 8)), M - min(M, 8)
        dims = h3b.make_dims(d, heads, hd, 4 * d, 256, split)
        cs = torch.empty((M, hd // 2, 2), dtype=torch.float32, device=DEV)
        h3b.rope_table(dims, h3b.make_grid(*grid, n_audio), False, cs)
        rope_cols = min(2 * d, N)
        kw = dict(rope_cs=cs, rope_cols=rope_cols, head_dim=hd)
        pos = O.rope_positions(grid, n_audio)
        want = pre.copy()
        for part in range(rope_cols // d):
            blk = pre[:, part * d:(part + 1) * d].reshape(M, heads, hd)
            want[:, part * d:(part + 1) * d] = O.rope_rotate(blk, pos, split, 1e4).reshape(M, d)
    h3b.gemm_bf16_ln(xd, wo, epi, out, fold_c=c, fold_dv=dv, stats_in=st,
                     ws=torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=DEV),
                     **kw)
    h3b.sync_status()
    got = np64(out)
    from tests.helpers import max_block_rel_l2
    assert rel_l2(got, want) < 6e-3
    assert max_block_rel_l2(got, want) < 1.2e-2


@pytest.mark.parametrize("M,N,K", [(1600, 3072, 3072), (40, 256, 1024), (1600, 3072, 12288)])
def test_gate_resid_gemm_writes_row_statistics(M, N, K):
    A = rnd((M, K), 1.0, seed=91)
    B = rnd((N, K), K ** -0.5, seed=92)
    bias = rnd((N,), 0.1, seed=93)
    resid = rnd((M, N), 1.0, seed=94)
    g = rnd((N,), 0.5, seed=95, dtype=torch.float32)
    out = resid.to(DEV)
    st = torch.empty((M, N // 256, 2), dtype=torch.float32, device=DEV)
    plain = resid.to(DEV)
    ws = torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=DEV)
    h3b.gemm_bf16_ln(A.to(DEV), B.to(DEV), h3b.EPI_GATE_RESID, out, bias=bias.to(DEV),
                     gate=g.to(DEV), stats_out=st, ws=ws)
    h3b.gemm_bf16(A.to(DEV), B.to(DEV), h3b.EPI_GATE_RESID, bias.to(DEV), plain, gate=g.to(DEV),
                  ws=ws)
    h3b.sync_status()
    # the output is that of the plain gated-residual epilogue, bit for bit
    assert torch.equal(out, plain)
    # the statistics are those of the exact (unrounded) output, per 256-column group
    want = O.gated_residual(np64(resid), np64(g), np64(A) @ np64(B).T + np64(bias))
    gr = want.reshape(M, N // 256, 256)
    mean = gr.mean(axis=2)
    m2 = ((gr - mean[..., None]) ** 2).sum(axis=2)
    s = st.cpu().numpy().astype(np.float64)
    scale = np.sqrt(m2 / 256.0) + np.abs(mean)
    assert np.max(np.abs(s[..., 0] - mean) / scale) < 2e-3
    assert rel_l2(s[..., 1], m2) < 2e-3


def test_ln_folded_gemm_large_row_offset():
    # rows far from zero mean: the statistics are taken about each group's first value
    M, d, N = 300, 1024, 1024
    x, w, b, shift, scale = _ln_gemm_inputs(M, d, N, seed=7, offset=50.0)
    wo, c, dv = _fold_on_gpu(w, b, shift, scale)
    xd = x.to(DEV)
    st = torch.empty((M, d // 256, 2), dtype=torch.float32, device=DEV)
    h3b.row_stats(xd, st)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    h3b.gemm_bf16_ln(xd, wo, h3b.EPI_LN_GELU, out, fold_c=c, fold_dv=dv, stats_in=st)
    h3b.sync_status()
    want = O.gelu_tanh(O.modulate(O.layer_norm(np64(x), 1e-6), np64(shift), np64(scale))
                       @ np64(w).T + np64(b))
    # the bf16 residual itself carries 50 * 2^-9 of rounding per element at this offset,
    # which LN amplifies by 1 / std: the bound scales with it
    assert rel_l2(np64(out), want) < 2e-2
