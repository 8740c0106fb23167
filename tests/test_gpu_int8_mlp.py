"""The int8 block path (dothoosh.com, "The powerful int8 path"): the AdaLN output
quantised per row inside the LayerNorm kernel, int8 QKV and FC1, the FC2 input quantised
per 1024-channel group and the grouped int8 FC2, against the oracle."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from oracle import workloads
from tests.helpers import max_block_rel_l2, np64, rel_l2, rnd

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("video_diffusion_transformer_03_b200.h3b")
from video_diffusion_transformer_03_b200 import synth  # noqa: E402
from video_diffusion_transformer_03_b200.pipeline import dims_of, grid_of  # noqa: E402

DEV = "cuda"


@pytest.mark.parametrize("n,d", [(5, 256), (1600, 3072), (77, 1024)])
def test_ln_modulate_q8_vs_oracle(n, d):
    x = rnd((n, d), 1.0, seed=n + d)
    shift = rnd((d,), 0.3, seed=1, dtype=torch.float32)
    scale = rnd((d,), 0.3, seed=2, dtype=torch.float32)
    q = torch.empty((n, d), dtype=torch.int8, device=DEV)
    s = torch.empty((n,), dtype=torch.float32, device=DEV)
    h3b.ln_modulate_q8(x.to(DEV), 1e-6, shift.to(DEV), scale.to(DEV), q, s)
    h3b.sync_status()
    h = O.modulate(O.layer_norm(np64(x), 1e-6), np64(shift), np64(scale))
    qo, so = O.quantize_rows(h.astype(np.float32))
    # h is fp32 on the GPU and fp64 here: a code may sit on the other side of a rounding
    # boundary, never further
    diff = np.abs(q.cpu().numpy().astype(int) - qo.astype(int))
    assert diff.max() <= 1 and (diff > 0).mean() < 1e-2
    assert rel_l2(s.cpu().numpy(), so) < 1e-5


@pytest.mark.parametrize("rows,cols", [(3, 1024), (1600, 12288), (257, 2048)])
def test_quantize_groups_bit_exact(rows, cols):
    z = rnd((rows, cols), 1.0, seed=rows, dtype=torch.float32)
    a = torch.nn.functional.gelu(z, approximate="tanh").to(torch.bfloat16)
    a[0, :1024] = 0                                 # a zero group
    q = torch.empty((rows, cols), dtype=torch.int8, device=DEV)
    s = torch.empty((rows, cols // 1024), dtype=torch.float32, device=DEV)
    h3b.quantize_groups(a.to(DEV), q, s)
    h3b.sync_status()
    qo, so = O.quantize_groups(a.float().numpy(), 1024)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


# With the scratch, a partial last wave of 256 x 128 tiles runs stream-K over the 1024-column
# groups: at 1,600 x 3,072 x 12,288, 20 of 168 tiles split over 74 pairs; at 2,048 x 3,072 x
# 8,192, 44 of 192 tiles of 8 groups.  The small shapes stay data-parallel either way.
@pytest.mark.parametrize("use_ws", [False, True])
@pytest.mark.parametrize("M,K,N", [(1600, 12288, 3072), (2048, 8192, 3072), (40, 1024, 256),
                                   (300, 2048, 640)])
def test_grouped_int8_gemm_vs_oracle(M, K, N, use_ws):
    z = rnd((M, K), 1.0, seed=M, dtype=torch.float32)
    a = torch.nn.functional.gelu(z, approximate="tanh").to(torch.bfloat16)
    w = rnd((N, K), 0.02, seed=M + 1)
    gate = rnd((N,), 1.0, seed=M + 2, dtype=torch.float32)
    bias = rnd((N,), 0.02, seed=M + 3)
    resid = rnd((M, N), 1.0, seed=M + 4)
    aq = torch.empty((M, K), dtype=torch.int8, device=DEV)
    asc = torch.empty((M, K // 1024), dtype=torch.float32, device=DEV)
    h3b.quantize_groups(a.to(DEV), aq, asc)
    wq = torch.empty((N, K), dtype=torch.int8, device=DEV)
    ws = torch.empty((N,), dtype=torch.float32, device=DEV)
    h3b.quantize_rows(w.to(DEV), wq, ws)
    out = resid.to(DEV)
    scratch = (torch.empty(h3b.gemm_workspace_size(), dtype=torch.uint8, device=DEV)
               if use_ws else None)
    h3b.gemm_i8_grouped(aq, asc, wq, ws, bias.to(DEV), gate.to(DEV), out, ws=scratch)
    h3b.sync_status()
    if use_ws:  # the split sums are added in a fixed order: a second call gives the same bits
        again = resid.to(DEV)
        h3b.gemm_i8_grouped(aq, asc, wq, ws, bias.to(DEV), gate.to(DEV), again, ws=scratch)
        h3b.sync_status()
        assert torch.equal(again, out)
    qo, so = O.quantize_groups(a.float().numpy(), 1024)
    wqo, wso = O.quantize_rows(w.float().numpy())
    y = O.int8_grouped_matmul(qo, so, wqo, wso, 1024) + np64(bias)[None, :]
    want = O.gated_residual(np64(resid), np64(gate), y)
    got = np64(out)
    assert rel_l2(got, want) < 4e-3
    assert max_block_rel_l2(got, want) < 8e-3
    # the gated branch itself, against the float product it approximates
    assert rel_l2(got - np64(resid), want - np64(resid)) < 2e-2


def _int8_block(cfg, params, c, x):
    dims, grid = dims_of(cfg), grid_of(cfg)
    n = x.shape[0]
    dev = {k: v.to(DEV) for k, v in params.items()}
    mod = torch.empty((6, cfg.d), dtype=torch.float32, device=DEV)
    h3b.adaln_modulation(dev.pop("w_ada"), dev.pop("b_ada"), c.to(DEV), mod)
    tq, wq = h3b.quantize_block_int8(dev)
    cs = torch.empty((n, cfg.head_dim // 2, 2), dtype=torch.float32, device=DEV)
    h3b.rope_table(dims, grid, False, cs)
    ws = h3b.workspace(h3b.workspace_size_int8(dims, n))
    xd = x.to(DEV)
    h3b.block_forward_int8(dims, h3b.make_block_weights(dev), wq, mod, cs, xd, ws)
    h3b.sync_status()
    host_q = {k: v.cpu().numpy() for k, v in tq.items()}
    return xd.cpu(), host_q, mod


@pytest.mark.parametrize("name", ["tiny", "dit512", "dit512_qknorm"])
def test_int8_block_vs_oracle(name):
    cfg = synth.CONFIGS[name]
    params = synth.block_params(cfg, 0)
    c = synth.conditioning(cfg)
    x = synth.latent_noise(cfg).to(torch.bfloat16)
    xg, hq, _ = _int8_block(cfg, params, c, x)
    rows = None
    if name != "tiny":
        nv, n = cfg.n_video, cfg.n_tokens
        rows = np.unique(np.concatenate([np.arange(3), np.linspace(3, nv - 1, 40).astype(int),
                                         np.arange(nv - 2, n)]))
    p64 = {k: v.float().numpy().astype(np.float64) for k, v in params.items()}
    for name_ in ("qkv", "fc1", "fc2"):
        p64[f"w_{name_}_q"], p64[f"s_{name_}"] = hq[f"w_{name_}_q"], hq[f"s_{name_}"]
        wqo, _ = O.quantize_rows(params[f"w_{name_}"].float().numpy())
        assert np.array_equal(hq[f"w_{name_}_q"], wqo)          # weights quantised bit-exactly
    mod = O.adaln_modulation(p64["w_ada"], p64["b_ada"], np64(c), cfg.d)
    pos = O.rope_positions(cfg.grid, cfg.n_audio)
    want = O.block_forward_int8(np64(x), p64, mod, pos, cfg.n_heads, cfg.rope_split,
                                cfg.rope_theta, cfg.ln_eps, rows=rows)
    got = np64(xg) if rows is None else np64(xg)[rows]
    xin = np64(x) if rows is None else np64(x)[rows]
    assert rel_l2(got, want) < 1e-2
    if rows is not None:
        assert rel_l2(got - xin, want - xin) < 2e-2
    # and the int8 block stays near the bf16 block (quantisation noise only)
    ref, _ = workloads.block(cfg, p64, np64(c), np64(x), rows=rows)
    assert rel_l2(got - xin, ref - xin) < (6e-2 if name == "tiny" else 4e-2)
