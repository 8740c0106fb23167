"""h3b_block_forward_noalloc: the block entry point for callers that cannot allocate device
memory (its workspace is a static array inside the library).  Checked through the C ABI
against h3b_block_forward with a caller workspace, on two calls in a row, so that a second
call over the first call's leftover workspace contents is covered too.  Both entry points
run the same kernels in the same order with the same schedules (the stream-K partial
tiles are merged in a fixed order), so the results must agree bit for bit: a wrong
offset into the static array, or a leftover value read from it, cannot hide under a
tolerance.  Kept in a file of its own that pytest collects after every other test
file."""
import numpy as np
import pytest
import torch

from tests.helpers import bf16_bits

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("video_diffusion_transformer_03_b200.h3b")
from video_diffusion_transformer_03_b200 import synth  # noqa: E402
from video_diffusion_transformer_03_b200.pipeline import dims_of, grid_of  # noqa: E402

DEV = "cuda"


def _block_inputs(cfg):
    dims, grid = dims_of(cfg), grid_of(cfg)
    n = cfg.n_tokens
    p = {k: v.to(DEV) for k, v in synth.block_params(cfg, 0).items()}
    pn = {k: v.to(DEV) for k, v in synth.block_params(cfg, 1).items()}
    c = synth.conditioning(cfg).to(DEV)
    mod = torch.empty((6, cfg.d), dtype=torch.float32, device=DEV)
    mod_next = torch.empty((6, cfg.d), dtype=torch.float32, device=DEV)
    h3b.adaln_modulation(p["w_ada"], p["b_ada"], c, mod)
    h3b.adaln_modulation(pn["w_ada"], pn["b_ada"], c, mod_next)
    cs = torch.empty((n, cfg.head_dim // 2, 2), dtype=torch.float32, device=DEV)
    h3b.rope_table(dims, grid, False, cs)
    x0 = synth.latent_noise(cfg).to(torch.bfloat16).to(DEV)
    return dims, h3b.make_block_weights(p), mod, mod_next, cs, x0, p


@pytest.mark.parametrize("name", ["tiny", "dit512"])
def test_noalloc_block_matches_workspace_entry_point(name):
    cfg = synth.CONFIGS[name]
    dims, w, mod, mod_next, cs, x0, _keep = _block_inputs(cfg)
    assert h3b.workspace_size(dims, cfg.n_tokens) <= h3b.NOALLOC_WORKSPACE_BYTES

    x_ref, h_ref = x0.clone(), torch.empty_like(x0)
    ws = h3b.workspace(h3b.workspace_size(dims, cfg.n_tokens))
    h3b.block_forward(dims, w, mod, mod_next, cs, x_ref, h_ref, ws, True)
    h3b.sync_status()

    for call in range(2):
        x, h = x0.clone(), torch.full_like(x0, float("nan"))
        h3b.block_forward_noalloc(dims, w, mod, mod_next, cs, x, h, True)
        h3b.sync_status()
        assert np.array_equal(bf16_bits(x), bf16_bits(x_ref)), f"call {call}: x differs"
        assert np.array_equal(bf16_bits(h), bf16_bits(h_ref)), f"call {call}: h differs"


def test_noalloc_rejects_blocks_beyond_the_static_workspace():
    cfg = synth.CONFIGS["dit512"]
    dims, w, mod, mod_next, cs, x0, _keep = _block_inputs(cfg)
    per_token = h3b.workspace_size(dims, 2) - h3b.workspace_size(dims, 1)
    too_many = h3b.NOALLOC_WORKSPACE_BYTES // per_token + 1
    assert h3b.workspace_size(dims, too_many) > h3b.NOALLOC_WORKSPACE_BYTES
    big = torch.empty((too_many, cfg.d), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(h3b.H3BError) as err:
        h3b.block_forward_noalloc(dims, w, mod, None, cs, big, big.clone(), True)
    assert err.value.code == h3b.H3B_EWORKSPACE
    assert "static" in str(err.value)
