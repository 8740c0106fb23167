"""The steps on either side of the block stack: per-stream patch embedding of the latent
and per-stream final heads with the final AdaLN folded in and the Euler update in the head
GEMM's epilogue (dothoosh.com, "DiT fusions and memory management": the final BF16 heads
apply the AdaLN as they load their tiles), through h3b_denoise_step_latent, against the
oracle's latent loop."""
import os

import numpy as np
import pytest
import torch

from oracle import workloads
from tests.helpers import rel_l2

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("video_diffusion_transformer_03_b200.h3b")
from video_diffusion_transformer_03_b200 import synth  # noqa: E402
from video_diffusion_transformer_03_b200.pipeline import DiTDenoiser  # noqa: E402

DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
f64 = lambda t: t.float().numpy().astype(np.float64)


def test_tiny_latent_denoise_vs_oracle():
    cfg = synth.CONFIGS["tiny_latent"]
    m = DiTDenoiser(cfg, keep_host_params=True)
    lat0 = synth.latent_state(cfg)
    lat = lat0.to(DEV)
    m.run(lat)
    h3b.sync_status()
    blocks = [{k: f64(v) for k, v in p.items()} for p in m.host_params]
    final = {k: f64(v) for k, v in m.host_final.items()}
    heads = {k: f64(v) for k, v in m.host_heads.items()}
    want = workloads.denoise_latent(cfg, blocks, final, heads, f64(synth.conditioning(cfg)),
                                    f64(lat0))
    got = lat.cpu().numpy().astype(np.float64)
    assert rel_l2(got, want) < 3e-2
    assert rel_l2(got - f64(lat0), want - f64(lat0)) < 3e-2


def test_512_latent_denoise_vs_golden():
    ref = np.load(os.path.join(GOLDEN, "dit512_latent_oracle.npz"))
    cfg = synth.CONFIGS["dit512_latent"]
    m = DiTDenoiser(cfg)
    lat0 = synth.latent_state(cfg)
    lat = lat0.to(DEV)
    rows = ref["rows"]
    base = f64(lat0)[rows]
    m.step(lat, 0)
    h3b.sync_status()
    s1 = lat.cpu().numpy()[rows].astype(np.float64)
    for i in range(1, cfg.run_steps):
        m.step(lat, i)
    h3b.sync_status()
    fin = lat.cpu().numpy()[rows].astype(np.float64)
    for got, key in ((s1, "step1"), (fin, "final")):
        want = ref[key].astype(np.float64)
        assert rel_l2(got, want) < 3e-2, key
        assert rel_l2(got - base, want - base) < 3e-2, key


def test_latent_step_is_deterministic_and_graph_replayable():
    cfg = synth.CONFIGS["dit512_latent"]
    m = DiTDenoiser(cfg)
    lat0 = synth.latent_state(cfg).to(DEV)
    a = lat0.clone()
    m.run(a)
    h3b.sync_status()
    b = lat0.clone()
    graph = m.capture(b)
    for _ in range(2):
        b.copy_(lat0)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(a, b)
    del graph
