"""Denoise-level parity: free-running Euler steps through h3b_denoise_step against the
oracle (tolerance: rel-L2 <= 3e-2 on x_state after the steps; the update x - x0 is held
to the same bound).  The 512x512-shaped references come from tests/golden (written by
tests/golden/make_golden.py from the oracle)."""
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from oracle import workloads
from tests.helpers import rel_l2

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("video_diffusion_transformer_03_b200.h3b")
from video_diffusion_transformer_03_b200 import synth  # noqa: E402
from video_diffusion_transformer_03_b200.pipeline import DiTDenoiser  # noqa: E402

DEV = "cuda"
TOL_STEPS = 3e-2
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def f64(t):
    return t.float().numpy().astype(np.float64)


@pytest.mark.parametrize("fold", [True, False], ids=["folded", "layernorm-pass"])
def test_tiny_denoise_vs_oracle(fold):
    cfg = synth.CONFIGS["tiny"]
    m = DiTDenoiser(cfg, keep_host_params=True, fold=fold)
    x0 = synth.latent_noise(cfg)
    x = x0.to(DEV)
    m.run(x)
    h3b.sync_status()
    blocks = [{k: f64(v) for k, v in p.items()} for p in m.host_params]
    final = {k: f64(v) for k, v in m.host_final.items()}
    want = workloads.denoise(cfg, blocks, final, f64(synth.conditioning(cfg)), f64(x0))
    got = x.cpu().numpy().astype(np.float64)
    assert rel_l2(got, want) < TOL_STEPS
    assert rel_l2(got - f64(x0), want - f64(x0)) < TOL_STEPS


@pytest.mark.parametrize("fold", [True, False], ids=["folded", "layernorm-pass"])
@pytest.mark.parametrize("name", ["dit512", "dit512_tokred", "dit256_halved"])
def test_denoise_vs_golden(name, fold):
    ref = np.load(os.path.join(GOLDEN, f"{name}_oracle.npz"))
    cfg = synth.CONFIGS[name]
    m = DiTDenoiser(cfg, fold=fold)
    active = np.ones(cfg.n_blocks, bool) if m.active is None else np.array(m.active)
    assert np.array_equal(active, ref["active"]), "layer-thinning mask differs from the oracle's"
    rows = ref["rows"]
    x0 = synth.latent_noise(cfg)
    x = x0.to(DEV)
    m.step(x, 0)
    h3b.sync_status()
    s1 = x.cpu().numpy()[rows].astype(np.float64)
    base = f64(x0)[rows]
    e1 = rel_l2(s1, ref["step1"])
    u1 = rel_l2(s1 - base, ref["step1"].astype(np.float64) - base)
    for i in range(1, cfg.run_steps):
        m.step(x, i)
    h3b.sync_status()
    fin = x.cpu().numpy()[rows].astype(np.float64)
    e4 = rel_l2(fin, ref["final"])
    u4 = rel_l2(fin - base, ref["final"].astype(np.float64) - base)
    msg = f"step1 {e1:.2e} (update {u1:.2e}); after {cfg.run_steps} steps {e4:.2e} (update {u4:.2e})"
    assert e1 < TOL_STEPS and u1 < TOL_STEPS, msg
    assert e4 < TOL_STEPS and u4 < TOL_STEPS, msg


@pytest.mark.parametrize("name", ["tiny", "dit512"])
def test_host_entry_matches_device_steps(name):
    cfg = synth.CONFIGS[name]
    m = DiTDenoiser(cfg)
    x0 = synth.latent_noise(cfg)
    xd = x0.to(DEV)
    m.run(xd)
    h3b.sync_status()
    host_in = x0.pin_memory()
    host_out = torch.empty_like(host_in).pin_memory()
    scratch = torch.empty_like(xd)
    m.run_host(host_in, host_out, scratch)
    assert torch.equal(host_out, xd.cpu())          # same kernels, same order: bit-equal


@pytest.mark.parametrize("name,requests", [("tiny", 5), ("dit512", 3), ("dit512_tokred", 2)])
def test_pipelined_host_entry_matches_device_runs(name, requests):
    cfg = synth.CONFIGS[name]
    m = DiTDenoiser(cfg)
    g = torch.Generator().manual_seed(5)
    x0 = torch.randn((requests, cfg.n_tokens, cfg.d), generator=g).to(torch.bfloat16).float()
    want = []
    for r in range(requests):
        xd = x0[r].to(DEV)
        m.run(xd)
        want.append(xd.cpu())
    h3b.sync_status()
    host_in = x0.pin_memory()
    host_out = torch.full_like(host_in, float("nan")).pin_memory()
    state2 = torch.empty((2, cfg.n_tokens, cfg.d), dtype=torch.float32, device=DEV)
    m.run_host_pipelined(host_in, host_out, state2)
    for r in range(requests):        # same kernels, same order per request: bit-equal
        assert torch.equal(host_out[r], want[r]), f"request {r}"


def test_host_entries_without_graphs_match_device_runs():
    # H3B_DEBUG=1 makes the host entry points launch the steps directly (no cached graph)
    # and check every launch; run in a child process, since the switch is read once
    import subprocess
    import sys
    code = (
        "import torch\n"
        "from video_diffusion_transformer_03_b200 import synth, h3b\n"
        "from video_diffusion_transformer_03_b200.pipeline import DiTDenoiser\n"
        "cfg = synth.CONFIGS['tiny']\n"
        "m = DiTDenoiser(cfg)\n"
        "g = torch.Generator().manual_seed(9)\n"
        "x0 = torch.randn((3, cfg.n_tokens, cfg.d), generator=g).to(torch.bfloat16).float()\n"
        "want = []\n"
        "for r in range(3):\n"
        "    xd = x0[r].to('cuda'); m.run(xd); want.append(xd.cpu())\n"
        "h3b.sync_status()\n"
        "hi, ho = x0.pin_memory(), torch.empty_like(x0).pin_memory()\n"
        "m.run_host_pipelined(hi, ho, torch.empty((2, cfg.n_tokens, cfg.d), device='cuda'))\n"
        "one = torch.empty_like(x0[0]).pin_memory()\n"
        "m.run_host(x0[1].pin_memory(), one, torch.empty_like(x0[0], device='cuda'))\n"
        "assert all(torch.equal(ho[r], want[r]) for r in range(3))\n"
        "assert torch.equal(one, want[1])\n"
        "print('ok')\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, H3B_DEBUG="1", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600, cwd=root)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


def test_768x1344_full_denoise_is_finite_and_deterministic():
    cfg = synth.CONFIGS["dit768x1344"]
    m = DiTDenoiser(cfg, gen_device="cuda")
    x0 = synth.latent_noise(cfg, device="cuda")
    a = x0.clone()
    b = x0.clone()
    m.run(a)
    m.run(b)
    h3b.sync_status()
    assert torch.isfinite(a).all()
    assert torch.equal(a, b)
    # the state moved by the four Euler updates
    assert (a - x0).abs().mean().item() > 0.1


@pytest.mark.parametrize("name", ["tiny", "dit512", "dit512_tokred"])
def test_cuda_graph_replay_matches_direct_run(name):
    # replays reuse every kernel argument, including the stream-K sequence numbers of the
    # long-K GEMMs, so this also checks that a replay waits for its own partial tiles
    cfg = synth.CONFIGS[name]
    m = DiTDenoiser(cfg)
    x0 = synth.latent_noise(cfg).to(DEV)
    ref = x0.clone()
    m.run(ref)
    h3b.sync_status()
    xg = x0.clone()
    graph = m.capture(xg)
    for _ in range(3):
        xg.copy_(x0)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(xg, ref)
    del graph


# ------------------------------------------------------------------------------ reuse policies
@pytest.mark.parametrize("mode,every", [("velocity", 2), ("core", 2), ("core", 3),
                                        ("velocity", 1)])
def test_tiny_reuse_policies_vs_oracle(mode, every):
    # a whole 4-step denoise of the tiny workload under a reuse policy
    # (dothoosh.com "Aggressive optimisation levers"; aihot.vn section 4)
    cfg = synth.CONFIGS["tiny"]
    m = DiTDenoiser(cfg, keep_host_params=True)
    x0 = synth.latent_noise(cfg)
    x = x0.to(DEV)
    fresh = m.run_reuse(x, every, mode)
    h3b.sync_status()
    assert fresh == int(O.reuse_schedule(cfg.steps, every).sum())
    blocks = [{k: f64(v) for k, v in p.items()} for p in m.host_params]
    final = {k: f64(v) for k, v in m.host_final.items()}
    want = workloads.denoise_reuse(cfg, blocks, final, f64(synth.conditioning(cfg)), f64(x0),
                                   every, mode)
    got = x.cpu().numpy().astype(np.float64)
    assert rel_l2(got, want) < TOL_STEPS
    assert rel_l2(got - f64(x0), want - f64(x0)) < TOL_STEPS


@pytest.mark.parametrize("name", ["dit512_reuse_velocity2", "dit512_reuse_core3"])
def test_512_reuse_policies_vs_golden(name):
    ref = np.load(os.path.join(GOLDEN, f"{name}_oracle.npz"))
    mode = "velocity" if "velocity" in name else "core"
    every = int(name[-1])
    cfg = synth.CONFIGS["dit512"]
    m = DiTDenoiser(cfg)
    x0 = synth.latent_noise(cfg)
    x = x0.to(DEV)
    m.run_reuse(x, every, mode)
    h3b.sync_status()
    rows = ref["rows"]
    got = x.cpu().numpy()[rows].astype(np.float64)
    base = f64(x0)[rows]
    want = ref["final"].astype(np.float64)
    assert rel_l2(got, want) < TOL_STEPS
    assert rel_l2(got - base, want - base) < TOL_STEPS


def test_reuse_every_one_matches_the_plain_run_bit_for_bit():
    cfg = synth.CONFIGS["dit512"]
    m = DiTDenoiser(cfg)
    x0 = synth.latent_noise(cfg).to(DEV)
    a, b, c = x0.clone(), x0.clone(), x0.clone()
    m.run(a)
    m.run_reuse(b, 1, "velocity")
    m.run_reuse(c, 1, "core")
    h3b.sync_status()
    assert torch.equal(a, b) and torch.equal(a, c)
