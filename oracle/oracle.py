"""CPU oracle of the DiT-block denoising path.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and ``bench.py``'s
cpu_baseline / reference leg may import or run this module.  The product (the CUDA
library under ``video_diffusion_transformer_03_b200/``) never calls it and shares no
code with it; it imports nothing but numpy.

Every function is the plain definition of one step, in float64 by default (``dt``
selects float32 for the self-consistency pin), written for readability, not speed.
Library primitives (numpy matmul, exp, tanh) serve as steps; there is no blocking,
fusion or reordering beyond what the definitions state.

Sources ("pages"):
  [ditty]   "h3: native MiniMax-H3 on Apple Silicon", news.ditty.ir
  [aihot]   "H3-metal: running MiniMax-H3 directly on Apple Silicon", aihot.vn
            (README translation; sections 2 "First fast video", 4 "Speed/quality
            presets", 5 "Resolution and duration")
  [dothoosh] "How h3.c cuts MiniMax-H3 video inference to 3.5 seconds", dothoosh.com
            (sections "DiT fusions and memory management", "Aggressive optimisation
            levers", "The powerful int8 path")
  [wqu]     "h3-metal: native MiniMax-H3 inference on Apple Silicon", wqu.guru
  [iitog]   "H3-metal: native inference of MiniMax-H3", iitog.ru

The pages name the block's pieces but print no equations, dimensions or values.  Where
they are silent this oracle takes the plain DiT reading, listed per function below:
LayerNorm without affine and eps 1e-6; modulation LN(x)*(1+scale)+shift; DiT order
(shift, scale, gate) x (attention, MLP) of the AdaLN vectors; tanh-form GELU; RoPE on
adjacent pairs within per-axis chunks of the head dimension; audio tokens at position
(0, 0, 0); Euler velocity = the final AdaLN output.

Parity pins: see tests/test_oracle_pins.py.  Parity of the composed block and of the
multi-step trajectory against the pages is unpinned (the pages print no values); the
pieces are pinned individually.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64

MOD_NAMES = ("shift_msa", "scale_msa", "gate_msa", "shift_mlp", "scale_mlp", "gate_mlp")


# --------------------------------------------------------------------------------------
# a1: AdaLN modulation vectors
# --------------------------------------------------------------------------------------
def adaln_modulation(w_ada, b_ada, c, d: int, dt=F64) -> np.ndarray:
    """mod = W_ada c + b_ada, reshaped to [6, d] in DiT order (shift, scale, gate) for the
    attention branch then the MLP branch.  A plain linear layer of the conditioning
    vector (no SiLU), as the tiny workload's recipe states.  The per-block gates that
    this produces are what layer thinning ranks ([dothoosh] "Aggressive optimisation
    levers")."""
    w = np.asarray(w_ada, dt)
    out = w @ np.asarray(c, dt) + np.asarray(b_ada, dt)
    return out.reshape(6, d)


def final_modulation(w_fin, b_fin, c, d: int, dt=F64) -> np.ndarray:
    """Final AdaLN vectors per stream: [2 streams (video, audio), 2 (shift, scale), d].
    One linear layer per stream ([dothoosh] "DiT fusions and memory management": the
    final AdaLN runs separately for the video and audio parts of one residual buffer)."""
    w = np.asarray(w_fin, dt)
    b = np.asarray(b_fin, dt)
    cc = np.asarray(c, dt)
    return np.stack([(w[s] @ cc + b[s]).reshape(2, d) for s in range(2)])


# --------------------------------------------------------------------------------------
# a2 / a6 / a8: LayerNorm + AdaLN modulation
# --------------------------------------------------------------------------------------
def layer_norm(x, eps: float, dt=F64) -> np.ndarray:
    """LayerNorm over the last axis without affine parameters, biased variance."""
    x = np.asarray(x, dt)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + dt(eps))


def modulate(xn, shift, scale, dt=F64) -> np.ndarray:
    """AdaLN modulation: xn * (1 + scale) + shift, vectors broadcast over tokens."""
    return np.asarray(xn, dt) * (1 + np.asarray(scale, dt)) + np.asarray(shift, dt)


def gated_residual(x, gate, y, dt=F64) -> np.ndarray:
    """x + gate * y ([dothoosh] "DiT fusions and memory management": each branch's
    output enters the residual stream through its AdaLN gate)."""
    return np.asarray(x, dt) + np.asarray(gate, dt) * np.asarray(y, dt)


# --------------------------------------------------------------------------------------
# a4: 3D RoPE
# --------------------------------------------------------------------------------------
def rope_positions(grid: Sequence[int], n_audio: int, halved: bool = False,
                   paired: bool = False, dt=F64) -> np.ndarray:
    """Token positions [N, 3] as (t, h, w).

    Video tokens come first in (t, h, w) raster order, then the audio tokens.
    * halved: spatial coordinates (h, w) divided by 2 -- the small-canvas variant
      ([aihot] section 5: at a 256x256 canvas the spatial RoPE coordinates are halved).
    * paired: after horizontal token pairing the grid has w/2 columns; merged token j
      sits at the mean of its two sources, w = 2j + 0.5.
    * audio tokens: position (0, 0, 0), an identity rotation (the pages give audio no
      grid; reading of this build).
    """
    t_n, h_n, w_n = grid
    if paired:
        w_idx = np.arange(w_n // 2, dtype=dt) * 2 + 0.5
    else:
        w_idx = np.arange(w_n, dtype=dt)
    tt, hh, ww = np.meshgrid(np.arange(t_n, dtype=dt), np.arange(h_n, dtype=dt), w_idx,
                             indexing="ij")
    vid = np.stack([tt.ravel(), hh.ravel(), ww.ravel()], axis=1)
    if halved:
        vid[:, 1] /= 2
        vid[:, 2] /= 2
    aud = np.zeros((n_audio, 3), dt)
    return np.concatenate([vid, aud], axis=0)


def rope_rotate(x, pos, split: Sequence[int], theta: float, dt=F64) -> np.ndarray:
    """Rotate x [N, H, hd] by 3D RoPE.

    The head dimension is cut into consecutive chunks of widths split = (D_t, D_h, D_w)
    for the axes (t, h, w).  Inside the chunk of axis a, pair k is the adjacent pair of
    channels (2k, 2k+1); its angle is pos[:, a] * theta ** (-2k / D_a), and the pair
    (x0, x1) becomes (x0 cos - x1 sin, x0 sin + x1 cos).
    """
    x = np.array(x, dtype=dt, copy=True)
    pos = np.asarray(pos, dt)
    out = x.copy()
    off = 0
    for axis, width in enumerate(split):
        for k in range(width // 2):
            freq = dt(theta) ** (-2.0 * k / width)
            ang = pos[:, axis] * freq                       # [N]
            cos = np.cos(ang)[:, None]
            sin = np.sin(ang)[:, None]
            i0 = off + 2 * k
            x0 = x[:, :, i0]
            x1 = x[:, :, i0 + 1]
            out[:, :, i0] = x0 * cos - x1 * sin
            out[:, :, i0 + 1] = x0 * sin + x1 * cos
        off += width
    assert off == x.shape[-1], "RoPE split must cover the head dimension"
    return out


# --------------------------------------------------------------------------------------
# f2: Q/K RMSNorm (before RoPE)
# --------------------------------------------------------------------------------------
def rms_norm(x, gain, eps: float, dt=F64) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gain.

    Applied to each head of q and k inside the QKV projection's tile, before the rotation
    ([dothoosh] "The powerful int8 path": RMS normalisation and RoPE for Q/K in the QKV
    tile).  Reading: per head over the head dimension, one learned gain vector [hd] for q
    and one for k, shared by the heads; eps as the LayerNorm's."""
    x = np.asarray(x, dt)
    ms = (x * x).mean(axis=-1, keepdims=True)
    return x / np.sqrt(ms + dt(eps)) * np.asarray(gain, dt)


# --------------------------------------------------------------------------------------
# a5: joint self-attention
# --------------------------------------------------------------------------------------
def attention(q, k, v, q_rows: Optional[np.ndarray] = None, dt=F64) -> np.ndarray:
    """Full (non-causal) softmax attention per head over all tokens of the joint
    video+audio stream: O = softmax(q k^T / sqrt(hd)) v, max-subtracted softmax.
    q, k, v: [N, H, hd].  q_rows selects the query tokens to evaluate (all if None)."""
    q = np.asarray(q, dt)
    k = np.asarray(k, dt)
    v = np.asarray(v, dt)
    if q_rows is not None:
        q = q[q_rows]
    hd = q.shape[-1]
    out = np.empty(q.shape, dt)
    for h in range(q.shape[1]):
        s = (q[:, h, :] @ k[:, h, :].T) / math.sqrt(hd)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out


# --------------------------------------------------------------------------------------
# a7: GELU
# --------------------------------------------------------------------------------------
def gelu_tanh(x, dt=F64) -> np.ndarray:
    """tanh-form GELU: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, dt)
    return 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))


# --------------------------------------------------------------------------------------
# one DiT block (a2..a8)
# --------------------------------------------------------------------------------------
def block_forward(x, w: Dict[str, np.ndarray], mod, pos, n_heads: int,
                  split: Sequence[int], theta: float, eps: float,
                  mod_next=None, rows: Optional[np.ndarray] = None,
                  dt=F64) -> Tuple[np.ndarray, Optional[np.ndarray]]:
    """One DiT block on the residual stream x [N, d]; returns (x_out, h_next).

    Steps in the pages' order ([dothoosh] "DiT fusions and memory management"):
      h  = LN(x) (1 + scale_msa) + shift_msa
      q, k, v = split(h W_qkv^T + b_qkv); q, k rotated by 3D RoPE (after a per-head
                RMSNorm with gains w["q_norm"], w["k_norm"] when the block has them)
      o  = attention(q, k, v)
      x1 = x + gate_msa (o W_o^T + b_o)           (attention gate -> MLP AdaLN)
      h2 = LN(x1) (1 + scale_mlp) + shift_mlp
      g  = GELU(h2 W_fc1^T + b_fc1)
      x2 = x1 + gate_mlp (g W_fc2^T + b_fc2)      (MLP gate -> next block's AdaLN)
      h_next = LN(x2) (1 + scale_msa') + shift_msa'  with the next block's vectors
    ``rows`` evaluates the block for a subset of query tokens (keys and values still
    come from every token); x_out / h_next then hold those rows only.
    """
    x = np.asarray(x, dt)
    mod = np.asarray(mod, dt)
    n, d = x.shape
    hd = d // n_heads
    sel = np.arange(n) if rows is None else np.asarray(rows)

    h = modulate(layer_norm(x, eps, dt), mod[0], mod[1], dt)
    w_qkv = np.asarray(w["w_qkv"], dt)
    b_qkv = np.asarray(w["b_qkv"], dt)
    # keys and values for every token, queries for the selected ones
    kv = h @ w_qkv[d:].T + b_qkv[d:]
    k = kv[:, :d].reshape(n, n_heads, hd)
    v = kv[:, d:].reshape(n, n_heads, hd)
    q = (h[sel] @ w_qkv[:d].T + b_qkv[:d]).reshape(len(sel), n_heads, hd)
    if w.get("q_norm") is not None:
        q = rms_norm(q, w["q_norm"], eps, dt)
        k = rms_norm(k, w["k_norm"], eps, dt)
    k = rope_rotate(k, pos, split, theta, dt)
    q = rope_rotate(q, np.asarray(pos)[sel], split, theta, dt)
    o = attention(q, k, v, dt=dt).reshape(len(sel), d)

    x1 = gated_residual(x[sel], mod[2], o @ np.asarray(w["w_o"], dt).T + np.asarray(w["b_o"], dt), dt)
    h2 = modulate(layer_norm(x1, eps, dt), mod[3], mod[4], dt)
    g = gelu_tanh(h2 @ np.asarray(w["w_fc1"], dt).T + np.asarray(w["b_fc1"], dt), dt)
    x2 = gated_residual(x1, mod[5], g @ np.asarray(w["w_fc2"], dt).T + np.asarray(w["b_fc2"], dt), dt)
    h_next = None
    if mod_next is not None:
        mn = np.asarray(mod_next, dt)
        h_next = modulate(layer_norm(x2, eps, dt), mn[0], mn[1], dt)
    return x2, h_next


# --------------------------------------------------------------------------------------
# a9: final AdaLN per stream + Euler update
# --------------------------------------------------------------------------------------
def final_adaln(x_l, final_mod, n_video: int, eps: float, dt=F64) -> np.ndarray:
    """Velocity v = LN(x_L)(1 + scale_s) + shift_s with s = video for the first n_video
    rows and audio for the rest, both read from one residual buffer ([dothoosh] "DiT
    fusions and memory management": final AdaLN bound to the stream offsets).  The
    patch/head projection is outside this path, so v lives in model space [N, d]."""
    fm = np.asarray(final_mod, dt)
    xn = layer_norm(x_l, eps, dt)
    v = np.empty_like(xn)
    v[:n_video] = modulate(xn[:n_video], fm[0, 0], fm[0, 1], dt)
    v[n_video:] = modulate(xn[n_video:], fm[1, 0], fm[1, 1], dt)
    return v


def sigma_grid(steps: int, dt=F64) -> np.ndarray:
    """Linear sigma grid from 1 to 0 with the endpoint included: steps + 1 values
    ([aihot] section 2: the retained schedule is the released linear base grid with one
    endpoint; --steps N means exactly N passes)."""
    return np.linspace(1.0, 0.0, steps + 1, dtype=dt)


def euler_update(x_state, v, sigma: float, sigma_next: float, dt=F64) -> np.ndarray:
    """x <- x + (sigma_next - sigma) v."""
    return np.asarray(x_state, dt) + (dt(sigma_next) - dt(sigma)) * np.asarray(v, dt)


# --------------------------------------------------------------------------------------
# a10: horizontal token pairing and its bypass restore
# --------------------------------------------------------------------------------------
def token_pair(x, grid: Sequence[int], n_audio: int, dt=F64) -> np.ndarray:
    """Average horizontally adjacent video tokens (t, h, 2j) and (t, h, 2j+1) into
    (t, h, j); audio tokens are copied ([ditty], [dothoosh] "Aggressive optimisation
    levers": horizontal video tokens are paired after block 3)."""
    x = np.asarray(x, dt)
    t_n, h_n, w_n = grid
    nv = t_n * h_n * w_n
    vid = x[:nv].reshape(t_n, h_n, w_n // 2, 2, -1)
    red = 0.5 * (vid[:, :, :, 0, :] + vid[:, :, :, 1, :])
    return np.concatenate([red.reshape(-1, x.shape[1]), x[nv:nv + n_audio]], axis=0)


def token_unpair(x_red, grid: Sequence[int], n_audio: int, saved=None, dt=F64) -> np.ndarray:
    """Restore full horizontal resolution.

    With ``saved`` (the full-resolution stream at the moment of pairing), the bypass
    restore: x[t,h,2j+k] = saved[t,h,2j+k] + (x_red[t,h,j] - pair(saved)[t,h,j]), so
    detail that pairing averaged away comes back from the bypass and the reduced
    blocks' update is added to both tokens ([dothoosh] "Aggressive optimisation levers":
    a bypass restores full resolution before the late blocks).
    Without ``saved``: each reduced token is duplicated into its two sources."""
    x_red = np.asarray(x_red, dt)
    t_n, h_n, w_n = grid
    nv_red = t_n * h_n * (w_n // 2)
    d = x_red.shape[1]
    upd = x_red[:nv_red].reshape(t_n, h_n, w_n // 2, 1, d)
    if saved is None:
        vid = np.broadcast_to(upd, (t_n, h_n, w_n // 2, 2, d))
    else:
        saved = np.asarray(saved, dt)
        delta = upd - token_pair(saved, grid, 0, dt)[:nv_red].reshape(t_n, h_n, w_n // 2, 1, d)
        vid = saved[:t_n * h_n * w_n].reshape(t_n, h_n, w_n // 2, 2, d) + delta
    return np.concatenate([vid.reshape(-1, d), x_red[nv_red:nv_red + n_audio]], axis=0)


# --------------------------------------------------------------------------------------
# layer thinning (host policy; the mask is an input of the denoise step)
# --------------------------------------------------------------------------------------
def layer_mask(mods, n_active: int) -> np.ndarray:
    """Choose the active blocks: rank blocks by their AdaLN gates and keep the first and
    last blocks ([dothoosh] "Aggressive optimisation levers").  Reading: score_b =
    mean|gate_msa| + mean|gate_mlp|; drop the lowest-scoring interior blocks, dropping
    the higher index first on ties."""
    mods = np.asarray(mods, F64)
    nb = mods.shape[0]
    keep = np.ones(nb, dtype=bool)
    n_drop = nb - n_active
    if n_drop <= 0:
        return keep
    assert n_drop <= nb - 2, "first and last blocks are always kept"
    score = np.abs(mods[:, 2]).mean(axis=1) + np.abs(mods[:, 5]).mean(axis=1)
    interior = list(range(1, nb - 1))
    interior.sort(key=lambda b: (score[b], -b))
    for b in interior[:n_drop]:
        keep[b] = False
    return keep


# --------------------------------------------------------------------------------------
# the Euler denoising loop (one evaluation of every active block per step)
# --------------------------------------------------------------------------------------
def denoise(x0, blocks: List[Dict[str, np.ndarray]], mods, final_mod, grid, n_audio: int,
            n_heads: int, split, theta: float, eps: float, steps: int, run_steps: int,
            active=None, reduce_after: int = -1, halved: bool = False,
            unpair_bypass: bool = True, dt=F64, trace: Optional[list] = None) -> np.ndarray:
    """Run ``run_steps`` Euler steps of the linear sigma grid.  Each step: the block input
    is the state rounded to bf16 (the residual stream is stored in bf16, as the pages'
    kernels do), every active block runs, tokens are paired after ``reduce_after``
    executed blocks and restored before the final AdaLN, then x += (s' - s) v."""
    x_state = np.asarray(x0, dt)
    sig = sigma_grid(steps, dt)
    nb = len(blocks)
    act = np.ones(nb, bool) if active is None else np.asarray(active, bool)
    order = [b for b in range(nb) if act[b]]
    nv = grid[0] * grid[1] * grid[2]
    pos_full = rope_positions(grid, n_audio, halved=halved, dt=dt)
    pos_red = rope_positions(grid, n_audio, halved=halved, paired=True, dt=dt)
    for i in range(run_steps):
        x = round_to_bf16(x_state).astype(dt)
        saved = None
        pos = pos_full
        for n_exec, b in enumerate(order, start=1):
            x, _ = block_forward(x, blocks[b], mods[b], pos, n_heads, split, theta, eps, dt=dt)
            if n_exec == reduce_after and n_exec < len(order):
                saved = x
                x = token_pair(x, grid, n_audio, dt)
                pos = pos_red
        if saved is not None:
            x = token_unpair(x, grid, n_audio, saved if unpair_bypass else None, dt)
        v = final_adaln(x, final_mod, nv, eps, dt)
        x_state = euler_update(x_state, v, sig[i], sig[i + 1], dt)
        if trace is not None:
            trace.append(x_state.copy())
    return x_state


def round_to_bf16(x) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even); returns float32."""
    a = np.ascontiguousarray(np.asarray(x, np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    nan = np.isnan(a)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    out = u.astype(np.uint32).view(np.float32).copy()
    out[nan] = np.nan
    return out


# --------------------------------------------------------------------------------------
# a11: int8 row-scaled FC2
# --------------------------------------------------------------------------------------
def quantize_rows(a) -> Tuple[np.ndarray, np.ndarray]:
    """Symmetric int8 quantisation with one fp32 scale per row ([aihot] section 4 /
    [dothoosh] "The powerful int8 path": one activation scale per FC2 row).

    In IEEE float32, round-to-nearest: absmax = max|a_row|, inv = 127 / absmax,
    q = clamp(round_half_even(a * inv), -127, 127), scale = absmax / 127.  A zero row
    gives q = 0 and scale = 0."""
    a = np.asarray(a, np.float32)
    absmax = np.max(np.abs(a), axis=1)
    q = np.zeros(a.shape, np.int8)
    scale = np.zeros(a.shape[0], np.float32)
    nz = absmax > 0
    inv = np.float32(127.0) / absmax[nz]
    prod = (a[nz] * inv[:, None]).astype(np.float32)
    q[nz] = np.clip(np.rint(prod), -127, 127).astype(np.int8)
    scale[nz] = absmax[nz] / np.float32(127.0)
    return q, scale


def int_matmul(qa, qb) -> np.ndarray:
    """Exact integer product acc[m, n] = sum_k qa[m, k] qb[n, k] as int64.

    Every product is at most 127^2 and every partial sum stays below 2^53 for K < 5.5e8,
    so float64 accumulation is exact whatever the summation order; the BLAS routine is
    used as the summation step."""
    K = qa.shape[1]
    assert K * 127 * 127 < 2 ** 53
    acc = np.asarray(qa, F64) @ np.asarray(qb, F64).T
    return acc.astype(np.int64)


def fc2_int8_row(act, w_q, w_scale, gate, resid, bias=None, rows=None):
    """Int8 row-scaled FC2 with gated residual.

    q, s_r = quantize_rows(act); acc = q w_q^T (exact integers);
    y = acc * s_r * s_c (+ bias); out = resid + gate * y.  Returns (q, s_r, acc, out);
    acc is int64, out float64.  ``rows`` restricts the evaluation to a subset of rows."""
    act = np.asarray(act, np.float32)
    if rows is not None:
        act = act[rows]
        resid = np.asarray(resid)[rows]
    q, s_r = quantize_rows(act)
    acc = int_matmul(q, w_q)
    y = acc.astype(F64) * np.asarray(s_r, F64)[:, None] * np.asarray(w_scale, F64)[None, :]
    if bias is not None:
        y = y + np.asarray(bias, F64)[None, :]
    out = np.asarray(resid, F64) + np.asarray(gate, F64)[None, :] * y
    return q, s_r, acc, out


# --------------------------------------------------------------------------------------
# reuse policies: whole-velocity reuse and core-residual reuse
# --------------------------------------------------------------------------------------
def reuse_schedule(steps: int, every: int) -> np.ndarray:
    """Which Euler steps evaluate the model when only every `every`-th one does.

    [aihot] section 4 and [dothoosh] "Aggressive optimisation levers": at 20 steps,
    reuse 1, 2 and 3 evaluate the denoiser 20, 11 and 8 times.  Reading that fits those
    counts: step i is fresh when i % every == 0, and the last step is always fresh."""
    i = np.arange(steps)
    return (i % every == 0) | (i == steps - 1)


def denoise_velocity_reuse(x0, blocks, mods, final_mod, grid, n_audio: int, n_heads: int,
                           split, theta: float, eps: float, steps: int, reuse: int,
                           active=None, reduce_after: int = -1, halved: bool = False,
                           unpair_bypass: bool = True, dt=F64) -> np.ndarray:
    """Euler loop with whole-velocity reuse ([dothoosh] "Aggressive optimisation levers":
    the skipped transitions are extrapolated).  Reading: a fresh step runs the model and
    keeps its velocity; a skipped step takes the Euler transition with the velocity of the
    last fresh step."""
    fresh = reuse_schedule(steps, reuse)
    sig = sigma_grid(steps, dt)
    x_state = np.asarray(x0, dt)
    v = None
    for i in range(steps):
        if fresh[i]:
            x_l = _core(x_state, blocks, mods, grid, n_audio, n_heads, split, theta, eps,
                        active, reduce_after, halved, unpair_bypass, dt)
            v = final_adaln(x_l, final_mod, grid[0] * grid[1] * grid[2], eps, dt)
        x_state = euler_update(x_state, v, sig[i], sig[i + 1], dt)
    return x_state


def denoise_core_reuse(x0, blocks, mods, final_mod, grid, n_audio: int, n_heads: int,
                       split, theta: float, eps: float, steps: int, reuse: int,
                       active=None, reduce_after: int = -1, halved: bool = False,
                       unpair_bypass: bool = True, dt=F64) -> np.ndarray:
    """Euler loop with core-residual reuse ([aihot] section 4, [dothoosh] "Aggressive
    optimisation levers": the work around the core is refreshed every step, the expensive
    core runs less often).  Reading: the core is the stack of DiT blocks, with residual
    r = x_L - x_in; a fresh step (same schedule as reuse_schedule) runs the core and keeps
    r; a skipped step takes x_L = bf16(x_in + r) with its own x_in = bf16(x_state), and
    the final AdaLN and the Euler update run every step."""
    fresh = reuse_schedule(steps, reuse)
    sig = sigma_grid(steps, dt)
    x_state = np.asarray(x0, dt)
    nv = grid[0] * grid[1] * grid[2]
    r = None
    for i in range(steps):
        x_in = round_to_bf16(x_state).astype(dt)
        if fresh[i]:
            x_l = _core(x_state, blocks, mods, grid, n_audio, n_heads, split, theta, eps,
                        active, reduce_after, halved, unpair_bypass, dt)
            r = x_l - x_in
        else:
            x_l = round_to_bf16(x_in + r).astype(dt)
        v = final_adaln(x_l, final_mod, nv, eps, dt)
        x_state = euler_update(x_state, v, sig[i], sig[i + 1], dt)
    return x_state


def _core(x_state, blocks, mods, grid, n_audio, n_heads, split, theta, eps, active,
          reduce_after, halved, unpair_bypass, dt):
    """The block stack of one Euler step on bf16(x_state): the same sequence as one step
    of denoise() up to (not including) the final AdaLN."""
    nb = len(blocks)
    act = np.ones(nb, bool) if active is None else np.asarray(active, bool)
    order = [b for b in range(nb) if act[b]]
    pos = rope_positions(grid, n_audio, halved=halved, dt=dt)
    pos_red = rope_positions(grid, n_audio, halved=halved, paired=True, dt=dt)
    x = round_to_bf16(x_state).astype(dt)
    saved = None
    for n_exec, b in enumerate(order, start=1):
        x, _ = block_forward(x, blocks[b], mods[b], pos, n_heads, split, theta, eps, dt=dt)
        if n_exec == reduce_after and n_exec < len(order):
            saved = x
            x = token_pair(x, grid, n_audio, dt)
            pos = pos_red
    if saved is not None:
        x = token_unpair(x, grid, n_audio, saved if unpair_bypass else None, dt)
    return x


# --------------------------------------------------------------------------------------
# f1: patch embedding and final heads (the steps on either side of the block stack)
# --------------------------------------------------------------------------------------
def patch_embed(latent, n_video: int, w_patch, b_patch, dt=F64) -> np.ndarray:
    """Model-space input of the block stack from the per-token latent [N, C]: one linear
    projection per stream (video rows [0, n_video), audio rows after), x = latent W^T + b.
    w_patch [2 streams, d, C], b_patch [2, d].  The latent enters as bf16 (the GPU's
    operand precision; the state itself stays fp32).  Reading: the pages name patch and
    head work around the core ([aihot] section 4: core-residual reuse refreshes patch/head
    every step) but give no dimensions; C is a parameter of the workload."""
    lat = round_to_bf16(latent).astype(dt)
    w = np.asarray(w_patch, dt)
    b = np.asarray(b_patch, dt)
    out = np.empty((lat.shape[0], w.shape[1]), dt)
    out[:n_video] = lat[:n_video] @ w[0].T + b[0]
    out[n_video:] = lat[n_video:] @ w[1].T + b[1]
    return out


def final_head(x_l, final_mod, n_video: int, eps: float, w_head, b_head, dt=F64) -> np.ndarray:
    """Latent velocity: the per-stream final AdaLN of x_L followed by that stream's linear
    head, v = (LN(x_L)(1 + scale_s) + shift_s) W_s^T + b_s ([dothoosh] "DiT fusions and
    memory management": the final BF16 heads apply the AdaLN as they load their tiles).
    w_head [2, C, d], b_head [2, C]."""
    h = final_adaln(x_l, final_mod, n_video, eps, dt)
    w = np.asarray(w_head, dt)
    b = np.asarray(b_head, dt)
    v = np.empty((h.shape[0], w.shape[1]), dt)
    v[:n_video] = h[:n_video] @ w[0].T + b[0]
    v[n_video:] = h[n_video:] @ w[1].T + b[1]
    return v


def denoise_latent(lat0, blocks, mods, final_mod, heads, grid, n_audio: int, n_heads: int,
                   split, theta: float, eps: float, steps: int, run_steps: int, active=None,
                   reduce_after: int = -1, halved: bool = False, unpair_bypass: bool = True,
                   dt=F64, first_step: int = 0) -> np.ndarray:
    """The Euler loop on the latent: each step x = bf16(patch_embed(latent)) (the residual
    stream is stored in bf16), the block stack as in denoise(), then
    latent += (s' - s) final_head(x_L).  heads: dict with w_patch, b_patch, w_head,
    b_head.  Runs steps first_step .. first_step + run_steps - 1 of the sigma grid."""
    sig = sigma_grid(steps, dt)
    lat = np.asarray(lat0, dt)
    nv = grid[0] * grid[1] * grid[2]
    for i in range(first_step, first_step + run_steps):
        x = patch_embed(lat, nv, heads["w_patch"], heads["b_patch"], dt)
        x_l = _core(x, blocks, mods, grid, n_audio, n_heads, split, theta, eps, active,
                    reduce_after, halved, unpair_bypass, dt)
        v = final_head(x_l, final_mod, nv, eps, heads["w_head"], heads["b_head"], dt)
        lat = euler_update(lat, v, sig[i], sig[i + 1], dt)
    return lat


# --------------------------------------------------------------------------------------
# f3: grouped int8 MLP and int8 QKV
# --------------------------------------------------------------------------------------
def quantize_groups(a, group: int) -> Tuple[np.ndarray, np.ndarray]:
    """Symmetric int8 quantisation with one fp32 scale per row and per `group` consecutive
    columns ([dothoosh] "The powerful int8 path": the FC2 input has one scale per 1024
    channels).  Each (row, group) follows quantize_rows' rule.  Returns q [M, K] int8 and
    scales [M, K / group] fp32."""
    a = np.asarray(a, np.float32)
    m, k = a.shape
    assert k % group == 0
    g = a.reshape(m * (k // group), group)
    q, s = quantize_rows(g)
    return q.reshape(m, k), s.reshape(m, k // group)


def int8_grouped_matmul(q, s_a, w_q, w_scale, group: int, dt=F64) -> np.ndarray:
    """y[m, n] = w_scale[n] sum_g s_a[m, g] acc_g[m, n] with the exact integer group sums
    acc_g = sum over the group's k of q[m, k] w_q[n, k]."""
    m, k = q.shape
    y = np.zeros((m, w_q.shape[0]), dt)
    for gi in range(k // group):
        sl = slice(gi * group, (gi + 1) * group)
        acc = int_matmul(q[:, sl], w_q[:, sl]).astype(dt)
        y += np.asarray(s_a[:, gi], dt)[:, None] * acc
    return y * np.asarray(w_scale, dt)[None, :]


def int8_linear_rows(a, w_q, w_scale, bias=None, dt=F64) -> np.ndarray:
    """Linear layer on int8 operands with one scale per activation row and per weight
    output channel: y = (q_a w_q^T) s_a s_w (+ b), q_a, s_a = quantize_rows(a)."""
    q, s = quantize_rows(a)
    y = int_matmul(q, w_q).astype(dt) * np.asarray(s, dt)[:, None] * np.asarray(w_scale, dt)[None, :]
    if bias is not None:
        y = y + np.asarray(bias, dt)[None, :]
    return y


def block_forward_int8(x, w: Dict[str, np.ndarray], mod, pos, n_heads: int, split,
                       theta: float, eps: float, group: int = 1024, rows=None,
                       dt=F64) -> np.ndarray:
    """block_forward with the int8 path of [dothoosh] "The powerful int8 path": the QKV and
    FC1 inputs (the AdaLN outputs) quantised per token row, the FC2 input (the GELU
    output) per token and per `group` channels, weights per output channel
    (w["w_qkv_q"], w["s_qkv"], ...: quantize_rows of the bf16 weights); the attention and
    the output projection stay bf16.  The QKV and FC1 inputs are quantised from fp32 values
    (in the LayerNorm kernel, before any storage); the FC2 input from the stored bf16 GELU
    output."""
    x = np.asarray(x, dt)
    mod = np.asarray(mod, dt)
    n, d = x.shape
    hd = d // n_heads
    sel = np.arange(n) if rows is None else np.asarray(rows)
    h = modulate(layer_norm(x, eps, dt), mod[0], mod[1], dt)
    qkv = int8_linear_rows(h.astype(np.float32), w["w_qkv_q"], w["s_qkv"],
                           np.asarray(w["b_qkv"], dt), dt)
    q = qkv[sel, :d].reshape(len(sel), n_heads, hd)
    k = qkv[:, d:2 * d].reshape(n, n_heads, hd)
    v = qkv[:, 2 * d:].reshape(n, n_heads, hd)
    if w.get("q_norm") is not None:
        q = rms_norm(q, w["q_norm"], eps, dt)
        k = rms_norm(k, w["k_norm"], eps, dt)
    k = rope_rotate(k, pos, split, theta, dt)
    q = rope_rotate(q, np.asarray(pos)[sel], split, theta, dt)
    o = attention(q, k, v, dt=dt).reshape(len(sel), d)
    x1 = gated_residual(x[sel], mod[2], o @ np.asarray(w["w_o"], dt).T + np.asarray(w["b_o"], dt), dt)
    # the residual is stored in bf16 between the two halves ([dothoosh] "DiT fusions and
    # memory management": the bf16-rounded residual feeds the MLP's AdaLN); the FC1 input
    # codes are decided on the LayerNorm of that stored value.  The gated residual add
    # keeps x1 itself, so zero gates still give the identity on any input.
    x1_stored = round_to_bf16(x1).astype(dt)
    h2 = modulate(layer_norm(x1_stored, eps, dt), mod[3], mod[4], dt)
    g = gelu_tanh(int8_linear_rows(h2.astype(np.float32), w["w_fc1_q"], w["s_fc1"],
                                   np.asarray(w["b_fc1"], dt), dt), dt)
    # the FC2 input is quantised as it is stored, in bf16 (the activations of the int8
    # FC2 workload are bf16 too)
    qg, sg = quantize_groups(round_to_bf16(g), group)
    y = int8_grouped_matmul(qg, sg, w["w_fc2_q"], w["s_fc2"], group, dt) + np.asarray(w["b_fc2"], dt)
    return gated_residual(x1, mod[5], y, dt)
