"""Pins of the CPU oracle against things other than itself: closed forms, brute force on
tiny inputs, library routines, invariants and exact identities.  No GPU needed."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O

RNG = np.random.default_rng(1234)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ----------------------------------------------------------------------------- attention
def test_attention_bruteforce_loops():
    n, h, hd = 5, 2, 4
    q, k, v = (RNG.standard_normal((n, h, hd)) for _ in range(3))
    out = O.attention(q, k, v)
    for head in range(h):
        for i in range(n):
            scores = [sum(q[i, head, c] * k[j, head, c] for c in range(hd)) / math.sqrt(hd)
                      for j in range(n)]
            w = [math.exp(s) for s in scores]          # no max subtraction: tiny values
            z = sum(w)
            for c in range(hd):
                ref = sum(w[j] * v[j, head, c] for j in range(n)) / z
                assert abs(out[i, head, c] - ref) < 1e-12


def test_attention_vs_torch_sdpa():
    n, h, hd = 37, 3, 16
    q, k, v = (RNG.standard_normal((n, h, hd)) * 2 for _ in range(3))
    out = O.attention(q, k, v)
    tq, tk, tv = (torch.from_numpy(a).permute(1, 0, 2) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(1, 0, 2).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12


def test_attention_q_rows_subset():
    n, h, hd = 20, 2, 8
    q, k, v = (RNG.standard_normal((n, h, hd)) for _ in range(3))
    rows = np.array([0, 7, 19])
    assert np.array_equal(O.attention(q, k, v, q_rows=rows), O.attention(q, k, v)[rows])


# ----------------------------------------------------------------------------- LayerNorm
def test_layer_norm_closed_form():
    eps = 1e-6
    out = O.layer_norm(np.array([[1.0, 3.0]]), eps)
    s = 1 / math.sqrt(1 + eps)          # mean 2, biased variance 1
    assert np.allclose(out, [[-s, s]], rtol=0, atol=1e-15)
    const = O.layer_norm(np.full((1, 8), 4.25), eps)
    assert np.array_equal(const, np.zeros((1, 8)))


def test_layer_norm_vs_torch_and_moments():
    x = RNG.standard_normal((6, 96)) * 3 + 1.5
    eps = 1e-6
    out = O.layer_norm(x, eps)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (96,), eps=eps).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12
    var = x.var(axis=1)
    assert np.allclose(out.mean(axis=1), 0, atol=1e-13)
    assert np.allclose(out.var(axis=1), var / (var + eps), rtol=1e-12)


def test_modulate_special_cases():
    xn = RNG.standard_normal((4, 10))
    assert np.array_equal(O.modulate(xn, np.zeros(10), np.zeros(10)), xn)
    shift = RNG.standard_normal(10)
    assert np.array_equal(O.modulate(xn, shift, -np.ones(10)), np.broadcast_to(shift, xn.shape))
    scale = RNG.standard_normal(10)
    assert np.allclose(O.modulate(xn, shift, scale), xn + xn * scale + shift, atol=1e-14)


# ----------------------------------------------------------------------------- RoPE
def test_rope_closed_form_unit_vectors():
    # hd 8 split (t 2, h 2, w 4), theta 100, position (t, h, w) = (1, 2, 3):
    # pair (0,1): angle 1; pair (2,3): angle 2; pair (4,5): angle 3;
    # pair (6,7): k = 1 of a width-4 chunk -> freq 100^(-2/4) = 0.1 -> angle 0.3
    pos = np.array([[1.0, 2.0, 3.0]])
    e_even = np.array([1, 0, 1, 0, 1, 0, 1, 0], float).reshape(1, 1, 8)
    e_odd = np.array([0, 1, 0, 1, 0, 1, 0, 1], float).reshape(1, 1, 8)
    ang = [1.0, 2.0, 3.0, 0.3]
    got = O.rope_rotate(e_even, pos, (2, 2, 4), 100.0).ravel()
    want = np.ravel([[math.cos(a), math.sin(a)] for a in ang])
    assert np.allclose(got, want, atol=1e-15)
    got = O.rope_rotate(e_odd, pos, (2, 2, 4), 100.0).ravel()
    want = np.ravel([[-math.sin(a), math.cos(a)] for a in ang])
    assert np.allclose(got, want, atol=1e-15)


def test_rope_matches_complex_formulation():
    # independent formulation: adjacent pairs as complex numbers times exp(i angle)
    n, h, split, theta = 11, 3, (16, 24, 24), 10000.0
    hd = sum(split)
    x = RNG.standard_normal((n, h, hd))
    pos = RNG.uniform(-5, 40, (n, 3))
    z = x[..., 0::2] + 1j * x[..., 1::2]
    angles = []
    for axis, width in enumerate(split):
        k = np.arange(width // 2)
        angles.append(pos[:, axis:axis + 1] * theta ** (-2.0 * k / width)[None, :])
    rot = np.exp(1j * np.concatenate(angles, axis=1))[:, None, :]
    zr = z * rot
    want = np.empty_like(x)
    want[..., 0::2] = zr.real
    want[..., 1::2] = zr.imag
    assert np.max(np.abs(O.rope_rotate(x, pos, split, theta) - want)) < 1e-12


def test_rope_norm_and_relative_position():
    n, h, split = 9, 2, (32, 48, 48)
    q = RNG.standard_normal((n, h, 128))
    k = RNG.standard_normal((n, h, 128))
    pos = RNG.integers(0, 20, (n, 3)).astype(float)
    rq = O.rope_rotate(q, pos, split, 1e4)
    pair_norm = lambda a: a[..., 0::2] ** 2 + a[..., 1::2] ** 2
    assert np.allclose(pair_norm(rq), pair_norm(q), rtol=1e-12)
    shift = np.array([5.0, -3.0, 7.0])
    s0 = np.einsum("ihc,jhc->hij", rq, O.rope_rotate(k, pos, split, 1e4))
    s1 = np.einsum("ihc,jhc->hij", O.rope_rotate(q, pos + shift, split, 1e4),
                   O.rope_rotate(k, pos + shift, split, 1e4))
    assert np.allclose(s0, s1, atol=1e-10)


def test_rope_positions_layout():
    pos = O.rope_positions((2, 2, 4), n_audio=3)
    assert pos.shape == (19, 3)
    assert pos[0].tolist() == [0, 0, 0] and pos[1].tolist() == [0, 0, 1]
    assert pos[4].tolist() == [0, 1, 0] and pos[8].tolist() == [1, 0, 0]
    assert pos[15].tolist() == [1, 1, 3]
    assert np.array_equal(pos[16:], np.zeros((3, 3)))
    pr = O.rope_positions((2, 2, 4), n_audio=3, paired=True)
    assert pr.shape == (11, 3)
    assert pr[0].tolist() == [0, 0, 0.5] and pr[1].tolist() == [0, 0, 2.5]
    assert pr[3].tolist() == [0, 1, 2.5]
    ph = O.rope_positions((2, 2, 4), n_audio=0, halved=True)
    assert ph[15].tolist() == [1, 0.5, 1.5]
    # halved and paired: the merged token's w is the mean of its sources' halved w
    php = O.rope_positions((2, 2, 4), n_audio=1, halved=True, paired=True)
    assert php.shape == (9, 3)
    assert php[0].tolist() == [0, 0, 0.25] and php[7].tolist() == [1, 0.5, 1.25]
    assert php[8].tolist() == [0, 0, 0]
    # audio tokens are left unrotated
    x = RNG.standard_normal((19, 1, 8))
    out = O.rope_rotate(x, pos, (2, 2, 4), 10.0)
    assert np.array_equal(out[16:], x[16:])


# ----------------------------------------------------------------------------- GELU
def test_gelu_vs_torch_and_identities():
    x = np.linspace(-8, 8, 2001)
    g = O.gelu_tanh(x)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.max(np.abs(g - ref)) < 1e-14
    erf = torch.nn.functional.gelu(torch.from_numpy(x)).numpy()
    assert np.max(np.abs(g - erf)) < 1e-3          # tanh form approximates the erf form
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert np.allclose(g - O.gelu_tanh(-x), x, atol=1e-14)   # odd part is x / 2


# ----------------------------------------------------------------------------- block
def _tiny_block(seed=0, d=64, heads=2, f=256, c=16):
    r = np.random.default_rng(seed)
    w = {"w_qkv": r.standard_normal((3 * d, d)) * 0.05, "b_qkv": r.standard_normal(3 * d) * 0.05,
         "w_o": r.standard_normal((d, d)) * 0.05, "b_o": r.standard_normal(d) * 0.05,
         "w_fc1": r.standard_normal((f, d)) * 0.05, "b_fc1": r.standard_normal(f) * 0.05,
         "w_fc2": r.standard_normal((d, f)) * 0.05, "b_fc2": r.standard_normal(d) * 0.05}
    mod = r.standard_normal((6, d)) * 0.3
    return w, mod


def test_block_zero_gate_is_identity():
    w, mod = _tiny_block()
    mod[2] = 0
    mod[5] = 0
    grid = (2, 2, 4)
    x = RNG.standard_normal((16 + 3, 64))
    pos = O.rope_positions(grid, 3)
    out, _ = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6)
    assert np.array_equal(out, x)


def test_block_zero_weights():
    w, mod = _tiny_block()
    w = {k: np.zeros_like(v) for k, v in w.items()}
    x = RNG.standard_normal((10, 64))
    pos = O.rope_positions((1, 2, 5), 0)
    out, hn = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6, mod_next=mod)
    assert np.array_equal(out, x)
    assert np.allclose(hn, O.modulate(O.layer_norm(x, 1e-6), mod[0], mod[1]), atol=0)


def _torch_block(x, w, mod, pos, heads, split, theta, eps):
    """Independent composition of the block from torch library routines (layer_norm,
    scaled_dot_product_attention, gelu) and a complex-number RoPE."""
    F = torch.nn.functional
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    x = t(x)
    m = t(mod)
    n, d = x.shape
    hd = d // heads
    h = F.layer_norm(x, (d,), eps=eps) * (1 + m[1]) + m[0]
    qkv = F.linear(h, t(w["w_qkv"]), t(w["b_qkv"]))
    q, k, v = (qkv[:, i * d:(i + 1) * d].reshape(n, heads, hd) for i in range(3))
    ang = []
    for axis, width in enumerate(split):
        kk = torch.arange(width // 2, dtype=torch.float64)
        ang.append(t(pos)[:, axis:axis + 1] * theta ** (-2.0 * kk / width))
    rot = torch.polar(torch.ones(n, hd // 2, dtype=torch.float64), torch.cat(ang, 1))[:, None]

    def rope(a):
        z = torch.view_as_complex(a.reshape(n, heads, hd // 2, 2).contiguous())
        return torch.view_as_real(z * rot).reshape(n, heads, hd)

    o = F.scaled_dot_product_attention(rope(q).transpose(0, 1), rope(k).transpose(0, 1),
                                       v.transpose(0, 1)).transpose(0, 1).reshape(n, d)
    x1 = x + m[2] * F.linear(o, t(w["w_o"]), t(w["b_o"]))
    h2 = F.layer_norm(x1, (d,), eps=eps) * (1 + m[4]) + m[3]
    g = F.gelu(F.linear(h2, t(w["w_fc1"]), t(w["b_fc1"])), approximate="tanh")
    return (x1 + m[5] * F.linear(g, t(w["w_fc2"]), t(w["b_fc2"]))).numpy()


def test_block_vs_torch_composition():
    w, mod = _tiny_block(seed=3)
    grid = (2, 3, 4)
    x = RNG.standard_normal((24 + 5, 64))
    pos = O.rope_positions(grid, 5)
    out, _ = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6)
    ref = _torch_block(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_block_rows_subset_and_permutation_equivariance():
    w, mod = _tiny_block(seed=5)
    grid = (2, 2, 4)
    x = RNG.standard_normal((16 + 4, 64))
    pos = O.rope_positions(grid, 4)
    full, _ = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6)
    rows = np.array([1, 6, 17])
    sub, _ = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6, rows=rows)
    assert np.allclose(sub, full[rows], atol=1e-13)
    perm = RNG.permutation(len(x))
    outp, _ = O.block_forward(x[perm], w, mod, pos[perm], 2, (8, 12, 12), 1e4, 1e-6)
    assert np.allclose(outp, full[perm], atol=1e-12)


def test_modulation_vectors():
    r = np.random.default_rng(9)
    w = r.standard_normal((6 * 8, 5))
    b = r.standard_normal(6 * 8)
    c = r.standard_normal(5)
    mod = O.adaln_modulation(w, b, c, 8)
    assert mod.shape == (6, 8)
    # row j of mod[i] is a dot product of weight row i*8+j
    assert abs(mod[4, 3] - (sum(w[35, k] * c[k] for k in range(5)) + b[35])) < 1e-12
    wf = r.standard_normal((2, 16, 5))
    bf = r.standard_normal((2, 16))
    fm = O.final_modulation(wf, bf, c, 8)
    assert fm.shape == (2, 2, 8)
    assert abs(fm[1, 1, 2] - (wf[1, 10] @ c + bf[1, 10])) < 1e-12


# ----------------------------------------------------------------------------- Euler
def test_sigma_grid_and_euler():
    assert O.sigma_grid(4).tolist() == [1.0, 0.75, 0.5, 0.25, 0.0]
    assert O.sigma_grid(1).tolist() == [1.0, 0.0]
    x = RNG.standard_normal((3, 4))
    v = RNG.standard_normal((3, 4))
    assert np.array_equal(O.euler_update(x, v, 0.5, 0.5), x)
    assert np.array_equal(O.euler_update(x, v, 1.0, 0.75), x - 0.25 * v)


def test_final_adaln_streams():
    x = RNG.standard_normal((7, 6))
    fm = RNG.standard_normal((2, 2, 6))
    v = O.final_adaln(x, fm, 4, 1e-6)
    xn = O.layer_norm(x, 1e-6)
    assert np.allclose(v[:4], xn[:4] * (1 + fm[0, 1]) + fm[0, 0], atol=1e-15)
    assert np.allclose(v[4:], xn[4:] * (1 + fm[1, 1]) + fm[1, 0], atol=1e-15)


# ----------------------------------------------------------------------------- pairing
def test_token_pair_bruteforce_and_identities():
    grid, na, d = (2, 3, 4), 2, 5
    x = RNG.standard_normal((24 + na, d))
    red = O.token_pair(x, grid, na)
    assert red.shape == (12 + na, d)
    for t in range(2):
        for h in range(3):
            for j in range(2):
                src = (t * 3 + h) * 4 + 2 * j
                dst = (t * 3 + h) * 2 + j
                assert np.allclose(red[dst], 0.5 * (x[src] + x[src + 1]), atol=0)
    assert np.array_equal(red[12:], x[24:])
    # duplicating then pairing is the identity; bypass restore of an unchanged stream too
    dup = O.token_unpair(red, grid, na)
    assert np.array_equal(O.token_pair(dup, grid, na), red)
    assert np.array_equal(dup[1], red[0]) and np.array_equal(dup[0], red[0])
    assert np.array_equal(O.token_unpair(red, grid, na, saved=x), x)
    # bypass adds the reduced update to both source tokens
    upd = RNG.standard_normal(red.shape)
    back = O.token_unpair(red + upd, grid, na, saved=x)
    assert np.allclose(back[2], x[2] + upd[1], atol=1e-14)
    assert np.allclose(back[3], x[3] + upd[1], atol=1e-14)
    assert np.allclose(back[24:], red[12:] + upd[12:], atol=0)


# ----------------------------------------------------------------------------- thinning
def test_layer_mask_policy():
    nb, d = 8, 4
    mods = np.zeros((nb, 6, d))
    score = [9, 1, 5, 0.5, 7, 1, 6, 0.1]
    for b, s in enumerate(score):
        mods[b, 2] = s / 2
        mods[b, 5] = -s / 2
    keep = O.layer_mask(mods, 6)
    # interior scores: b1=1, b2=5, b3=0.5, b4=7, b5=1, b6=6 -> drop b3 then the tie b1/b5 -> b5
    assert keep.tolist() == [True, True, True, False, True, False, True, True]
    assert O.layer_mask(mods, 8).all()


# ----------------------------------------------------------------------------- int8
def test_quantize_rows_rules():
    a = np.array([[0.5, -1.0, 0.25, 0.0], [0, 0, 0, 0], [3.0, 1.0, -2.9, 1.5]], np.float32)
    q, s = O.quantize_rows(a)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert q[0].tolist() == [64, -127, 32, 0]        # 63.5 rounds half to even -> 64; 31.75 -> 32
    assert q[1].tolist() == [0, 0, 0, 0] and s[1] == 0
    assert q[2, 0] == 127 and s[2] == np.float32(3.0) / np.float32(127)
    big = (RNG.standard_normal((50, 300)) * 3).astype(np.float32)
    q, s = O.quantize_rows(big)
    assert np.all(np.abs(q.astype(int)) <= 127)
    assert np.all(np.max(np.abs(q.astype(int)), axis=1) == 127)
    err = np.abs(big - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None] * 0.5 + 1e-6 * np.abs(big))


def test_int_matmul_exact():
    qa = RNG.integers(-127, 128, (3, 7)).astype(np.int8)
    qb = RNG.integers(-127, 128, (2, 7)).astype(np.int8)
    acc = O.int_matmul(qa, qb)
    for m in range(3):
        for n in range(2):
            assert acc[m, n] == sum(int(qa[m, k]) * int(qb[n, k]) for k in range(7))
    # full FC2 depth with extreme values: exact against numpy's integer dot
    K = 12288
    qa = RNG.choice([-127, 127, -126, 125], (2, K)).astype(np.int8)
    qb = RNG.choice([-127, 127], (3, K)).astype(np.int8)
    ref = qa.astype(np.int64) @ qb.astype(np.int64).T
    assert np.array_equal(O.int_matmul(qa, qb), ref)


def test_fc2_int8_row_composition():
    act = (RNG.standard_normal((4, 64))).astype(np.float32)
    w = (RNG.standard_normal((5, 64)) * 0.02).astype(np.float32)
    wq, ws = O.quantize_rows(w)
    gate = RNG.standard_normal(5)
    resid = RNG.standard_normal((4, 5))
    q, s, acc, out = O.fc2_int8_row(act, wq, ws, gate, resid)
    m, n = 2, 3
    acc_ref = sum(int(q[m, k]) * int(wq[n, k]) for k in range(64))
    assert acc[m, n] == acc_ref
    assert abs(out[m, n] - (resid[m, n] + gate[n] * acc_ref * float(s[m]) * float(ws[n]))) < 1e-12
    # the dequantised product approximates the float product
    assert rel_l2(out - resid, gate * (act.astype(float) @ w.astype(float).T)) < 2e-2


# ----------------------------------------------------------------------------- misc
def test_round_to_bf16_matches_torch():
    x = np.concatenate([RNG.standard_normal(1000) * 10 ** RNG.uniform(-6, 6, 1000),
                        [0.0, -0.0, 1.0, 65504.0, 1e-40]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(O.round_to_bf16(x), ref)


def test_fp32_matches_fp64_on_tiny_block():
    w, mod = _tiny_block(seed=7)
    x = RNG.standard_normal((19, 64))
    pos = O.rope_positions((1, 4, 4), 3)
    a, _ = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6, dt=np.float64)
    b, _ = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6, dt=np.float32)
    assert rel_l2(b, a) < 1e-5


def test_denoise_update_with_constant_velocity():
    # final scale -1 makes v = shift for every token: the trajectory is then closed form
    w, mod = _tiny_block(seed=11)
    grid, na = (1, 2, 4), 2
    x0 = RNG.standard_normal((8 + na, 64))
    fm = np.zeros((2, 2, 64))
    fm[:, 1] = -1
    fm[0, 0] = 0.5
    fm[1, 0] = -2.0
    out = O.denoise(x0, [w], mod[None], fm, grid, na, 2, (8, 12, 12), 1e4, 1e-6,
                    steps=4, run_steps=4)
    want = x0.copy()
    want[:8] -= 0.5
    want[8:] += 2.0
    assert np.allclose(out, want, atol=1e-12)


# ----------------------------------------------------------------------------- denoise loop
# The Euler loop with token reduction composed independently of oracle.denoise: torch
# average pooling for the pairing (positions pooled the same way as the tokens, so the
# merged token's position is the mean of its sources), repeat_interleave for the bypass
# restore, torch layer_norm for the final AdaLN, and _torch_block for every block.
F = torch.nn.functional


def _grid_positions(grid, n_audio, halved):
    t_n, h_n, w_n = grid
    vid = torch.cartesian_prod(torch.arange(t_n, dtype=torch.float64),
                               torch.arange(h_n, dtype=torch.float64),
                               torch.arange(w_n, dtype=torch.float64))
    if halved:
        vid[:, 1:] *= 0.5
    return torch.cat([vid, torch.zeros((n_audio, 3), dtype=torch.float64)])


def _pool_w(x, grid):
    """Width-2 average pool over the w axis of the video rows of x [N, c]."""
    t_n, h_n, w_n = grid
    nv = t_n * h_n * w_n
    vid = x[:nv].reshape(t_n * h_n, w_n, -1).transpose(1, 2)            # [t h, c, w]
    return F.avg_pool1d(vid, 2).transpose(1, 2).reshape(nv // 2, -1)


def _torch_pair(x, grid, n_audio):
    nv = grid[0] * grid[1] * grid[2]
    return torch.cat([_pool_w(x, grid), x[nv:nv + n_audio]])


def _torch_unpair(x_red, grid, n_audio, saved):
    nv = grid[0] * grid[1] * grid[2]
    red = x_red[:nv // 2]
    if saved is None:
        vid = red.repeat_interleave(2, dim=0)
    else:
        vid = saved[:nv] + (red - _pool_w(saved, grid)).repeat_interleave(2, dim=0)
    return torch.cat([vid, x_red[nv // 2:nv // 2 + n_audio]])


def _torch_denoise(x0, blocks, mods, fm, grid, n_audio, heads, split, theta, eps, steps,
                   active=None, reduce_after=-1, halved=False, bypass=True):
    x_state = torch.from_numpy(np.asarray(x0, np.float64))
    fm = torch.from_numpy(np.asarray(fm, np.float64))
    nv = grid[0] * grid[1] * grid[2]
    pos_full = _grid_positions(grid, n_audio, halved)
    pos_red = torch.cat([_pool_w(pos_full, grid), pos_full[nv:]])
    order = [b for b in range(len(blocks)) if active is None or active[b]]
    for i in range(steps):
        s, s_next = 1.0 - i / steps, 1.0 - (i + 1) / steps
        x = x_state.to(torch.bfloat16).to(torch.float64)
        saved, pos = None, pos_full
        for k, b in enumerate(order):
            x = torch.from_numpy(_torch_block(x.numpy(), blocks[b], mods[b], pos.numpy(),
                                              heads, split, theta, eps))
            if k + 1 == reduce_after and k + 1 < len(order):
                saved, x, pos = x, _torch_pair(x, grid, n_audio), pos_red
        if saved is not None:
            x = _torch_unpair(x, grid, n_audio, saved if bypass else None)
        xn = F.layer_norm(x, (x.shape[1],), eps=eps)
        v = torch.cat([xn[:nv] * (1 + fm[0, 1]) + fm[0, 0], xn[nv:] * (1 + fm[1, 1]) + fm[1, 0]])
        x_state = x_state + (s_next - s) * v
    return x_state.numpy()


def _denoise_case(n_blocks=4, seed=21):
    blocks, mods = [], []
    for b in range(n_blocks):
        w, mod = _tiny_block(seed=seed + b)
        blocks.append(w)
        mods.append(mod)
    r = np.random.default_rng(seed + 100)
    fm = r.standard_normal((2, 2, 64)) * 0.3
    grid, na = (2, 2, 4), 3
    x0 = O.round_to_bf16(r.standard_normal((16 + na, 64))).astype(np.float64)
    return blocks, np.stack(mods), fm, grid, na, x0


_DENOISE_ARGS = dict(heads=2, split=(8, 12, 12), theta=1e4, eps=1e-6)


@pytest.mark.parametrize("reduce_after,active,halved,bypass", [
    (2, None, False, True), (1, [1, 1, 0, 1], False, True), (2, [1, 0, 1, 1], True, True),
    (3, None, False, False), (-1, [1, 1, 0, 1], True, True)])
def test_denoise_matches_independent_torch_composition(reduce_after, active, halved, bypass):
    blocks, mods, fm, grid, na, x0 = _denoise_case()
    a = _DENOISE_ARGS
    want = _torch_denoise(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"],
                          a["eps"], 2, active, reduce_after, halved, bypass)
    got = O.denoise(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"],
                    a["eps"], steps=2, run_steps=2, active=active, reduce_after=reduce_after,
                    halved=halved, unpair_bypass=bypass)
    assert np.max(np.abs(got - want)) < 1e-10


def _oracle_denoise_2(blocks, mods, fm, grid, na, x0, **kw):
    a = _DENOISE_ARGS
    return O.denoise(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"],
                     a["eps"], steps=2, run_steps=2, **kw)


def test_denoise_with_identity_reduced_blocks_equals_the_unreduced_prefix():
    # blocks after the pairing with zero gates are identities, so the bypass restore gets
    # back exactly the stream saved at the pairing: the trajectory is that of the first
    # reduce_after blocks alone, without any reduction
    blocks, mods, fm, grid, na, x0 = _denoise_case()
    mods = mods.copy()
    mods[2:, 2] = 0
    mods[2:, 5] = 0
    got = _oracle_denoise_2(blocks, mods, fm, grid, na, x0, reduce_after=2)
    want = _oracle_denoise_2(blocks[:2], mods[:2], fm, grid, na, x0)
    assert np.max(np.abs(got - want)) < 1e-12
    # the duplicate restore instead gives each video token its pair's mean
    got_dup = _oracle_denoise_2(blocks, mods, fm, grid, na, x0, reduce_after=2,
                                unpair_bypass=False)
    assert np.max(np.abs(got_dup - want)) > 1e-3


def test_denoise_duplicate_restore_closed_form_one_step():
    # one step, identity blocks after the pairing, duplicate restore: the final AdaLN sees
    # each video token replaced by the mean of its horizontal pair (audio untouched)
    blocks, mods, fm, grid, na, x0 = _denoise_case()
    mods = mods.copy()
    mods[1:, 2] = 0
    mods[1:, 5] = 0
    a = _DENOISE_ARGS
    got = O.denoise(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"],
                    a["eps"], steps=4, run_steps=1, reduce_after=1, unpair_bypass=False)
    pos = O.rope_positions(grid, na)
    x = O.round_to_bf16(x0).astype(np.float64)
    x1, _ = O.block_forward(x, blocks[0], mods[0], pos, a["heads"], a["split"], a["theta"],
                            a["eps"])
    dup = x1.copy()
    dup[0:16:2] = dup[1:16:2] = 0.5 * (x1[0:16:2] + x1[1:16:2])
    v = O.final_adaln(dup, fm, 16, a["eps"])
    assert np.max(np.abs(got - (x0 - 0.25 * v))) < 1e-12


@pytest.mark.parametrize("mistake", ["pair_late", "full_positions", "unpair_saved_early",
                                     "final_on_reduced"])
def test_denoise_comparison_catches_planted_mistakes(mistake, monkeypatch):
    # each plausible slip in the orchestration, planted in the oracle, makes the
    # comparison with the independent composition fail
    blocks, mods, fm, grid, na, x0 = _denoise_case()
    a = _DENOISE_ARGS
    want = _torch_denoise(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"],
                          a["eps"], 2, None, 2)
    kw = dict(reduce_after=2)
    if mistake == "pair_late":
        kw["reduce_after"] = 3
    elif mistake == "full_positions":
        real = O.rope_positions
        monkeypatch.setattr(O, "rope_positions",
                            lambda g, n, halved=False, paired=False, dt=np.float64:
                            real(g, n, halved, False, dt)
                            if not paired else
                            real(g, n, halved, False, dt)[np.r_[0:16:2, 16:16 + n]])
    elif mistake == "unpair_saved_early":
        real_pair = O.token_pair
        first = {}

        def pair_and_keep(x, g, n, dt=np.float64):
            first.setdefault("x", x)
            return real_pair(x, g, n, dt)
        real_unpair = O.token_unpair
        monkeypatch.setattr(O, "token_pair", pair_and_keep)
        monkeypatch.setattr(O, "token_unpair",
                            lambda xr, g, n, saved=None, dt=np.float64:
                            real_unpair(xr, g, n, first["x"] * 0.5 + saved * 0.5, dt))
    elif mistake == "final_on_reduced":
        real_unpair = O.token_unpair
        monkeypatch.setattr(O, "token_unpair",
                            lambda xr, g, n, saved=None, dt=np.float64:
                            real_unpair(xr, g, n, None, dt))
    got = _oracle_denoise_2(blocks, mods, fm, grid, na, x0, **kw)
    assert np.max(np.abs(got - want)) > 1e-4


# ----------------------------------------------------------------------------- reuse policies
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_reuse_schedule_matches_the_pages_counts():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "reuse_counts.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for steps, reuse, fresh in rows:
        assert int(O.reuse_schedule(int(steps), int(reuse)).sum()) == int(fresh)
    s = O.reuse_schedule(7, 3)
    assert s.tolist() == [True, False, False, True, False, False, True]
    assert O.reuse_schedule(5, 1).all()


def _torch_denoise_reuse(x0, blocks, mods, fm, grid, n_audio, steps, reuse, mode):
    """Independent composition of the two reuse loops from _torch_block and torch ops."""
    a = _DENOISE_ARGS
    nv = grid[0] * grid[1] * grid[2]
    pos = _grid_positions(grid, n_audio, False).numpy()
    fmt = torch.from_numpy(np.asarray(fm, np.float64))
    x_state = torch.from_numpy(np.asarray(x0, np.float64))
    held = None
    for i in range(steps):
        fresh = i % reuse == 0 or i == steps - 1
        x_in = x_state.to(torch.bfloat16).to(torch.float64)
        if fresh:
            x = x_in
            for b in range(len(blocks)):
                x = torch.from_numpy(_torch_block(x.numpy(), blocks[b], mods[b], pos,
                                                  a["heads"], a["split"], a["theta"], a["eps"]))
            x_l = x
            if mode == "core":
                held = x_l - x_in
        elif mode == "core":
            x_l = (x_in + held).to(torch.bfloat16).to(torch.float64)
        if fresh or mode == "core":
            xn = F.layer_norm(x_l, (x_l.shape[1],), eps=a["eps"])
            v = torch.cat([xn[:nv] * (1 + fmt[0, 1]) + fmt[0, 0],
                           xn[nv:] * (1 + fmt[1, 1]) + fmt[1, 0]])
            if mode == "velocity":
                held = v
        else:
            v = held
        x_state = x_state + ((1.0 - (i + 1) / steps) - (1.0 - i / steps)) * v
    return x_state.numpy()


@pytest.mark.parametrize("mode", ["velocity", "core"])
@pytest.mark.parametrize("steps,reuse", [(5, 2), (7, 3), (4, 1)])
def test_reuse_loops_match_independent_composition(mode, steps, reuse):
    blocks, mods, fm, grid, na, x0 = _denoise_case(n_blocks=2)
    a = _DENOISE_ARGS
    fn = O.denoise_velocity_reuse if mode == "velocity" else O.denoise_core_reuse
    got = fn(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"], a["eps"],
             steps, reuse)
    want = _torch_denoise_reuse(x0, blocks, mods, fm, grid, na, steps, reuse, mode)
    assert np.max(np.abs(got - want)) < 1e-10


@pytest.mark.parametrize("mode", ["velocity", "core"])
def test_reuse_one_is_the_plain_loop(mode):
    blocks, mods, fm, grid, na, x0 = _denoise_case(n_blocks=3)
    a = _DENOISE_ARGS
    fn = O.denoise_velocity_reuse if mode == "velocity" else O.denoise_core_reuse
    kw = dict(active=[1, 0, 1], reduce_after=1)
    got = fn(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"], a["eps"],
             4, 1, **kw)
    want = O.denoise(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"],
                     a["eps"], steps=4, run_steps=4, **kw)
    assert np.array_equal(got, want)


def test_reuse_closed_forms():
    blocks, mods, fm, grid, na, x0 = _denoise_case(n_blocks=2)
    a = _DENOISE_ARGS
    args = (grid, na, a["heads"], a["split"], a["theta"], a["eps"])
    # constant velocity (final scale -1): every policy follows the same trajectory
    fc = np.zeros_like(fm)
    fc[:, 1] = -1
    fc[0, 0], fc[1, 0] = 0.7, -0.4
    base = O.denoise(x0, blocks, mods, fc, *args, steps=6, run_steps=6)
    for fn in (O.denoise_velocity_reuse, O.denoise_core_reuse):
        assert np.allclose(fn(x0, blocks, mods, fc, *args, 6, 3), base, atol=1e-12)
    # identity core (zero gates): the core residual is zero, so core reuse is exact
    mz = mods.copy()
    mz[:, 2] = 0
    mz[:, 5] = 0
    full = O.denoise(x0, blocks, mz, fm, *args, steps=6, run_steps=6)
    assert np.array_equal(O.denoise_core_reuse(x0, blocks, mz, fm, *args, 6, 4), full)
    # ... while velocity reuse holds a stale velocity and departs from it
    assert np.max(np.abs(O.denoise_velocity_reuse(x0, blocks, mz, fm, *args, 6, 4) - full)) > 1e-3


# ----------------------------------------------------------------------------- Q/K RMSNorm
def test_rms_norm_closed_form_and_torch():
    out = O.rms_norm(np.array([[3.0, 4.0]]), np.ones(2), 0.0)
    r = math.sqrt(12.5)
    assert np.allclose(out, [[3 / r, 4 / r]], atol=1e-15)
    x = RNG.standard_normal((7, 3, 128)) * 2.5
    g = 1 + RNG.standard_normal(128) * 0.1
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (128,), torch.from_numpy(g),
                                       eps=1e-6).numpy()
    assert np.max(np.abs(O.rms_norm(x, g, 1e-6) - ref)) < 1e-13
    # scale invariance and unit mean square with unit gains
    assert np.allclose(O.rms_norm(5.0 * x, g, 0.0), O.rms_norm(x, g, 0.0), atol=1e-13)
    y = O.rms_norm(x, np.ones(128), 0.0)
    assert np.allclose((y * y).mean(axis=-1), 1.0, atol=1e-13)


def _torch_block_qk(x, w, mod, pos, heads, split, theta, eps):
    """_torch_block with torch's rms_norm on each head of q and k before the rotation."""
    F_ = torch.nn.functional
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    xt, m = t(x), t(mod)
    n, d = xt.shape
    hd = d // heads
    h = F_.layer_norm(xt, (d,), eps=eps) * (1 + m[1]) + m[0]
    qkv = F_.linear(h, t(w["w_qkv"]), t(w["b_qkv"]))
    q, k, v = (qkv[:, i * d:(i + 1) * d].reshape(n, heads, hd) for i in range(3))
    q = F_.rms_norm(q, (hd,), t(w["q_norm"]), eps=eps)
    k = F_.rms_norm(k, (hd,), t(w["k_norm"]), eps=eps)
    ang = []
    for axis, width in enumerate(split):
        kk = torch.arange(width // 2, dtype=torch.float64)
        ang.append(t(pos)[:, axis:axis + 1] * theta ** (-2.0 * kk / width))
    rot = torch.polar(torch.ones(n, hd // 2, dtype=torch.float64), torch.cat(ang, 1))[:, None]

    def rope(a):
        z = torch.view_as_complex(a.reshape(n, heads, hd // 2, 2).contiguous())
        return torch.view_as_real(z * rot).reshape(n, heads, hd)

    o = F_.scaled_dot_product_attention(rope(q).transpose(0, 1), rope(k).transpose(0, 1),
                                        v.transpose(0, 1)).transpose(0, 1).reshape(n, d)
    x1 = xt + m[2] * F_.linear(o, t(w["w_o"]), t(w["b_o"]))
    h2 = F_.layer_norm(x1, (d,), eps=eps) * (1 + m[4]) + m[3]
    g = F_.gelu(F_.linear(h2, t(w["w_fc1"]), t(w["b_fc1"])), approximate="tanh")
    return (x1 + m[5] * F_.linear(g, t(w["w_fc2"]), t(w["b_fc2"]))).numpy()


def test_block_with_qk_norm_vs_torch_composition():
    w, mod = _tiny_block(seed=31)
    r = np.random.default_rng(32)
    w["q_norm"] = 1 + r.standard_normal(32) * 0.1
    w["k_norm"] = 1 + r.standard_normal(32) * 0.1
    grid = (2, 3, 4)
    x = RNG.standard_normal((24 + 5, 64))
    pos = O.rope_positions(grid, 5)
    out, _ = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6)
    ref = _torch_block_qk(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6)
    assert np.max(np.abs(out - ref)) < 1e-12
    # the norm matters: without it the block differs
    w0 = {k: v for k, v in w.items() if k not in ("q_norm", "k_norm")}
    plain, _ = O.block_forward(x, w0, mod, pos, 2, (8, 12, 12), 1e4, 1e-6)
    assert np.max(np.abs(plain - out)) > 1e-3


# ----------------------------------------------------------------------------- patch / heads
def test_patch_embed_and_head_per_stream_vs_torch():
    r = np.random.default_rng(41)
    n, nv, C, d = 11, 7, 16, 24
    lat = O.round_to_bf16(r.standard_normal((n, C))).astype(np.float64)
    wp, bp = r.standard_normal((2, d, C)), r.standard_normal((2, d))
    x = O.patch_embed(lat, nv, wp, bp)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    want = torch.cat([F.linear(t(lat[:nv]), t(wp[0]), t(bp[0])),
                      F.linear(t(lat[nv:]), t(wp[1]), t(bp[1]))]).numpy()
    assert np.max(np.abs(x - want)) < 1e-12
    fm = r.standard_normal((2, 2, d)) * 0.3
    wh, bh = r.standard_normal((2, C, d)), r.standard_normal((2, C))
    v = O.final_head(x, fm, nv, 1e-6, wh, bh)
    xn = F.layer_norm(t(x), (d,), eps=1e-6)
    hv = xn[:nv] * (1 + t(fm[0, 1])) + t(fm[0, 0])
    ha = xn[nv:] * (1 + t(fm[1, 1])) + t(fm[1, 0])
    want = torch.cat([F.linear(hv, t(wh[0]), t(bh[0])), F.linear(ha, t(wh[1]), t(bh[1]))])
    assert np.max(np.abs(v - want.numpy())) < 1e-12


def test_latent_loop_with_identity_patch_and_head_is_the_model_space_loop():
    blocks, mods, fm, grid, na, x0 = _denoise_case(n_blocks=3)
    a = _DENOISE_ARGS
    d = x0.shape[1]
    eye = np.stack([np.eye(d)] * 2)
    heads = {"w_patch": eye, "b_patch": np.zeros((2, d)), "w_head": eye,
             "b_head": np.zeros((2, d))}
    kw = dict(active=[1, 0, 1], reduce_after=1)
    got = O.denoise_latent(x0, blocks, mods, fm, heads, grid, na, a["heads"], a["split"],
                           a["theta"], a["eps"], 4, 4, **kw)
    want = O.denoise(x0, blocks, mods, fm, grid, na, a["heads"], a["split"], a["theta"],
                     a["eps"], steps=4, run_steps=4, **kw)
    assert np.array_equal(got, want)


def test_latent_loop_constant_head_closed_form():
    # final scale -1: the head sees shift_s on every row, so each step adds
    # (s' - s)(W_s shift_s + b_s) to the latent whatever the blocks do
    blocks, mods, fm, grid, na, x0 = _denoise_case(n_blocks=2)
    a = _DENOISE_ARGS
    r = np.random.default_rng(43)
    d, C, n, nv = 64, 8, x0.shape[0], 16
    fc = np.zeros((2, 2, d))
    fc[:, 1] = -1
    fc[:, 0] = r.standard_normal((2, d))
    heads = {"w_patch": r.standard_normal((2, d, C)) * 0.1, "b_patch": r.standard_normal((2, d)),
             "w_head": r.standard_normal((2, C, d)) * 0.1, "b_head": r.standard_normal((2, C))}
    lat0 = r.standard_normal((n, C))
    got = O.denoise_latent(lat0, blocks, mods, fc, heads, grid, na, a["heads"], a["split"],
                           a["theta"], a["eps"], 4, 3)
    vv = heads["w_head"][0] @ fc[0, 0] + heads["b_head"][0]
    va = heads["w_head"][1] @ fc[1, 0] + heads["b_head"][1]
    want = lat0.copy()
    want[:nv] += -0.75 * vv
    want[nv:] += -0.75 * va
    assert np.allclose(got, want, atol=1e-12)


# ----------------------------------------------------------------------------- grouped int8
def test_quantize_groups_is_rows_per_group():
    a = (RNG.standard_normal((5, 12)) * [1, 1, 1, 1, 10, 10, 10, 10, 0, 0, 0, 0]).astype(np.float32)
    q, s = O.quantize_groups(a, 4)
    assert q.shape == (5, 12) and s.shape == (5, 3)
    for g in range(3):
        qg, sg = O.quantize_rows(a[:, 4 * g:4 * g + 4])
        assert np.array_equal(q[:, 4 * g:4 * g + 4], qg) and np.array_equal(s[:, g], sg)
    assert np.all(s[:, 2] == 0) and np.all(q[:, 8:] == 0)         # a zero group
    assert np.all(np.max(np.abs(q[:, :8].astype(int).reshape(5, 2, 4)), axis=2) == 127)


def test_int8_grouped_matmul_bruteforce_and_single_group():
    qa = RNG.integers(-127, 128, (3, 8)).astype(np.int8)
    wq = RNG.integers(-127, 128, (2, 8)).astype(np.int8)
    sa = RNG.uniform(0.01, 0.1, (3, 2)).astype(np.float32)
    sw = RNG.uniform(0.001, 0.01, 2).astype(np.float32)
    y = O.int8_grouped_matmul(qa, sa, wq, sw, 4)
    for m in range(3):
        for n in range(2):
            ref = sum(float(sa[m, k // 4]) * int(qa[m, k]) * int(wq[n, k]) for k in range(8))
            assert abs(y[m, n] - ref * float(sw[n])) < 1e-12
    # one group spanning K is the row-scaled product
    y1 = O.int8_grouped_matmul(qa, sa[:, :1], wq, sw, 8)
    ref = O.int_matmul(qa, wq) * sa[:, :1].astype(float) * sw[None, :].astype(float)
    assert np.allclose(y1, ref, atol=1e-14)


def test_int8_block_close_to_bf16_block_and_exact_parts():
    w, mod = _tiny_block(seed=51)
    for name in ("qkv", "fc1", "fc2"):
        w[f"w_{name}_q"], w[f"s_{name}"] = O.quantize_rows(w[f"w_{name}"].astype(np.float32))
    grid = (2, 2, 4)
    x = RNG.standard_normal((16 + 3, 64))
    pos = O.rope_positions(grid, 3)
    ref, _ = O.block_forward(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6)
    got = O.block_forward_int8(x, w, mod, pos, 2, (8, 12, 12), 1e4, 1e-6, group=64)
    # quantisation noise only: the int8 update stays close to the float update
    assert rel_l2(got - x, ref - x) < 3e-2
    # zero gates: identity, as in the float block
    mz = mod.copy()
    mz[2] = 0
    mz[5] = 0
    assert np.array_equal(O.block_forward_int8(x, w, mz, pos, 2, (8, 12, 12), 1e4, 1e-6, 64), x)
