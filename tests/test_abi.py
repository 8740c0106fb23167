"""The C-ABI library: it loads, exports every entry point that include/h3b.h declares,
rejects bad arguments before touching a GPU, and its host-side policy matches the
oracle.  No GPU needed."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import oracle as O
from video_diffusion_transformer_03_b200 import h3b, synth
from video_diffusion_transformer_03_b200.pipeline import dims_of, grid_of

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "h3b.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(h3b_[a-z0-9_]+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("h3b_block_forward", "h3b_denoise_step", "h3b_token_reduce",
                     "h3b_fc2_int8_row", "h3b_workspace_size", "h3b_last_error", "h3b_version"):
        assert required in names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", h3b.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (h3b_\w+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(h3b.LIB_PATH)
    for n in names:
        assert getattr(lib, n) is not None
    # the binding wraps exactly the declared entry points
    assert sorted(h3b.EXPORTS) == names


def test_version_and_error_string():
    assert h3b.version() == 1
    assert isinstance(h3b.lib.h3b_last_error(), bytes)


def _err(fn, *args):
    rc = fn(*args)
    return rc, h3b.lib.h3b_last_error().decode()


def test_validation_rejects_before_any_launch():
    L = h3b.lib
    p = ctypes.c_void_p(4096)       # aligned, never dereferenced: validation fails first
    rc, msg = _err(L.h3b_gemm_bf16, p, p, 64, 256, 65, 0, p, None, None, 0, 128, p, None, 0, None)
    assert rc == h3b.H3B_EINVAL and "K=65" in msg
    rc, _ = _err(L.h3b_gemm_bf16, p, p, 64, 200, 64, 0, p, None, None, 0, 128, p, None, 0, None)
    assert rc == h3b.H3B_EINVAL
    rc, _ = _err(L.h3b_gemm_bf16, p, p, 64, 256, 64, 3, p, None, None, 0, 128, p, None, 0, None)
    assert rc == h3b.H3B_EINVAL                                  # gate missing
    rc, _ = _err(L.h3b_gemm_bf16, ctypes.c_void_p(4097), p, 64, 256, 64, 0, p, None, None, 0,
                 128, p, None, 0, None)
    assert rc == h3b.H3B_EINVAL                                  # misaligned A
    rc, _ = _err(L.h3b_attention, p, 10, 2, 96, p, None, 0, None)
    assert rc == h3b.H3B_EINVAL                                  # head_dim 96
    rc, _ = _err(L.h3b_attention, p, 10, 2, 128, p, ctypes.c_void_p(4100), 1 << 30, None)
    assert rc == h3b.H3B_EINVAL                                  # misaligned scratch
    rc, _ = _err(L.h3b_token_reduce, 0, p, p, None, 2, 2, 3, 0, 64, None)
    assert rc == h3b.H3B_EINVAL                                  # odd w
    rc, _ = _err(L.h3b_token_reduce, 7, p, p, None, 2, 2, 4, 0, 64, None)
    assert rc == h3b.H3B_EINVAL                                  # unknown mode
    rc, _ = _err(L.h3b_quantize_rows, p, 4, 40, p, p, None)
    assert rc == h3b.H3B_EINVAL                                  # cols % 16
    rc, _ = _err(L.h3b_fc2_int8_row, p, 8, 100, 256, p, p, None, p, p, p, p, None, None, 0, None)
    assert rc == h3b.H3B_EINVAL                                  # K % 128
    rc, _ = _err(L.h3b_ln_modulate, p, 4, 300, ctypes.c_float(1e-6), p, p, p, None)
    assert rc == h3b.H3B_EINVAL                                  # d % 256


def test_block_and_step_validation():
    cfg = synth.CONFIGS["tiny"]
    dims = dims_of(cfg)
    bad = h3b.make_dims(250, 4, 64, 1024, 256, (16, 24, 24))
    w = h3b.BlockWeights(*([4096] * 8))
    p = ctypes.c_void_p(4096)
    rc = h3b.lib.h3b_block_forward(ctypes.byref(bad), ctypes.byref(w), p, None, p, 40, 1, p, p,
                                   p, 1 << 30, None)
    assert rc == h3b.H3B_EINVAL
    odd = h3b.make_dims(256, 4, 64, 1024, 256, (16, 23, 25))
    assert h3b.lib.h3b_block_forward(ctypes.byref(odd), ctypes.byref(w), p, None, p, 40, 1, p,
                                     p, p, 1 << 30, None) == h3b.H3B_EINVAL
    need = h3b.workspace_size(dims, 40)
    rc = h3b.lib.h3b_block_forward(ctypes.byref(dims), ctypes.byref(w), p, None, p, 40, 1, p, p,
                                   p, need - 1, None)
    assert rc == h3b.H3B_EWORKSPACE
    grid = grid_of(cfg)
    arr = (h3b.BlockWeights * 1)(w)
    need = h3b.denoise_workspace_size(dims, grid, False)
    rc = h3b.lib.h3b_denoise_step(ctypes.byref(dims), ctypes.byref(grid), 1, arr, None, p, p,
                                  -1, 1, 1.0, 0.75, p, p, need - 256, None)
    assert rc == h3b.H3B_EWORKSPACE
    odd_grid = h3b.make_grid(2, 4, 3, 8)
    rc = h3b.lib.h3b_denoise_step(ctypes.byref(dims), ctypes.byref(odd_grid), 1, arr, None, p, p,
                                  1, 1, 1.0, 0.75, p, p, 1 << 30, None)
    assert rc == h3b.H3B_EINVAL


def test_workspace_sizes():
    for name in ("tiny", "dit512", "dit512_tokred", "dit768x1344"):
        cfg = synth.CONFIGS[name]
        dims = dims_of(cfg)
        n = cfg.n_tokens
        arena = h3b.workspace_size(dims, n)
        assert arena % 256 == 0
        assert arena >= n * max(4 * cfg.d, cfg.d_ff) * 2
        step = h3b.denoise_workspace_size(dims, grid_of(cfg), cfg.reduce_after > 0)
        assert step >= arena + 2 * n * cfg.d * 2 + n * cfg.head_dim * 4
        if cfg.reduce_after > 0:
            assert step > h3b.denoise_workspace_size(dims, grid_of(cfg), False)


def test_layer_mask_matches_oracle():
    rng = np.random.default_rng(0)
    for trial in range(50):
        nb = int(rng.integers(3, 12))
        d = int(rng.integers(1, 40))
        mods = rng.standard_normal((nb, 6, d)).astype(np.float32)
        if trial % 5 == 0:
            mods[1] = mods[2]                       # exact tie between two interior blocks
        n_active = int(rng.integers(2, nb + 1))
        assert np.array_equal(h3b.layer_mask(mods, n_active), O.layer_mask(mods, n_active))
    with pytest.raises(h3b.H3BError):
        h3b.layer_mask(np.zeros((4, 6, 8), np.float32), 1)
