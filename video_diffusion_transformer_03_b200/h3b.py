"""ctypes binding of libh3b.so (argument marshalling only).

Every function takes torch tensors that already live where the C ABI expects them
(device tensors for device pointers) and passes their data pointers, sizes and the
current CUDA stream.  All computation happens in the CUDA library; there is no fallback:
importing this module fails if libh3b.so has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libh3b.so")

H3B_OK, H3B_EINVAL, H3B_EWORKSPACE, H3B_ECUDA, H3B_ETIMEOUT, H3B_EUNSUPPORTED = 0, -1, -2, -3, -4, -5
PAIR, UNPAIR = 0, 1
EPI_BIAS, EPI_BIAS_GELU, EPI_BIAS_ROPE, EPI_GATE_RESID = 0, 1, 2, 3
EPI_LN_ROPE, EPI_LN_GELU = 4, 5


class H3BError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"h3b error {code}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("d_ff", ctypes.c_int), ("c_dim", ctypes.c_int), ("rope_split", ctypes.c_int * 3),
                ("rope_theta", ctypes.c_float), ("ln_eps", ctypes.c_float)]


class Grid(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int),
                ("n_audio", ctypes.c_int), ("rope_halved", ctypes.c_int)]


WEIGHT_FIELDS = ("w_qkv", "b_qkv", "w_o", "b_o", "w_fc1", "b_fc1", "w_fc2", "b_fc2")
FOLD_FIELDS = ("w_qkv_fold", "c_qkv", "d_qkv", "w_fc1_fold", "c_fc1", "d_fc1")
QK_FIELDS = ("q_norm", "k_norm")


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS + FOLD_FIELDS + QK_FIELDS]


class LatentHeads(ctypes.Structure):
    _fields_ = [("c_lat", ctypes.c_int), ("w_patch", ctypes.c_void_p * 2),
                ("b_patch", ctypes.c_void_p * 2), ("w_head_fold", ctypes.c_void_p * 2),
                ("c_head", ctypes.c_void_p * 2), ("dv_head", ctypes.c_void_p * 2)]


class Int8Block(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_qkv_q", "s_qkv", "w_fc1_q", "s_fc1", "w_fc2_q", "s_fc2")]


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_SIGS = {
    "h3b_version": (_I, []),
    "h3b_last_error": (ctypes.c_char_p, []),
    "h3b_launch_count": (ctypes.c_uint64, []),
    "h3b_sync_status": (_I, [_P]),
    "h3b_workspace_size": (_SZ, [ctypes.POINTER(Dims), _I]),
    "h3b_gemm_workspace_size": (_SZ, []),
    "h3b_denoise_workspace_size": (_SZ, [ctypes.POINTER(Dims), ctypes.POINTER(Grid), _I]),
    "h3b_gemm_schedule": (_I, [_I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int), _I]),
    "h3b_set_gemm_override": (_I, [_I, _I, _I]),
    "h3b_set_attention_variant": (_I, [_I]),
    "h3b_adaln_modulation": (_I, [_P, _P, _P, _I, _I, _P, _P]),
    "h3b_rope_table": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(Grid), _I, _P, _P]),
    "h3b_ln_modulate": (_I, [_P, _I, _I, _F, _P, _P, _P, _P]),
    "h3b_block_forward": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights), _P, _P, _P,
                               _I, _I, _P, _P, _P, _SZ, _P]),
    "h3b_block_forward_noalloc": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights), _P,
                                       _P, _P, _I, _I, _P, _P, _P]),
    "h3b_fold_adaln": (_I, [_P, _P, _P, _P, _I, _I, _P, _P, _P, _P]),
    "h3b_row_stats": (_I, [_P, _I, _I, _P, _P]),
    "h3b_block_forward_folded": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights), _P, _P,
                                      _I, _P, _P, _P, _SZ, _P]),
    "h3b_final_euler": (_I, [_P, _I, _I, _I, _F, _P, _F, _F, _P, _P]),
    "h3b_denoise_step": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(Grid), _I,
                              ctypes.POINTER(BlockWeights), _P, _P, _P, _I, _I, _F, _F, _P, _P,
                              _SZ, _P]),
    "h3b_denoise_host": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(Grid), _I,
                              ctypes.POINTER(BlockWeights), _P, _P, _P, _I, _I, _I, _I, _I, _P,
                              _P, _P, _P, _SZ, _P]),
    "h3b_denoise_host_pipelined": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(Grid), _I,
                                        ctypes.POINTER(BlockWeights), _P, _P, _P, _I, _I, _I,
                                        _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "h3b_denoise_latent_workspace_size": (_SZ, [ctypes.POINTER(Dims), ctypes.POINTER(Grid), _I,
                                                _I]),
    "h3b_denoise_step_latent": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(Grid), _I,
                                     ctypes.POINTER(BlockWeights), _P, _P,
                                     ctypes.POINTER(LatentHeads), _I, _I, _F, _F, _P, _P, _SZ,
                                     _P]),
    "h3b_workspace_size_int8": (_SZ, [ctypes.POINTER(Dims), _I]),
    "h3b_block_forward_int8": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights),
                                    ctypes.POINTER(Int8Block), _P, _P, _I, _P, _P, _SZ, _P]),
    "h3b_ln_modulate_q8": (_I, [_P, _I, _I, _F, _P, _P, _P, _P, _P]),
    "h3b_quantize_groups": (_I, [_P, _I, _I, _P, _P, _P]),
    "h3b_gemm_i8_grouped": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "h3b_reuse_schedule": (_I, [_I, _I, _P]),
    "h3b_denoise_step_keep": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(Grid), _I,
                                   ctypes.POINTER(BlockWeights), _P, _P, _P, _I, _I, _F, _F, _P,
                                   _P, _P, _P, _SZ, _P]),
    "h3b_euler_velocity": (_I, [_P, _I, _I, _F, _F, _P, _P]),
    "h3b_euler_core_reuse": (_I, [_P, _I, _I, _I, _F, _P, _F, _F, _P, _P]),
    "h3b_token_reduce": (_I, [_I, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "h3b_quantize_rows": (_I, [_P, _I, _I, _P, _P, _P]),
    "h3b_fc2_int8_row": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "h3b_gemm_bf16": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _I, _I, _P, _P, _SZ, _P]),
    "h3b_gemm_bf16_ln": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _F, _P, _I, _I,
                              _P, _P, _P, _P, _SZ, _P]),
    "h3b_attention": (_I, [_P, _I, _I, _I, _P, _P, _SZ, _P]),
    "h3b_layer_mask": (_I, [_P, _I, _I, _I, _P]),
}

EXPORTS = tuple(_SIGS)


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m video_diffusion_transformer_03_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()
LIB_PATH = _LIB_PATH


def _check(rc: int) -> None:
    if rc != H3B_OK:
        raise H3BError(rc, lib.h3b_last_error().decode(errors="replace"))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to h3b must be contiguous")
    return t.data_ptr()


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if not t.is_cuda or t.dtype != dtype:
        raise TypeError(f"{name}: expected a CUDA {dtype} tensor, got {t.device} {t.dtype}")


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


# ---------------------------------------------------------------------- plumbing
def version() -> int:
    return lib.h3b_version()


def launch_count() -> int:
    return int(lib.h3b_launch_count())


def sync_status(stream=None) -> None:
    _check(lib.h3b_sync_status(_stream(stream)))


def make_dims(d, n_heads, head_dim, d_ff, c_dim, rope_split, rope_theta=10000.0, ln_eps=1e-6) -> Dims:
    return Dims(d, n_heads, head_dim, d_ff, c_dim, (ctypes.c_int * 3)(*rope_split),
                rope_theta, ln_eps)


def make_grid(t, h, w, n_audio, rope_halved=False) -> Grid:
    return Grid(t, h, w, n_audio, int(bool(rope_halved)))


def make_block_weights(p) -> BlockWeights:
    """p: mapping with the eight bf16 CUDA tensors w_qkv, b_qkv, w_o, b_o, w_fc1, b_fc1,
    w_fc2, b_fc2, and optionally the six folded ones (fold_block): w_qkv_fold, w_fc1_fold
    (bf16) and c_qkv, d_qkv, c_fc1, d_fc1 (fp32)."""
    for k in WEIGHT_FIELDS:
        _dev(p[k], torch.bfloat16, k)
    folded = all(k in p for k in FOLD_FIELDS)
    if folded:
        for k in FOLD_FIELDS:
            _dev(p[k], torch.bfloat16 if k.startswith("w_") else torch.float32, k)
    qk = all(p.get(k) is not None for k in QK_FIELDS)
    if qk:
        for k in QK_FIELDS:
            _dev(p[k], torch.float32, k)
    return BlockWeights(*[_ptr(p[k]) for k in WEIGHT_FIELDS],
                        *[_ptr(p[k]) if folded else None for k in FOLD_FIELDS],
                        *[_ptr(p[k]) if qk else None for k in QK_FIELDS])


def gemm_workspace_size() -> int:
    return int(lib.h3b_gemm_workspace_size())


SCHED_DATA_PARALLEL, SCHED_HYBRID_STREAM_K, SCHED_STREAM_K = 0, 1, 2
SCHED_REMAINDER_STREAM_K = 3  # h3b_gemm_schedule only: the grouped int8 kernel's form


def gemm_schedule(tiles: int, k_blocks: int, units: int, mode: int, unit: int):
    """Work items (tile, first K slice, end K slice, merge) of one GEMM scheduling unit, in
    processing order, as the kernels compute them (host only, no GPU)."""
    cap = 16
    while True:
        buf = (ctypes.c_int * (4 * cap))()
        n = int(lib.h3b_gemm_schedule(tiles, k_blocks, units, mode, unit, buf, cap))
        if n < 0:
            _check(n)
        if n <= cap:
            return [tuple(buf[4 * i:4 * i + 4]) for i in range(n)]
        cap = n


TILE_PAIR256, TILE_PAIR128, TILE_SINGLE256, TILE_SINGLE128 = 0, 1, 2, 3


def set_gemm_override(tile: int = -1, sched: int = -1, trans: int = -1) -> None:
    """Force the GEMM tile configuration / schedule / transposed kernel for later launches
    of this process (tests and measurements); -1 restores the automatic choice."""
    _check(lib.h3b_set_gemm_override(tile, sched, trans))


ATTN_AUTO, ATTN_ONE_TILE, ATTN_TWO_TILES, ATTN_TWO_TILES_POLY = 0, 1, 2, 3


def set_attention_variant(variant: int) -> None:
    """Attention form for later launches (tests and measurements)."""
    _check(lib.h3b_set_attention_variant(variant))


class attention_variant:
    """Context manager around set_attention_variant that restores the automatic form."""

    def __init__(self, variant: int):
        self.variant = variant

    def __enter__(self):
        set_attention_variant(self.variant)
        return self

    def __exit__(self, *exc):
        set_attention_variant(ATTN_AUTO)
        return False


class gemm_override:
    """Context manager around set_gemm_override that restores the automatic choice."""

    def __init__(self, tile: int = -1, sched: int = -1, trans: int = -1):
        self.args = (tile, sched, trans)

    def __enter__(self):
        set_gemm_override(*self.args)
        return self

    def __exit__(self, *exc):
        set_gemm_override(-1, -1, -1)
        return False


def _wsargs(ws):
    if ws is None:
        return None, 0
    return _ptr(ws), ws.numel() * ws.element_size()


def workspace_size(dims: Dims, n_tokens: int) -> int:
    return lib.h3b_workspace_size(ctypes.byref(dims), n_tokens)


def denoise_workspace_size(dims: Dims, grid: Grid, reduce: bool) -> int:
    return lib.h3b_denoise_workspace_size(ctypes.byref(dims), ctypes.byref(grid), int(bool(reduce)))


def workspace(nbytes: int, device=None) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device or "cuda")


# ---------------------------------------------------------------------- steps
def adaln_modulation(w, b, c, out, stream=None) -> None:
    _dev(w, torch.bfloat16, "w"); _dev(b, torch.bfloat16, "b"); _dev(c, torch.bfloat16, "c")
    _dev(out, torch.float32, "out")
    c_dim = w.shape[-1]
    n_out = w.numel() // c_dim
    _check(lib.h3b_adaln_modulation(_ptr(w), _ptr(b), _ptr(c), n_out, c_dim, _ptr(out),
                                    _stream(stream)))


def rope_table(dims: Dims, grid: Grid, paired: bool, out, stream=None) -> None:
    _dev(out, torch.float32, "rope_cs")
    _check(lib.h3b_rope_table(ctypes.byref(dims), ctypes.byref(grid), int(bool(paired)),
                              _ptr(out), _stream(stream)))


def ln_modulate(x, eps, shift, scale, h, stream=None) -> None:
    _dev(x, torch.bfloat16, "x"); _dev(h, torch.bfloat16, "h")
    _check(lib.h3b_ln_modulate(_ptr(x), x.shape[0], x.shape[1], eps, _ptr(shift), _ptr(scale),
                               _ptr(h), _stream(stream)))


def block_forward(dims: Dims, weights: BlockWeights, mod, mod_next, rope_cs, x, h, ws,
                  compute_h: bool, stream=None) -> None:
    _dev(x, torch.bfloat16, "x"); _dev(h, torch.bfloat16, "h"); _dev(mod, torch.float32, "mod")
    _check(lib.h3b_block_forward(ctypes.byref(dims), ctypes.byref(weights), _ptr(mod),
                                 _ptr(mod_next), _ptr(rope_cs), x.shape[0], int(bool(compute_h)),
                                 _ptr(x), _ptr(h), _ptr(ws), ws.numel() * ws.element_size(),
                                 _stream(stream)))


def fold_adaln(w, b, shift, scale, w_out, c_out, d_out, stream=None) -> None:
    """W' = bf16(W diag(1 + scale)), c = row sums of W', d = W shift + b (h3b_fold_adaln)."""
    _dev(w, torch.bfloat16, "w"); _dev(b, torch.bfloat16, "b"); _dev(w_out, torch.bfloat16, "w_out")
    _dev(shift, torch.float32, "shift"); _dev(scale, torch.float32, "scale")
    _dev(c_out, torch.float32, "c_out"); _dev(d_out, torch.float32, "d_out")
    n_out, d = w.shape
    _check(lib.h3b_fold_adaln(_ptr(w), _ptr(b), _ptr(shift), _ptr(scale), n_out, d, _ptr(w_out),
                              _ptr(c_out), _ptr(d_out), _stream(stream)))


def fold_block(p, mod, stream=None):
    """The folded fields of one block (device tensors) from its weights p and its AdaLN
    vectors mod [6, d]: (shift_msa, scale_msa) into w_qkv, (shift_mlp, scale_mlp) into w_fc1."""
    out = {}
    for name, sh, sc in (("qkv", 0, 1), ("fc1", 3, 4)):
        w, b = p["w_" + name], p["b_" + name]
        out["w_%s_fold" % name] = torch.empty_like(w)
        out["c_" + name] = torch.empty(w.shape[0], dtype=torch.float32, device=w.device)
        out["d_" + name] = torch.empty(w.shape[0], dtype=torch.float32, device=w.device)
        fold_adaln(w, b, mod[sh].contiguous(), mod[sc].contiguous(), out["w_%s_fold" % name],
                   out["c_" + name], out["d_" + name], stream)
    return out


def row_stats(x, stats, stream=None) -> None:
    """stats [n, d / 256, 2] fp32: per row and 256-column group, (mean, M2) of x."""
    _dev(x, torch.bfloat16, "x"); _dev(stats, torch.float32, "stats")
    _check(lib.h3b_row_stats(_ptr(x), x.shape[0], x.shape[1], _ptr(stats), _stream(stream)))


def block_forward_folded(dims: Dims, weights: BlockWeights, mod, rope_cs, x, stats, ws,
                         stream=None) -> None:
    _dev(x, torch.bfloat16, "x"); _dev(stats, torch.float32, "stats"); _dev(mod, torch.float32, "mod")
    _check(lib.h3b_block_forward_folded(ctypes.byref(dims), ctypes.byref(weights), _ptr(mod),
                                        _ptr(rope_cs), x.shape[0], _ptr(x), _ptr(stats), _ptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)))


NOALLOC_WORKSPACE_BYTES = 64 << 20


def block_forward_noalloc(dims: Dims, weights: BlockWeights, mod, mod_next, rope_cs, x, h,
                          compute_h: bool, stream=None) -> None:
    """h3b_block_forward with the library's static workspace instead of a caller buffer
    (for callers that cannot allocate device memory).  Calls that overlap on the GPU
    share that workspace and race; serialise them."""
    _dev(x, torch.bfloat16, "x"); _dev(h, torch.bfloat16, "h"); _dev(mod, torch.float32, "mod")
    _check(lib.h3b_block_forward_noalloc(ctypes.byref(dims), ctypes.byref(weights), _ptr(mod),
                                         _ptr(mod_next), _ptr(rope_cs), x.shape[0],
                                         int(bool(compute_h)), _ptr(x), _ptr(h),
                                         _stream(stream)))


def final_euler(x_l, n_video, eps, final_mod, sigma, sigma_next, x_state, stream=None) -> None:
    _dev(x_l, torch.bfloat16, "x_l"); _dev(x_state, torch.float32, "x_state")
    _check(lib.h3b_final_euler(_ptr(x_l), x_l.shape[0], n_video, x_l.shape[1], eps,
                               _ptr(final_mod), sigma, sigma_next, _ptr(x_state), _stream(stream)))


def _blocks_array(blocks: Sequence[BlockWeights]):
    arr = (BlockWeights * max(len(blocks), 1))()
    for i, b in enumerate(blocks):
        arr[i] = b
    return arr


def _mask_array(active, n):
    if active is None:
        return None, None
    buf = (ctypes.c_ubyte * n)(*[1 if a else 0 for a in active])
    return buf, ctypes.cast(buf, ctypes.c_void_p)


def denoise_step(dims: Dims, grid: Grid, blocks: Sequence[BlockWeights], active, mods, final_mod,
                 reduce_after: int, unpair_bypass: bool, sigma: float, sigma_next: float, x_state,
                 ws, stream=None) -> None:
    _dev(x_state, torch.float32, "x_state")
    arr = _blocks_array(blocks)
    keep, mask = _mask_array(active, len(blocks))
    _check(lib.h3b_denoise_step(ctypes.byref(dims), ctypes.byref(grid), len(blocks), arr, mask,
                                _ptr(mods), _ptr(final_mod), reduce_after, int(bool(unpair_bypass)),
                                sigma, sigma_next, _ptr(x_state), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def make_latent_heads(c_lat: int, t) -> LatentHeads:
    """t: mapping with per-stream lists of device tensors w_patch, b_patch (bf16),
    w_head_fold (bf16), c_head, dv_head (fp32), each of length 2 (video, audio)."""
    h = LatentHeads()
    h.c_lat = c_lat
    for name in ("w_patch", "b_patch", "w_head_fold", "c_head", "dv_head"):
        arr = getattr(h, name)
        for st in range(2):
            arr[st] = _ptr(t[name][st])
    return h


def denoise_latent_workspace_size(dims: Dims, grid: Grid, reduce: bool, c_lat: int) -> int:
    return lib.h3b_denoise_latent_workspace_size(ctypes.byref(dims), ctypes.byref(grid),
                                                 int(bool(reduce)), c_lat)


def denoise_step_latent(dims: Dims, grid: Grid, blocks: Sequence[BlockWeights], active, mods,
                        heads: LatentHeads, reduce_after: int, unpair_bypass: bool, sigma: float,
                        sigma_next: float, latent, ws, stream=None) -> None:
    _dev(latent, torch.float32, "latent")
    arr = _blocks_array(blocks)
    keep, mask = _mask_array(active, len(blocks))
    _check(lib.h3b_denoise_step_latent(ctypes.byref(dims), ctypes.byref(grid), len(blocks), arr,
                                       mask, _ptr(mods), ctypes.byref(heads), reduce_after,
                                       int(bool(unpair_bypass)), sigma, sigma_next, _ptr(latent),
                                       _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def quantize_block_int8(p, stream=None):
    """Int8 weights of one block (device tensors) from its bf16 weights p: per-output-
    channel quantize_rows of w_qkv, w_fc1, w_fc2.  Returns (tensors, Int8Block)."""
    t = {}
    for name in ("qkv", "fc1", "fc2"):
        w = p["w_" + name]
        t["w_%s_q" % name] = torch.empty(w.shape, dtype=torch.int8, device=w.device)
        t["s_" + name] = torch.empty(w.shape[0], dtype=torch.float32, device=w.device)
        quantize_rows(w, t["w_%s_q" % name], t["s_" + name], stream)
    return t, Int8Block(*[_ptr(t[k]) for k in ("w_qkv_q", "s_qkv", "w_fc1_q", "s_fc1",
                                                 "w_fc2_q", "s_fc2")])


def workspace_size_int8(dims: Dims, n_tokens: int) -> int:
    return lib.h3b_workspace_size_int8(ctypes.byref(dims), n_tokens)


def block_forward_int8(dims: Dims, weights: BlockWeights, wq: Int8Block, mod, rope_cs, x, ws,
                       stream=None) -> None:
    _dev(x, torch.bfloat16, "x"); _dev(mod, torch.float32, "mod")
    _check(lib.h3b_block_forward_int8(ctypes.byref(dims), ctypes.byref(weights), ctypes.byref(wq),
                                      _ptr(mod), _ptr(rope_cs), x.shape[0], _ptr(x), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)))


def ln_modulate_q8(x, eps, shift, scale, q, q_scale, stream=None) -> None:
    _dev(x, torch.bfloat16, "x"); _dev(q, torch.int8, "q"); _dev(q_scale, torch.float32, "q_scale")
    _check(lib.h3b_ln_modulate_q8(_ptr(x), x.shape[0], x.shape[1], eps, _ptr(shift), _ptr(scale),
                                  _ptr(q), _ptr(q_scale), _stream(stream)))


def quantize_groups(a, q, scale, stream=None) -> None:
    _dev(a, torch.bfloat16, "a"); _dev(q, torch.int8, "q"); _dev(scale, torch.float32, "scale")
    _check(lib.h3b_quantize_groups(_ptr(a), a.shape[0], a.shape[1], _ptr(q), _ptr(scale),
                                   _stream(stream)))


def gemm_i8_grouped(A, a_scale, w_q, w_scale, bias, gate, resid, ws=None,
                    stream=None) -> None:
    """ws: None (data-parallel) or a device buffer of gemm_workspace_size() bytes (a partial
    last wave of tiles runs stream-K over the 1024-column groups)."""
    _dev(A, torch.int8, "A"); _dev(w_q, torch.int8, "w_q"); _dev(resid, torch.bfloat16, "resid")
    M, K = A.shape
    _check(lib.h3b_gemm_i8_grouped(_ptr(A), _ptr(a_scale), M, K, w_q.shape[0], _ptr(w_q),
                                   _ptr(w_scale), _ptr(bias), _ptr(gate), _ptr(resid),
                                   _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                   _stream(stream)))


def reuse_schedule(steps: int, every: int) -> np.ndarray:
    """Host policy: which of `steps` Euler steps run the model (h3b_reuse_schedule)."""
    out = (ctypes.c_ubyte * max(steps, 1))()
    n = int(lib.h3b_reuse_schedule(steps, every, ctypes.cast(out, ctypes.c_void_p)))
    if n < 0:
        _check(n)
    return np.array(list(out)[:steps], dtype=bool)


def denoise_step_keep(dims: Dims, grid: Grid, blocks: Sequence[BlockWeights], active, mods,
                      final_mod, reduce_after: int, unpair_bypass: bool, sigma: float,
                      sigma_next: float, x_state, v_out, core_res_out, ws, stream=None) -> None:
    _dev(x_state, torch.float32, "x_state")
    arr = _blocks_array(blocks)
    keep, mask = _mask_array(active, len(blocks))
    _check(lib.h3b_denoise_step_keep(ctypes.byref(dims), ctypes.byref(grid), len(blocks), arr,
                                     mask, _ptr(mods), _ptr(final_mod), reduce_after,
                                     int(bool(unpair_bypass)), sigma, sigma_next, _ptr(x_state),
                                     _ptr(v_out), _ptr(core_res_out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def euler_velocity(v, sigma, sigma_next, x_state, stream=None) -> None:
    _dev(v, torch.float32, "v"); _dev(x_state, torch.float32, "x_state")
    _check(lib.h3b_euler_velocity(_ptr(v), x_state.shape[0], x_state.shape[1], sigma, sigma_next,
                                  _ptr(x_state), _stream(stream)))


def euler_core_reuse(core_res, n_video, eps, final_mod, sigma, sigma_next, x_state,
                     stream=None) -> None:
    _dev(core_res, torch.float32, "core_res"); _dev(x_state, torch.float32, "x_state")
    _check(lib.h3b_euler_core_reuse(_ptr(core_res), x_state.shape[0], n_video, x_state.shape[1],
                                    eps, _ptr(final_mod), sigma, sigma_next, _ptr(x_state),
                                    _stream(stream)))


def denoise_host(dims: Dims, grid: Grid, blocks: Sequence[BlockWeights], active, mods, final_mod,
                 reduce_after: int, unpair_bypass: bool, n_steps: int, first_step: int, n_run: int,
                 x_host_in, x_host_out, x_state_dev, ws, stream=None) -> None:
    """x_host_in / x_host_out: CPU float32 tensors (pinned for full bandwidth)."""
    if x_host_in.is_cuda or x_host_out.is_cuda:
        raise TypeError("denoise_host takes host buffers")
    arr = _blocks_array(blocks)
    keep, mask = _mask_array(active, len(blocks))
    _check(lib.h3b_denoise_host(ctypes.byref(dims), ctypes.byref(grid), len(blocks), arr, mask,
                                _ptr(mods), _ptr(final_mod), reduce_after, int(bool(unpair_bypass)),
                                n_steps, first_step, n_run, _ptr(x_host_in), _ptr(x_host_out),
                                _ptr(x_state_dev), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)))
    del keep


def denoise_host_pipelined(dims: Dims, grid: Grid, blocks: Sequence[BlockWeights], active, mods,
                           final_mod, reduce_after: int, unpair_bypass: bool, n_steps: int,
                           first_step: int, n_run: int, x_host_in, x_host_out, x_state_dev2,
                           ws, stream=None) -> None:
    """x_host_in / x_host_out: CPU float32 [requests, n_tokens, d] (pinned);
    x_state_dev2: device float32 [2, n_tokens, d]."""
    if x_host_in.is_cuda or x_host_out.is_cuda:
        raise TypeError("denoise_host_pipelined takes host buffers")
    if x_host_in.shape != x_host_out.shape or x_state_dev2.shape[0] != 2:
        raise ValueError("denoise_host_pipelined: shapes")
    arr = _blocks_array(blocks)
    keep, mask = _mask_array(active, len(blocks))
    _check(lib.h3b_denoise_host_pipelined(
        ctypes.byref(dims), ctypes.byref(grid), len(blocks), arr, mask, _ptr(mods),
        _ptr(final_mod), reduce_after, int(bool(unpair_bypass)), n_steps, first_step, n_run,
        x_host_in.shape[0], _ptr(x_host_in), _ptr(x_host_out), _ptr(x_state_dev2), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def token_reduce(mode: int, src, dst, saved, t, h, w, n_audio, stream=None) -> None:
    _dev(src, torch.bfloat16, "src"); _dev(dst, torch.bfloat16, "dst")
    _check(lib.h3b_token_reduce(mode, _ptr(src), _ptr(dst), _ptr(saved), t, h, w, n_audio,
                                src.shape[1], _stream(stream)))


def quantize_rows(a, q, scale, stream=None) -> None:
    _dev(a, torch.bfloat16, "a"); _dev(q, torch.int8, "q"); _dev(scale, torch.float32, "scale")
    _check(lib.h3b_quantize_rows(_ptr(a), a.shape[0], a.shape[1], _ptr(q), _ptr(scale),
                                 _stream(stream)))


def fc2_int8_row(act, w_q, w_scale, bias, gate, resid, act_q, row_scale, acc_out=None,
                 ws=None, stream=None) -> None:
    _dev(act, torch.bfloat16, "act"); _dev(w_q, torch.int8, "w_q"); _dev(resid, torch.bfloat16, "resid")
    M, K = act.shape
    wp, wb = _wsargs(ws)
    _check(lib.h3b_fc2_int8_row(_ptr(act), M, K, w_q.shape[0], _ptr(w_q), _ptr(w_scale),
                                _ptr(bias), _ptr(gate), _ptr(resid), _ptr(act_q), _ptr(row_scale),
                                _ptr(acc_out), wp, wb, _stream(stream)))


def gemm_bf16(A, B, epilogue, bias, out, gate=None, rope_cs=None, rope_cols=0, head_dim=128,
              ws=None, stream=None) -> None:
    _dev(A, torch.bfloat16, "A"); _dev(B, torch.bfloat16, "B"); _dev(out, torch.bfloat16, "out")
    M, K = A.shape
    N = B.shape[0]
    wp, wb = _wsargs(ws)
    _check(lib.h3b_gemm_bf16(_ptr(A), _ptr(B), M, N, K, epilogue, _ptr(bias), _ptr(gate),
                             _ptr(rope_cs), rope_cols, head_dim, _ptr(out), wp, wb,
                             _stream(stream)))


def gemm_bf16_ln(A, B, epilogue, out, bias=None, gate=None, fold_c=None, fold_dv=None,
                 stats_in=None, stats_out=None, ln_eps=1e-6, rope_cs=None, rope_cols=0,
                 head_dim=128, q_gain=None, k_gain=None, ws=None, stream=None) -> None:
    """The folded block's GEMM forms (h3b_gemm_bf16_ln): EPI_LN_ROPE / EPI_LN_GELU read the
    raw residual A with its row statistics stats_in; EPI_GATE_RESID may write stats_out;
    the RoPE forms take optional Q/K RMSNorm gains."""
    _dev(A, torch.bfloat16, "A"); _dev(B, torch.bfloat16, "B"); _dev(out, torch.bfloat16, "out")
    M, K = A.shape
    N = B.shape[0]
    wp, wb = _wsargs(ws)
    _check(lib.h3b_gemm_bf16_ln(_ptr(A), _ptr(B), M, N, K, epilogue, _ptr(bias), _ptr(gate),
                                _ptr(fold_c), _ptr(fold_dv), _ptr(stats_in), _ptr(stats_out),
                                ln_eps, _ptr(rope_cs), rope_cols, head_dim, _ptr(q_gain),
                                _ptr(k_gain), _ptr(out), wp, wb, _stream(stream)))


def attention(qkv, n_heads, head_dim, out, ws=None, stream=None) -> None:
    _dev(qkv, torch.bfloat16, "qkv"); _dev(out, torch.bfloat16, "out")
    wp, wb = _wsargs(ws)
    _check(lib.h3b_attention(_ptr(qkv), qkv.shape[0], n_heads, head_dim, _ptr(out), wp, wb,
                             _stream(stream)))


def layer_mask(mods_host: np.ndarray, n_active: int) -> np.ndarray:
    """mods_host: float32 [n_blocks, 6, d] on the host; returns a bool mask."""
    m = np.ascontiguousarray(mods_host, dtype=np.float32)
    nb, _, d = m.shape
    out = (ctypes.c_ubyte * nb)()
    _check(lib.h3b_layer_mask(m.ctypes.data, nb, d, n_active, ctypes.cast(out, ctypes.c_void_p)))
    return np.array(list(out), dtype=bool)
