"""Shared helpers for the parity tests (no arithmetic of the method)."""
import numpy as np
import torch


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def rel_l2(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def max_block_rel_l2(got, want, rows: int = 128) -> float:
    """Largest rel-L2 over consecutive row blocks (a wrong tile cannot hide in the total)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    worst = 0.0
    for r0 in range(0, want.shape[0], rows):
        worst = max(worst, rel_l2(got[r0:r0 + rows], want[r0:r0 + rows]))
    return worst


def rnd(shape, std=1.0, seed=0, dtype=torch.bfloat16) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * std).to(dtype)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy()
