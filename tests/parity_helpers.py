"""Shared helpers for the GPU parity tests (test infrastructure)."""

from __future__ import annotations

import numpy as np
import torch

# Tolerances for bf16 attention against the fp64 oracle, N(0,1) inputs, scale 1/sqrt(d).
MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def sample_rows(w, count: int, seed: int = 0) -> np.ndarray:
    """Deterministic sample of output rows (token*heads + head): uniform random tokens plus
    every frame/grid corner and the last real row and column (the pad-adjacent tokens)."""
    rng = np.random.default_rng(seed)
    B, T, H, W, heads = w.B, w.T, w.H, w.W, w.heads
    ntok = B * T * H * W
    toks = set(rng.integers(0, ntok, size=count).tolist())
    for b in (0, B - 1):
        for t in (0, T - 1):
            for h in (0, H - 1, H // 2):
                for ww in (0, W - 1, W // 2):
                    toks.add(((b * T + t) * H + h) * W + ww)
            for ww in range(W):  # the whole last real row of the last frame
                toks.add(((b * T + t) * H + (H - 1)) * W + ww)
    toks = np.array(sorted(toks), dtype=np.int64)
    hd = rng.integers(0, heads, size=toks.shape[0])
    hd[: min(heads, toks.shape[0])] = np.arange(min(heads, toks.shape[0]))
    return toks * heads + hd


def gpu_rows(out: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    d = out.shape[-1]
    idx = torch.from_numpy(rows).to(out.device)
    return out.reshape(-1, d).index_select(0, idx).to(torch.float64).cpu().numpy()


def check_close(got: np.ndarray, want: np.ndarray, what: str):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max|err|={mx:.3e} mean|err|={mean:.3e}"
    return mx, mean
