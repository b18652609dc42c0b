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


def sample_rows_one_class(w, mode: int, count: int, cls: int = 0, head: int = 0, seed: int = 0) -> np.ndarray:
    """Rows (token*heads + head) of one (class, head) subsequence of batch element 0: its first
    and last real tokens plus `count` random ones (class rule from the brute force's own
    restatement). One subsequence keeps the backward oracle's per-subsequence cost bounded."""
    from oracle import brute
    step = w.P * w.P
    Hp, Wp = -(-w.H // step) * step, -(-w.W // step) * step
    grid = brute.class_grid(Hp, Wp, w.P, mode)[: w.H, : w.W]
    hh, ww = np.nonzero(grid == cls)
    toks = (np.arange(w.T)[:, None] * w.H * w.W + (hh * w.W + ww)[None, :]).reshape(-1)
    rng = np.random.default_rng(seed)
    pick = np.unique(np.concatenate([toks[:2], toks[-2:], rng.choice(toks, size=min(count, len(toks)), replace=False)]))
    return pick.astype(np.int64) * w.heads + head


def sample_rows_one_class_1d(w, mode: int, count: int, cls: int = 0, head: int = 0, seed: int = 0) -> np.ndarray:
    """sample_rows_one_class for Skiparse-1D: the class of in-frame index x = h*W + w from the
    brute force's own restatement of the 1D rule."""
    from oracle import brute
    k2 = (w.P * w.P) ** 2
    L = w.H * w.W
    Lp = -(-L // k2) * k2
    xs = np.nonzero(brute.class_1d(Lp, w.P, mode)[:L] == cls)[0]
    toks = (np.arange(w.T)[:, None] * L + xs[None, :]).reshape(-1)
    rng = np.random.default_rng(seed)
    pick = np.unique(np.concatenate([toks[:2], toks[-2:], rng.choice(toks, size=min(count, len(toks)), replace=False)]))
    return pick.astype(np.int64) * w.heads + head


def subsequence_rows(w, mode: int, cls: int, head: int, b: int = 0) -> np.ndarray:
    """Every row (token*heads + head) of one whole (b, class, head) subsequence, in token order,
    with the class rule from the brute force's own restatement."""
    from oracle import brute
    step = w.P * w.P
    Hp, Wp = -(-w.H // step) * step, -(-w.W // step) * step
    grid = brute.class_grid(Hp, Wp, w.P, mode)[: w.H, : w.W]
    hh, ww = np.nonzero(grid == cls)
    toks = (b * w.T * w.H * w.W + np.arange(w.T)[:, None] * w.H * w.W + (hh * w.W + ww)[None, :]).reshape(-1)
    return np.sort(toks).astype(np.int64) * w.heads + head
