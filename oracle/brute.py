"""Second, independent oracle: brute-force dense attention with an explicit 2-D mask.

TEST INFRASTRUCTURE ONLY (tiny shapes). It shares nothing with skiparse_oracle.c: it
never forms subsequences. Instead it runs ONE dense fp64 attention over the whole
padded token grid and removes pairs with a 2-D mask
    M[x, y] = [class(x) == class(y)] and [y is a real token],
which is what the OSP-Next summary page's 前置知识 (prerequisites) section contrasts
with Skiparse (a dynamic 2-D mask, which Skiparse's fixed rearrangement avoids). Its
class rule is written here separately from the C oracle's, from the 核心方法 (core
method) section: token-wise (h mod P, w mod P), group-wise ((h div P) mod P,
(w div P) mod P).
"""

from __future__ import annotations

import numpy as np


def class_grid(Hp: int, Wp: int, P: int, mode: int) -> np.ndarray:
    h = np.arange(Hp)[:, None]
    w = np.arange(Wp)[None, :]
    if mode == 0:
        ci, cj = h % P, w % P
    else:
        ci, cj = (h // P) % P, (w // P) % P
    return (ci * P + cj).astype(np.int64)


def attention(q, k, v, P: int, mode: int) -> np.ndarray:
    """q, k, v: float64 (B,T,H,W,heads,d). Returns float64 (B,T,H,W,heads,d)."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, T, H, W, heads, d = q.shape
    step = P * P
    Hp = -(-H // step) * step
    Wp = -(-W // step) * step
    pad = ((0, 0), (0, 0), (0, Hp - H), (0, Wp - W), (0, 0), (0, 0))
    qp, kp, vp = (np.pad(a, pad) for a in (q, k, v))
    cls = np.broadcast_to(class_grid(Hp, Wp, P, mode), (T, Hp, Wp)).reshape(-1)
    real = np.zeros((T, Hp, Wp), dtype=bool)
    real[:, :H, :W] = True
    real = real.reshape(-1)
    mask = (cls[:, None] == cls[None, :]) & real[None, :]
    N = T * Hp * Wp
    out = np.zeros_like(qp)
    for b in range(B):
        for hd in range(heads):
            Q = qp[b, ..., hd, :].reshape(N, d)
            K = kp[b, ..., hd, :].reshape(N, d)
            V = vp[b, ..., hd, :].reshape(N, d)
            S = (Q[real] @ K.T) / np.sqrt(d)  # real queries only: pads give no output
            S = np.where(mask[real], S, -np.inf)
            S = S - S.max(axis=1, keepdims=True)
            E = np.exp(S)
            A = E / E.sum(axis=1, keepdims=True)
            O = np.zeros((N, d))
            O[real] = A @ V
            out[b, ..., hd, :] = O.reshape(T, Hp, Wp, d)
    return out[:, :, :H, :W]


def attention_torch(q, k, v, P: int, mode: int):
    """The same dense masked attention in torch fp64, differentiable (autograd gives the
    backward pass of the definition). Returns (out, lse) with lse the natural-log
    log-sum-exp of q.k/sqrt(d) over each real query's allowed keys."""
    import torch
    B, T, H, W, heads, d = q.shape
    step = P * P
    Hp = -(-H // step) * step
    Wp = -(-W // step) * step
    pad = (0, 0, 0, 0, 0, Wp - W, 0, Hp - H)
    qp, kp, vp = (torch.nn.functional.pad(a, pad) for a in (q, k, v))
    cls = torch.from_numpy(np.broadcast_to(class_grid(Hp, Wp, P, mode), (T, Hp, Wp)).reshape(-1).copy())
    real = torch.zeros((T, Hp, Wp), dtype=torch.bool)
    real[:, :H, :W] = True
    real = real.reshape(-1)
    mask = (cls[:, None] == cls[None, :]) & real[None, :]
    N = T * Hp * Wp
    outs, lses = [], []
    for b in range(B):
        ob, lb = [], []
        for hd in range(heads):
            Q = qp[b, ..., hd, :].reshape(N, d)[real]
            K = kp[b, ..., hd, :].reshape(N, d)
            V = vp[b, ..., hd, :].reshape(N, d)
            S = (Q @ K.T) / (d ** 0.5)
            S = S.masked_fill(~mask[real], float("-inf"))
            lse = torch.logsumexp(S, dim=1)
            A = torch.exp(S - lse[:, None])
            ob.append(A @ V)
            lb.append(lse)
        outs.append(torch.stack(ob, dim=1))   # (Nreal, heads, d)
        lses.append(torch.stack(lb, dim=1))   # (Nreal, heads)
    out = torch.stack(outs)                    # (B, Nreal, heads, d)
    lse = torch.stack(lses)
    # back to (B, T, H, W, heads, ...): real tokens in (t, h, w) order are exactly [:, :, :H, :W]
    return out.reshape(B, T, H, W, heads, d), lse.reshape(B, T, H, W, heads)


# ---------------------------------------------------------------------------- Skiparse-1D
# The 1D skip pattern on the flattened sequence (the variant the summary page's 技术新颖性 and
# 实验结果 sections compare Skiparse-2D with). Reading: the flattened in-frame index
# x = h*W + w, ratio k = P^2; token-wise class x mod k, group-wise class (x div k) mod k; each
# frame's H*W positions padded at the end to a multiple of k^2. Written here from that reading,
# separately from the C oracle.

def class_1d(Lp: int, P: int, mode: int) -> np.ndarray:
    x = np.arange(Lp)
    k = P * P
    return (x % k if mode == 0 else (x // k) % k).astype(np.int64)


def _frames_1d(a, P: int):
    """(B,T,H,W,heads,d) -> (B, T, Lp, heads, d) with the in-frame index flattened and padded."""
    B, T, H, W, heads, d = a.shape
    k2 = (P * P) ** 2
    L = H * W
    Lp = -(-L // k2) * k2
    flat = a.reshape(B, T, L, heads, d)
    return flat, L, Lp


def attention_1d(q, k, v, P: int, mode: int) -> np.ndarray:
    """Skiparse-1D forward by one dense fp64 attention per (batch, head) over all padded
    positions of all frames with the mask [class(x) == class(y)] and [y real]."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, T, H, W, heads, d = q.shape
    (qf, L, Lp), (kf, _, _), (vf, _, _) = (_frames_1d(a, P) for a in (q, k, v))
    pad = ((0, 0), (0, 0), (0, Lp - L), (0, 0), (0, 0))
    qp, kp, vp = (np.pad(a, pad) for a in (qf, kf, vf))
    cls = np.broadcast_to(class_1d(Lp, P, mode), (T, Lp)).reshape(-1)
    real = np.zeros((T, Lp), dtype=bool)
    real[:, :L] = True
    real = real.reshape(-1)
    mask = (cls[:, None] == cls[None, :]) & real[None, :]
    N = T * Lp
    out = np.zeros_like(qp)
    for b in range(B):
        for hd in range(heads):
            Q = qp[b, :, :, hd, :].reshape(N, d)
            K = kp[b, :, :, hd, :].reshape(N, d)
            V = vp[b, :, :, hd, :].reshape(N, d)
            S = (Q[real] @ K.T) / np.sqrt(d)
            S = np.where(mask[real], S, -np.inf)
            S = S - S.max(axis=1, keepdims=True)
            E = np.exp(S)
            O = np.zeros((N, d))
            O[real] = (E / E.sum(axis=1, keepdims=True)) @ V
            out[b, :, :, hd, :] = O.reshape(T, Lp, d)
    return out[:, :, :L].reshape(B, T, H, W, heads, d)


def attention_1d_torch(q, k, v, P: int, mode: int):
    """attention_1d in torch fp64, differentiable. Returns (out, lse)."""
    import torch
    B, T, H, W, heads, d = q.shape
    k2 = (P * P) ** 2
    L = H * W
    Lp = -(-L // k2) * k2
    qp, kp, vp = (torch.nn.functional.pad(a.reshape(B, T, L, heads, d), (0, 0, 0, 0, 0, Lp - L))
                  for a in (q, k, v))
    cls = torch.from_numpy(np.broadcast_to(class_1d(Lp, P, mode), (T, Lp)).reshape(-1).copy())
    real = torch.zeros((T, Lp), dtype=torch.bool)
    real[:, :L] = True
    real = real.reshape(-1)
    mask = (cls[:, None] == cls[None, :]) & real[None, :]
    N = T * Lp
    outs, lses = [], []
    for b in range(B):
        ob, lb = [], []
        for hd in range(heads):
            Q = qp[b, :, :, hd, :].reshape(N, d)[real]
            K = kp[b, :, :, hd, :].reshape(N, d)
            V = vp[b, :, :, hd, :].reshape(N, d)
            S = ((Q @ K.T) / (d ** 0.5)).masked_fill(~mask[real], float("-inf"))
            lse = torch.logsumexp(S, dim=1)
            ob.append(torch.exp(S - lse[:, None]) @ V)
            lb.append(lse)
        outs.append(torch.stack(ob, dim=1))
        lses.append(torch.stack(lb, dim=1))
    # real positions in (t, x) order are exactly the original tokens in (t, h, w) order
    return (torch.stack(outs).reshape(B, T, H, W, heads, d),
            torch.stack(lses).reshape(B, T, H, W, heads))
