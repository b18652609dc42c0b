"""Pins for the Skiparse-1D functions of the CPU oracle (the flattened-sequence variant).

The pages compare Skiparse-2D with Skiparse-1D (summary page, 技术新颖性 and 实验结果) but give
no formula for the latter. The reading the oracle takes: the flattened in-frame index
x = h*W + w, ratio k = P^2, token-wise class x mod k, group-wise class (x div k) mod k, and
each frame's H*W positions padded at the end to a multiple of k^2. Each test below names what
fixes the expected answer independently of the oracle's C code: numpy strided slicing and
reshape (the textbook form of a 1D skip and a 1D group skip), brute force over small
ranges, an independent dense attention with an explicit 1-D class mask, closed forms for
frames whose width is a multiple of the ratio, scaled_dot_product_attention at P = 1, and
torch autograd for the backward pass.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import skiparse_synth as synth
from oracle import brute

TOK, GRP = oracle.TOKEN_WISE, oracle.GROUP_WISE


def iota(B, T, H, W):
    n = B * T * H * W
    assert n < 65535
    return (np.arange(n, dtype=np.uint16) + 1).reshape(B, T, H, W, 1, 1)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def padded_frames(x: np.ndarray, P: int) -> np.ndarray:
    """(B,T,H,W,...) -> (B,T,Lp,...) flattened frames zero-padded at their end to P^4."""
    B, T, H, W = x.shape[:4]
    k2 = P ** 4
    L = H * W
    Lp = -(-L // k2) * k2
    flat = x.reshape((B, T, L) + x.shape[4:])
    pad = [(0, 0), (0, 0), (0, Lp - L)] + [(0, 0)] * (x.ndim - 4)
    return np.pad(flat, pad)


# -------------------------------------------------------------------------------- geometry

def test_padded_length_brute_force():
    for L in range(1, 300, 7):
        for P in range(1, 4):
            k2 = P ** 4
            smallest = next(m for m in range(L, L + k2 + 1) if m % k2 == 0)
            assert oracle.padded_length_1d(L, P) == smallest


def test_index_map_is_a_bijection_onto_classes_times_positions():
    for P in (1, 2, 3):
        k = P * P
        Lp = 2 * k * k
        seen = set()
        for x in range(Lp):
            c, s = oracle.index_map_1d(x, P, TOK)
            assert c == x % k and 0 <= s < Lp // k
            seen.add((c, s))
        assert len(seen) == Lp
        seen = set()
        for x in range(Lp):
            c, s = oracle.index_map_1d(x, P, GRP)
            assert c == (x // k) % k and 0 <= s < Lp // k
            seen.add((c, s))
        assert len(seen) == Lp


def test_subsequence_length():
    for T, H, W, P in [(2, 8, 8, 2), (3, 10, 14, 2), (21, 45, 80, 2), (21, 30, 52, 2), (1, 5, 7, 1),
                       (2, 9, 9, 3)]:
        Lp = oracle.padded_length_1d(H * W, P)
        assert oracle.subseq_len(T, H, W, P, dims=1) * P * P == T * Lp


def test_720p_latent_needs_no_padding_and_480p_does():
    """The pages' 720P latent grid (45 x 80) holds 3600 = 225 * 16 tokens per frame, so the
    1D reading with P = 2 pads nothing; the 480P grid (30 x 52 = 1560) pads to 1568."""
    assert oracle.padded_length_1d(45 * 80, 2) == 3600
    assert oracle.padded_length_1d(30 * 52, 2) == 1568


# ------------------------------------------------------------------------------- rearrange

@pytest.mark.parametrize("B,T,H,W,P", [(1, 1, 4, 4, 2), (2, 3, 4, 8, 2), (1, 2, 5, 7, 2),
                                       (1, 2, 9, 9, 3), (2, 2, 3, 5, 1), (1, 2, 13, 17, 5),
                                       (1, 1, 30, 70, 8)])
def test_token_wise_is_strided_slicing(B, T, H, W, P):
    """A 1D token skip with ratio k: subsequence c is x[c::k] of each (padded) frame."""
    k = P * P
    x = iota(B, T, H, W)
    y, valid = oracle.rearrange(x, P, TOK, with_valid=True, dims=1)
    xf = padded_frames(x, P)[..., 0, 0]           # (B, T, Lp)
    for b in range(B):
        for c in range(k):
            want = xf[b, :, c::k].reshape(-1)      # frames in order, strided inside a frame
            assert np.array_equal(y[b * k + c, :, 0, 0], want)
            assert np.array_equal(valid[b * k + c], (want != 0).astype(np.uint8))


@pytest.mark.parametrize("B,T,H,W,P", [(1, 1, 4, 4, 2), (2, 2, 4, 8, 2), (1, 2, 5, 7, 2),
                                       (1, 1, 9, 9, 3), (1, 2, 2, 3, 1), (1, 2, 13, 17, 5),
                                       (1, 1, 30, 70, 8)])
def test_group_wise_is_group_reshape(B, T, H, W, P):
    """A 1D group skip with ratio k: cut each padded frame into runs of k consecutive tokens;
    run m goes to subsequence m mod k, runs kept whole and in order -- a reshape of the frame to
    (Lp/k^2, k, k) taking [:, c, :]."""
    k = P * P
    x = iota(B, T, H, W)
    y = oracle.rearrange(x, P, GRP, dims=1)
    xf = padded_frames(x, P)[..., 0, 0]
    Lp = xf.shape[2]
    for b in range(B):
        for c in range(k):
            want = xf[b].reshape(T, Lp // (k * k), k, k)[:, :, c, :].reshape(-1)
            assert np.array_equal(y[b * k + c, :, 0, 0], want)


@pytest.mark.parametrize("mode", [TOK, GRP])
@pytest.mark.parametrize("shape,P", [((2, 2, 5, 7, 3, 8), 2), ((1, 3, 9, 9, 2, 8), 3),
                                     ((1, 1, 1, 1, 1, 8), 2)])
def test_unrearrange_inverts_rearrange(mode, shape, P):
    x = synth.randn_bf16(shape, seed=11)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    y = oracle.rearrange(x, P, mode, dims=1)
    back = oracle.unrearrange(y, shape, P, mode, dims=1)
    assert np.array_equal(back, bits)
    # every row of y is either a row of x or a zero pad row
    assert (y.reshape(-1, shape[4] * shape[5]) == 0).all(axis=1).sum() == y.shape[0] * y.shape[1] - np.prod(shape[:4])


@pytest.mark.parametrize("src", [TOK, GRP])
@pytest.mark.parametrize("shape,P", [((2, 2, 5, 7, 2, 8), 2), ((1, 2, 9, 9, 1, 8), 3)])
def test_switch_is_unrearrange_then_rearrange(src, shape, P):
    x = synth.randn_bf16(shape, seed=12)
    ys = oracle.rearrange(x, P, src, dims=1)
    want = oracle.rearrange(oracle.unrearrange(ys, shape, P, src, dims=1).view(np.int16)
                            .view(np.uint16), P, 1 - src, dims=1)
    got = oracle.switch_mode(ys, shape, P, src, dims=1)
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.switch_mode(got, shape, P, 1 - src, dims=1), ys)


# ----------------------------------------------------------------------------------- forward

@pytest.mark.parametrize("shape", [(1, 2, 3, 5, 2, 16), (2, 1, 4, 4, 1, 32)])
def test_p1_is_dense_attention(shape):
    """P = 1: one class holding the whole sequence, which is plain full attention."""
    q, k, v = (synth.randn_bf16(shape, seed=s) for s in (1, 2, 3))
    got = oracle.attn_fwd(q, k, v, 1, TOK, dims=1)
    B, T, H, W, heads, d = shape
    flat = lambda a: torch.from_numpy(to_f64(a)).reshape(B, T * H * W, heads, d).transpose(1, 2)
    ref = F.scaled_dot_product_attention(flat(q), flat(k), flat(v))
    want = ref.transpose(1, 2).reshape(shape).numpy()
    assert np.max(np.abs(got - want)) < 1e-12


@pytest.mark.parametrize("mode", [TOK, GRP])
@pytest.mark.parametrize("shape,P", [((1, 2, 4, 4, 2, 8), 2), ((2, 2, 3, 7, 1, 16), 2),
                                     ((1, 1, 9, 10, 1, 8), 3), ((1, 2, 1, 3, 2, 8), 2),
                                     ((1, 1, 13, 17, 1, 8), 5), ((1, 1, 30, 70, 1, 4), 8)])
def test_forward_matches_brute_force_mask(mode, shape, P):
    q, k, v = (synth.randn_bf16(shape, seed=s) for s in (21, 22, 23))
    got = oracle.attn_fwd(q, k, v, P, mode, dims=1)
    want = brute.attention_1d(to_f64(q), to_f64(k), to_f64(v), P, mode)
    assert np.max(np.abs(got - want)) < 1e-12


def column_closed_form(q, k, v, key_class):
    """Attention where query (t, h, w) sees every real key (t', h', w') with
    key_class(w') == key_class(w)."""
    B, T, H, W, heads, d = q.shape
    out = np.zeros_like(q)
    cols = np.array([key_class(w) for w in range(W)])
    for w in range(W):
        same = np.nonzero(cols == cols[w])[0]
        K = k[:, :, :, same]                      # (B, T, H, ncol, heads, d)
        V = v[:, :, :, same]
        for b in range(B):
            for hd in range(heads):
                Kb = K[b, ..., hd, :].reshape(-1, d)
                Vb = V[b, ..., hd, :].reshape(-1, d)
                Q = q[b, :, :, w, hd, :].reshape(-1, d)
                S = Q @ Kb.T / np.sqrt(d)
                S -= S.max(axis=1, keepdims=True)
                A = np.exp(S)
                A /= A.sum(axis=1, keepdims=True)
                out[b, :, :, w, hd, :] = (A @ Vb).reshape(T, H, d)
    return out


def test_token_wise_with_width_multiple_of_ratio_is_column_stripes():
    """W a multiple of P^2: (h*W + w) mod P^2 = w mod P^2, so each class is the columns
    w = c (mod P^2) of every row and frame."""
    P, shape = 2, (1, 2, 3, 8, 2, 8)
    q, k, v = (synth.randn_bf16(shape, seed=s) for s in (31, 32, 33))
    got = oracle.attn_fwd(q, k, v, P, TOK, dims=1)
    want = column_closed_form(to_f64(q), to_f64(k), to_f64(v), lambda w: w % (P * P))
    assert np.max(np.abs(got - want)) < 1e-12


def test_group_wise_with_width_multiple_of_ratio_squared_is_column_blocks():
    """W a multiple of P^4: ((h*W + w) div P^2) mod P^2 = (w div P^2) mod P^2, so each class is
    a set of P^2-wide column blocks of every row and frame; no padding."""
    P, shape = 2, (1, 2, 3, 16, 1, 8)
    q, k, v = (synth.randn_bf16(shape, seed=s) for s in (41, 42, 43))
    got = oracle.attn_fwd(q, k, v, P, GRP, dims=1)
    want = column_closed_form(to_f64(q), to_f64(k), to_f64(v), lambda w: (w // (P * P)) % (P * P))
    assert np.max(np.abs(got - want)) < 1e-12


def test_rows_equal_full_forward():
    shape, P = (2, 2, 5, 7, 2, 16), 2
    q, k, v = (synth.randn_bf16(shape, seed=s) for s in (51, 52, 53))
    for mode in (TOK, GRP):
        full = oracle.attn_fwd(q, k, v, P, mode, dims=1).reshape(-1, shape[-1])
        rows = np.array([0, 5, 17, 69, full.shape[0] - 1])
        got = oracle.attn_fwd_rows(q, k, v, rows, P, mode, dims=1)
        assert np.array_equal(got, full[rows])


def test_one_token_frame_attends_to_itself_class():
    """H = W = 1 with P = 2: every frame's single token is class 0 in both modes, so each token
    attends over all T frames' tokens (P = 1 result)."""
    shape = (1, 3, 1, 1, 1, 8)
    q, k, v = (synth.randn_bf16(shape, seed=s) for s in (61, 62, 63))
    for mode in (TOK, GRP):
        got = oracle.attn_fwd(q, k, v, 2, mode, dims=1)
        want = oracle.attn_fwd(q, k, v, 1, mode, dims=1)
        assert np.max(np.abs(got - want)) < 1e-12


# ---------------------------------------------------------------------------------- backward

@pytest.mark.parametrize("mode", [TOK, GRP])
@pytest.mark.parametrize("shape,P", [((1, 2, 3, 5, 2, 8), 2), ((1, 1, 9, 9, 1, 8), 3)])
def test_backward_matches_autograd(mode, shape, P):
    q, k, v, g = (synth.randn_bf16(shape, seed=s) for s in (71, 72, 73, 74))
    dq, dk, dv, lse = oracle.attn_bwd(q, k, v, g, P, mode, dims=1)
    qt, kt, vt = (a.to(torch.float64).requires_grad_(True) for a in (q, k, v))
    out, lse_ref = brute.attention_1d_torch(qt, kt, vt, P, mode)
    out.backward(g.to(torch.float64))
    for got, want in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad), (lse, lse_ref.detach())):
        assert np.max(np.abs(got - want.numpy())) < 1e-11


def test_backward_rows_equal_full():
    shape, P = (1, 2, 5, 7, 2, 8), 2
    q, k, v, g = (synth.randn_bf16(shape, seed=s) for s in (81, 82, 83, 84))
    for mode in (TOK, GRP):
        dq, dk, dv, _ = oracle.attn_bwd(q, k, v, g, P, mode, dims=1)
        rows = np.array([0, 3, 29, 69])
        rq, rk, rv = oracle.attn_bwd_rows(q, k, v, g, rows, P, mode, dims=1)
        d = shape[-1]
        for got, full in ((rq, dq), (rk, dk), (rv, dv)):
            assert np.max(np.abs(got - full.reshape(-1, d)[rows])) < 1e-12
