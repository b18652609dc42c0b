"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test names what fixes the expected answer: a value the pages fix (golden files
under tests/golden/, each cited), a library routine the pages liken the method to
(pixel unshuffle), textbook attention (fp64 scaled_dot_product_attention), an
independent brute force with an explicit 2-D mask, closed forms, or an invariant the
pages state (inverse rearrange, local equivalence, two-hop interaction).
"""

from __future__ import annotations

import itertools
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import skiparse_synth as synth
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOK, GRP = oracle.TOKEN_WISE, oracle.GROUP_WISE


# ----------------------------------------------------------------------------- helpers

def parse_class_maps():
    grids = []
    cur = None
    section = None
    with open(os.path.join(GOLDEN, "class_maps.txt")) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("grid"):
                _, Hp, Wp, P, mode = line.split()
                cur = dict(Hp=int(Hp), Wp=int(Wp), P=int(P), mode=TOK if mode == "token" else GRP,
                           cls=[], sub_r=None, sub_s=None)
                grids.append(cur)
                section = None
            elif line in ("class", "sub_r", "sub_s"):
                section = line
            elif section == "class":
                cur["cls"].append([int(v) for v in line.split()])
            else:
                cur[section] = [int(v) for v in line.split()]
    return grids


def iota_tokens(B, T, H, W):
    """A (B,T,H,W,1,1) uint16 tensor whose entry is 1 + the flat token index."""
    n = B * T * H * W
    assert n < 65535
    return (np.arange(n, dtype=np.uint16) + 1).reshape(B, T, H, W, 1, 1)


def random_bits(shape, seed):
    """Arbitrary 16-bit patterns of finite bf16 values (bit-exact tests)."""
    return synth.randn_bf16(shape, seed)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


# ------------------------------------------------------------------- geometry pins

def test_padding_golden():
    """方法步骤详情: pad to the nearest multiple of P^2; 实验结果: 720P pads, 768P does not."""
    with open(os.path.join(GOLDEN, "padding.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert rows
    for X, P, Xp, needs in rows:
        assert oracle.padded_extent(int(X), int(P)) == int(Xp)
        assert (int(Xp) != int(X)) == bool(int(needs))


def test_padding_brute_force():
    for X in range(1, 60):
        for P in range(1, 5):
            smallest = next(m for m in range(X, X + P * P + 1) if m % (P * P) == 0)
            assert oracle.padded_extent(X, P) == smallest


def test_subsequence_length_is_n_over_p2():
    """方法步骤详情: each of the P^2 subsequences has 1/P^2 of the (padded) length."""
    for T, H, W, P in [(2, 8, 8, 2), (3, 10, 14, 2), (21, 45, 80, 2), (21, 48, 84, 3), (1, 5, 7, 1)]:
        Hp, Wp = oracle.padded_extent(H, P), oracle.padded_extent(W, P)
        assert oracle.subseq_len(T, H, W, P) * P * P == T * Hp * Wp


def test_class_maps_golden():
    grids = parse_class_maps()
    assert len(grids) == 5
    for g in grids:
        P, mode = g["P"], g["mode"]
        for h in range(g["Hp"]):
            for w in range(g["Wp"]):
                ci, r = oracle.axis_map(h, P, mode)
                cj, s = oracle.axis_map(w, P, mode)
                assert ci * P + cj == g["cls"][h][w], (g["Hp"], P, mode, h, w)
                assert r == g["sub_r"][h] and s == g["sub_s"][w]
        # and the rearrange places every token exactly where the golden map says
        x = iota_tokens(1, 1, g["Hp"], g["Wp"])
        y = oracle.rearrange(x, P, mode)
        S = g["Wp"] // P
        for h in range(g["Hp"]):
            for w in range(g["Wp"]):
                c = g["cls"][h][w]
                pos = g["sub_r"][h] * S + g["sub_s"][w]
                assert y[c, pos, 0, 0] == h * g["Wp"] + w + 1


@pytest.mark.parametrize("T,Hp,Wp,P,C", [(1, 4, 4, 2, 3), (2, 8, 12, 2, 5), (2, 9, 18, 3, 2),
                                         (1, 16, 16, 4, 1), (3, 6, 5, 1, 2), (1, 25, 50, 5, 1),
                                         (1, 64, 64, 8, 1)])
def test_token_wise_is_pixel_unshuffle(T, Hp, Wp, P, C):
    """核心方法: token-wise rearrange is pixel unshuffle (torch's library routine)."""
    x = torch.randint(0, 60000, (1, T, Hp, Wp, 1, C), dtype=torch.int32)
    y = oracle.rearrange(x.to(torch.int16).numpy().view(np.uint16), P, TOK)
    pu = F.pixel_unshuffle(x[0, :, :, :, 0, :].permute(0, 3, 1, 2).double(), P)  # (T, C*P^2, R, S)
    R, S = Hp // P, Wp // P
    pu = pu.reshape(T, C, P * P, R, S).permute(2, 0, 3, 4, 1).reshape(P * P, T * R * S, C)
    got = torch.from_numpy(y[:, :, 0, :].view(np.int16).astype(np.int64))
    want = pu.to(torch.int64).to(torch.int16).to(torch.int64)
    assert torch.equal(got, want)


@pytest.mark.parametrize("T,Hp,Wp,P,C", [(1, 4, 4, 2, 3), (2, 8, 12, 2, 2), (1, 9, 18, 3, 2),
                                         (1, 16, 32, 4, 1), (1, 25, 50, 5, 1), (1, 64, 128, 8, 1)])
def test_group_wise_is_patch_unshuffle(T, Hp, Wp, P, C):
    """核心方法: group-wise is patch unshuffle: fold each P x P patch into channels
    (pixel_unshuffle), distribute the patch grid the pixel-unshuffle way
    (pixel_unshuffle again), then unfold the patch back into space (pixel_shuffle)."""
    x = torch.randint(0, 60000, (1, T, Hp, Wp, 1, C), dtype=torch.int32)
    y = oracle.rearrange(x.to(torch.int16).numpy().view(np.uint16), P, GRP)
    img = x[0, :, :, :, 0, :].permute(0, 3, 1, 2).double()                # (T, C, Hp, Wp)
    patches = F.pixel_unshuffle(img, P)                                     # (T, C*P^2, Hp/P, Wp/P)
    classes = F.pixel_unshuffle(patches, P)                                 # (T, C*P^4, Hp/P^2, Wp/P^2)
    q = P * P
    classes = classes.reshape(T, C * q, q, Hp // q, Wp // q)               # [.., (c,ph,pw), class, hb, wb]
    R, S = Hp // P, Wp // P
    for cls in range(q):
        sub = F.pixel_shuffle(classes[:, :, cls], P)                        # (T, C, R, S)
        want = sub.permute(0, 2, 3, 1).reshape(T * R * S, C).to(torch.int64).to(torch.int16)
        got = torch.from_numpy(y[cls, :, 0, :].view(np.int16).copy())
        assert torch.equal(got, want), cls


# ------------------------------------------------------------------ rearrange pins

SHAPES = [(1, 2, 8, 8, 2, 4, 2), (2, 3, 10, 14, 1, 8, 2), (1, 2, 5, 7, 3, 2, 3),
          (1, 1, 3, 20, 1, 2, 4), (2, 2, 6, 5, 2, 2, 1), (1, 1, 1, 1, 1, 1, 2)]


@pytest.mark.parametrize("B,T,H,W,heads,d,P", SHAPES)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_rearrange_is_a_permutation_with_zero_pads(B, T, H, W, heads, d, P, mode):
    x = iota_tokens(B, T, H, W)
    y, valid = oracle.rearrange(x, P, mode, with_valid=True)
    flat = y[:, :, 0, 0].reshape(-1)
    assert np.array_equal(np.sort(flat[flat > 0]), np.arange(1, B * T * H * W + 1))
    assert np.all((flat > 0) == (valid.reshape(-1) == 1))
    # every subsequence holds only its own batch's tokens
    q = P * P
    for seq in range(B * q):
        toks = y[seq, :, 0, 0]
        toks = toks[toks > 0].astype(np.int64) - 1
        assert np.all(toks // (T * H * W) == seq // q)


@pytest.mark.parametrize("B,T,H,W,heads,d,P", SHAPES)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_unrearrange_inverts_rearrange(B, T, H, W, heads, d, P, mode):
    """方法步骤详情: the result is rearranged back to the original layout."""
    x = random_bits((B, T, H, W, heads, d), 7 + P + mode)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    y = oracle.rearrange(x, P, mode)
    assert np.array_equal(oracle.unrearrange(y, x.shape, P, mode), xb)
    # the other way round holds on inputs whose pad slots are zero
    y2 = oracle.rearrange(oracle.unrearrange(y, x.shape, P, mode), P, mode)
    assert np.array_equal(y2, y)


@pytest.mark.parametrize("P", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_local_equivalence(P, mode):
    """核心方法: rearranging the whole sequence equals rearranging each minimal repeating
    unit (a P^2 x P^2 tile of one frame) on its own; the tile (hb, wb) lands as the P x P
    block at sub-grid rows hb*P.., columns wb*P.. of each class."""
    q = P * P
    T, H, W, heads, d = 2, 2 * q + 1, 3 * q - 1, 1, 3
    x = random_bits((1, T, H, W, heads, d), 100 + P)
    Hp, Wp = oracle.padded_extent(H, P), oracle.padded_extent(W, P)
    xp = torch.zeros((1, T, Hp, Wp, heads, d), dtype=torch.bfloat16)
    xp[:, :, :H, :W] = x
    whole = oracle.rearrange(x, P, mode)
    R, S = Hp // P, Wp // P
    whole = whole.reshape(q, T, R, S, heads, d)
    for t in range(T):
        for hb in range(Hp // q):
            for wb in range(Wp // q):
                tile = xp[:, t:t + 1, hb * q:(hb + 1) * q, wb * q:(wb + 1) * q]
                local = oracle.rearrange(tile, P, mode).reshape(q, P, P, heads, d)
                block = whole[:, t, hb * P:(hb + 1) * P, wb * P:(wb + 1) * P]
                assert np.array_equal(local, block)


def class_membership(H, W, P, mode):
    """Class of each real (h, w), read off the oracle's rearrange of an index tensor."""
    y = oracle.rearrange(iota_tokens(1, 1, H, W), P, mode)
    cls = np.empty(H * W, dtype=np.int64)
    for c in range(P * P):
        toks = y[c, :, 0, 0]
        cls[toks[toks > 0].astype(np.int64) - 1] = c
    return cls


@pytest.mark.parametrize("P,H,W", [(2, 8, 8), (2, 12, 16), (3, 9, 18), (2, 5, 7), (4, 16, 32),
                                   (5, 25, 25)])
def test_two_hop_interaction(P, H, W):
    """核心方法: with the two modes alternating, any two tokens interact within at most
    two attention operations (token-wise then group-wise, and the other way round)."""
    tok = class_membership(H, W, P, TOK)
    grp = class_membership(H, W, P, GRP)
    Hp, Wp = oracle.padded_extent(H, P), oracle.padded_extent(W, P)
    if (Hp, Wp) != (H, W):
        pytest.skip("two-hop is a statement about full P^2 x P^2 tiles")
    n = H * W
    same_tok = tok[:, None] == tok[None, :]
    same_grp = grp[:, None] == grp[None, :]
    # b -> c in a token-wise layer, c -> a in a group-wise layer
    reach_tg = (same_grp.astype(np.int64) @ same_tok.astype(np.int64)) > 0
    reach_gt = (same_tok.astype(np.int64) @ same_grp.astype(np.int64)) > 0
    assert reach_tg.all() and reach_gt.all()
    # and one layer alone is not enough (the pattern really is sparse)
    if P > 1:
        assert not same_tok.all() and not same_grp.all()
    assert same_tok.sum() == n * n // (P * P) and same_grp.sum() == n * n // (P * P)


# ------------------------------------------------------------------ attention pins

@pytest.mark.parametrize("T,H,W,heads,d", [(2, 5, 6, 2, 16), (1, 7, 3, 3, 32), (2, 4, 4, 1, 8)])
def test_p1_is_full_attention(T, H, W, heads, d):
    """P = 1 is the dense baseline (实验结果 compares Skiparse with full attention):
    it must equal textbook softmax(Q K^T / sqrt(d)) V, here torch's fp64 SDPA."""
    q, k, v = (synth.randn_bf16((1, T, H, W, heads, d), 300 + i) for i in range(3))
    got = oracle.attn_fwd(q, k, v, P=1, mode=TOK)
    for mode in (TOK, GRP):  # P = 1 makes the two modes identical
        assert np.array_equal(oracle.attn_fwd(q, k, v, P=1, mode=mode), got)
    N = T * H * W
    Q, K, V = (a.double().reshape(N, heads, d).permute(1, 0, 2) for a in (q, k, v))
    want = F.scaled_dot_product_attention(Q, K, V).permute(1, 0, 2).reshape(1, T, H, W, heads, d)
    np.testing.assert_allclose(got, want.numpy(), rtol=0, atol=1e-12)


BRUTE_CASES = [synth.WORKLOADS["tiny"], synth.WORKLOADS["anyres"],
               synth.custom(2, 2, 5, 7, 2, 8, 3), synth.custom(1, 1, 3, 17, 1, 4, 4),
               synth.custom(1, 2, 6, 6, 2, 16, 1), synth.custom(1, 1, 26, 31, 1, 8, 5),
               synth.custom(1, 1, 20, 23, 1, 4, 8)]


@pytest.mark.parametrize("w", BRUTE_CASES, ids=lambda w: w.name + f"_P{w.P}_H{w.H}W{w.W}")
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_oracle_equals_brute_force(w, mode):
    """Independent brute force: one dense attention over the padded grid with an explicit
    same-class and real-key 2-D mask."""
    q, k, v = synth.qkv(w)
    got = oracle.attn_fwd(q, k, v, w.P, mode)
    want = brute.attention(to_f64(q), to_f64(k), to_f64(v), w.P, mode)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", [TOK, GRP])
def test_constant_values_give_constant_output(mode):
    w = synth.WORKLOADS["anyres"]
    q, k, _ = synth.qkv(w)
    per_head = torch.linspace(-2, 3, w.heads * w.d).reshape(w.heads, w.d).to(torch.bfloat16)
    v = per_head.expand(w.shape).contiguous()
    got = oracle.attn_fwd(q, k, v, w.P, mode)
    np.testing.assert_allclose(got, np.broadcast_to(to_f64(per_head), got.shape), atol=1e-12, rtol=0)


@pytest.mark.parametrize("mode", [TOK, GRP])
def test_zero_query_gives_class_mean(mode):
    """Q = 0 makes every score equal, so each output is the mean of V over the real keys
    of the query's class (class rule taken from the brute force's own restatement)."""
    w = synth.WORKLOADS["anyres"]
    _, k, v = synth.qkv(w)
    q = torch.zeros(w.shape, dtype=torch.bfloat16)
    got = oracle.attn_fwd(q, k, v, w.P, mode)
    Hp, Wp = oracle.padded_extent(w.H, w.P), oracle.padded_extent(w.W, w.P)
    cls = brute.class_grid(Hp, Wp, w.P, mode)[: w.H, : w.W]
    vf = to_f64(v)
    for c in range(w.P * w.P):
        sel = cls == c
        mean = vf[:, :, sel].mean(axis=(1, 2))  # over t and the class's (h, w)
        np.testing.assert_allclose(got[:, :, sel], np.broadcast_to(mean[:, None, None], got[:, :, sel].shape),
                                   atol=1e-12, rtol=0)


def test_single_token_classes_copy_v():
    """A class holding one real token attends only to itself: output = V."""
    q, k, v = (synth.randn_bf16((1, 1, 2, 2, 3, 8), 400 + i) for i in range(3))
    got = oracle.attn_fwd(q, k, v, P=2, mode=TOK)  # each of the 4 classes has 1 real token
    np.testing.assert_array_equal(got, to_f64(v))
    q, k, v = (synth.randn_bf16((1, 1, 1, 1, 2, 8), 410 + i) for i in range(3))
    for mode in (TOK, GRP):
        np.testing.assert_array_equal(oracle.attn_fwd(q, k, v, P=3, mode=mode), to_f64(v))


@pytest.mark.parametrize("mode", [TOK, GRP])
def test_pad_slot_values_and_extra_padding_do_not_matter(mode):
    w = synth.WORKLOADS["anyres"]
    q, k, v = synth.qkv(w)
    (yq, valid), yk, yv = oracle.rearrange(q, w.P, mode, True), oracle.rearrange(k, w.P, mode), \
        oracle.rearrange(v, w.P, mode)
    base = oracle.masked_attention(yq, yk, yv, valid)
    rng = np.random.default_rng(5)
    junk = [a.copy() for a in (yq, yk, yv)]
    for a in junk:
        pads = valid == 0
        a[pads] = rng.integers(0x3F00, 0x4100, size=a[pads].shape, dtype=np.uint16)  # |x| in [0.5, 8)
    again = oracle.masked_attention(*junk, valid)
    np.testing.assert_array_equal(again[valid == 1], base[valid == 1])
    # enlarge the padding: append 37 more pad slots of garbage to every subsequence
    extra = 37
    big = [np.concatenate([a, rng.integers(0x3F00, 0x4100, size=(a.shape[0], extra) + a.shape[2:],
                                           dtype=np.uint16)], axis=1) for a in (yq, yk, yv)]
    bigvalid = np.concatenate([valid, np.zeros((valid.shape[0], extra), np.uint8)], axis=1)
    bigout = oracle.masked_attention(*big, bigvalid)
    np.testing.assert_array_equal(bigout[:, : valid.shape[1]][valid == 1], base[valid == 1])


@pytest.mark.parametrize("mode", [TOK, GRP])
def test_sampled_rows_equal_full_output(mode):
    w = synth.WORKLOADS["anyres"]
    q, k, v = synth.qkv(w)
    full = oracle.attn_fwd(q, k, v, w.P, mode).reshape(-1, w.d)
    rows = np.array([0, 5, 17, 100, full.shape[0] - 1, 333, 1234 % full.shape[0]])
    np.testing.assert_array_equal(oracle.attn_fwd_rows(q, k, v, rows, w.P, mode), full[rows])


def test_modes_differ_and_threads_do_not_matter():
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.qkv(w)
    a = oracle.attn_fwd(q, k, v, w.P, TOK, nthreads=1)
    b = oracle.attn_fwd(q, k, v, w.P, GRP, nthreads=1)
    assert np.abs(a - b).max() > 1e-3
    np.testing.assert_array_equal(oracle.attn_fwd(q, k, v, w.P, TOK, nthreads=3), a)


def test_bad_arguments_are_rejected():
    L = oracle.lib()
    assert L.oracle_padded_extent(0, 2) < 0 and L.oracle_padded_extent(4, 0) < 0
    with pytest.raises(RuntimeError):
        oracle.axis_map(3, 2, 7)


# --------------------------------------------------------------- pattern-switch pins

@pytest.mark.parametrize("B,T,H,W,heads,d,P", SHAPES)
@pytest.mark.parametrize("src", [TOK, GRP])
def test_switch_mode_is_unrearrange_then_rearrange(B, T, H, W, heads, d, P, src):
    """核心方法: the two modes alternate between layers; the switch of one tensor between the
    modes' layouts is the inverse rearrange of one followed by the rearrange of the other."""
    x = random_bits((B, T, H, W, heads, d), 500 + P + src)
    ysrc = oracle.rearrange(x, P, src)
    got = oracle.switch_mode(ysrc, x.shape, P, src)
    want = oracle.rearrange(oracle.unrearrange(ysrc, x.shape, P, src), P, 1 - src)
    assert np.array_equal(got, want)
    # and back again gives the source layout (its pad slots are zero already)
    assert np.array_equal(oracle.switch_mode(got, x.shape, P, 1 - src), ysrc)


def test_switch_mode_ignores_source_pad_slots():
    w = synth.WORKLOADS["anyres"]
    x, _, _ = synth.qkv(w)
    y, valid = oracle.rearrange(x, w.P, TOK, with_valid=True)
    junk = y.copy()
    junk[valid == 0] = 0x4000
    a = oracle.switch_mode(y, w.shape, w.P, TOK)
    b = oracle.switch_mode(junk, w.shape, w.P, TOK)
    assert np.array_equal(a, b)
    _, gvalid = oracle.rearrange(x, w.P, GRP, with_valid=True)
    assert np.all(a[gvalid == 0] == 0)
