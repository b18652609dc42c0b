"""Pins for the backward-pass oracle: torch autograd through an independent dense masked fp64
attention (oracle/brute.py's definition, differentiated by the library), autograd of fp64
scaled_dot_product_attention at P = 1, and the sampled-rows entry against the full one."""

from __future__ import annotations

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import skiparse_synth as synth
from oracle import brute

TOK, GRP = oracle.TOKEN_WISE, oracle.GROUP_WISE

CASES = [synth.WORKLOADS["tiny"], synth.WORKLOADS["anyres"], synth.custom(2, 2, 5, 7, 2, 8, 3),
         synth.custom(1, 1, 3, 17, 1, 4, 4), synth.custom(1, 2, 6, 6, 2, 16, 1),
         synth.custom(1, 1, 26, 31, 1, 8, 5), synth.custom(1, 1, 9, 11, 1, 4, 8)]


def grads_by_autograd(q, k, v, dout, P, mode):
    qt, kt, vt = (t.to(torch.float64).requires_grad_(True) for t in (q, k, v))
    out, lse = brute.attention_torch(qt, kt, vt, P, mode)
    (out * dout.to(torch.float64)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy(), lse.detach().numpy()


@pytest.mark.parametrize("w", CASES, ids=lambda w: f"{w.name}_P{w.P}_H{w.H}W{w.W}")
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_backward_equals_autograd_of_masked_dense_attention(w, mode):
    q, k, v = synth.qkv(w)
    dout = synth.randn_bf16(w.shape, 900 + w.family)
    dq, dk, dv, lse = oracle.attn_bwd(q, k, v, dout, w.P, mode)
    gq, gk, gv, glse = grads_by_autograd(q, k, v, dout, w.P, mode)
    for got, want in ((dq, gq), (dk, gk), (dv, gv), (lse, glse)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


def test_backward_p1_equals_sdpa_autograd():
    B, T, H, W, heads, d = 1, 2, 4, 5, 2, 16
    q, k, v = (synth.randn_bf16((B, T, H, W, heads, d), 950 + i) for i in range(3))
    dout = synth.randn_bf16((B, T, H, W, heads, d), 960)
    dq, dk, dv, _ = oracle.attn_bwd(q, k, v, dout, 1, TOK)
    N = T * H * W
    qt, kt, vt = (a.double().reshape(N, heads, d).permute(1, 0, 2).requires_grad_(True) for a in (q, k, v))
    o = F.scaled_dot_product_attention(qt, kt, vt)
    (o * dout.double().reshape(N, heads, d).permute(1, 0, 2)).sum().backward()
    for got, g in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        want = g.permute(1, 0, 2).reshape(B, T, H, W, heads, d).numpy()
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


@pytest.mark.parametrize("mode", [TOK, GRP])
def test_backward_rows_equal_full(mode):
    w = synth.custom(1, 2, 10, 14, 3, 32, 2, "rows")
    q, k, v = synth.qkv(w)
    dout = synth.randn_bf16(w.shape, 970)
    dq, dk, dv, _ = oracle.attn_bwd(q, k, v, dout, w.P, mode)
    rows = np.array([0, 7, 19, 100, 333, w.B * w.T * w.H * w.W * w.heads - 1])
    rq, rk, rv = oracle.attn_bwd_rows(q, k, v, dout, rows, w.P, mode)
    np.testing.assert_allclose(rq, dq.reshape(-1, w.d)[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(rk, dk.reshape(-1, w.d)[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(rv, dv.reshape(-1, w.d)[rows], rtol=0, atol=1e-12)


def test_backward_lse_matches_forward_normaliser():
    """exp(q.k/sqrt(d) - lse) summed over the class is 1: checked through the forward oracle
    with V = ones, whose output is then exactly the sum of the weights."""
    w = synth.WORKLOADS["anyres"]
    q, k, _ = synth.qkv(w)
    ones = torch.ones(w.shape, dtype=torch.bfloat16)
    out = oracle.attn_fwd(q, k, ones, w.P, TOK)
    np.testing.assert_allclose(out, 1.0, atol=1e-12)
    _, _, _, lse = oracle.attn_bwd(q, k, ones, ones, w.P, TOK)
    assert np.all(np.isfinite(lse))
