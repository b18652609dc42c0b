"""GPU parity of the backward pass (through the C ABI) against the fp64 CPU oracle.

Tolerance (derived in the design notes from the arithmetic): the kernels round P and dS to
bf16 before their tensor-core products and round the gradients to bf16 once; relative to the
largest gradient entry that gives errors of a few bf16 half-ulps (2^-9). We require
max|err| <= 2e-2 * max|ref| and mean|err| <= 2e-3 * max|ref| for each of dq, dk, dv (max|ref|
floored at 1e-3 for gradients that are exactly zero), and the forward's lse within 1e-3.
Full-size shapes are checked on sampled rows of one (class, head) subsequence, the last class
and head (ragged in the padded workloads)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import skiparse_synth as synth
from parity_helpers import sample_rows_one_class

pytestmark = pytest.mark.gpu
TOK, GRP = 0, 1


@pytest.fixture(scope="module")
def fps():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as m
    return m


def check_grad(got, want, what):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    scale = max(np.abs(want).max(), 1e-3)  # exact zeros (e.g. a single-token class's dq) need a floor
    err = np.abs(got - want)
    print(f"{what}: max|err|/max|ref| = {err.max() / scale:.3e}, mean|err|/max|ref| = {err.mean() / scale:.3e}")
    assert err.max() <= 2e-2 * scale and err.mean() <= 2e-3 * scale, what


SMALL = [synth.WORKLOADS["tiny"], synth.WORKLOADS["anyres"], synth.custom(2, 3, 13, 22, 3, 64, 2, "b2_ragged"),
         synth.custom(1, 2, 20, 30, 2, 128, 3, "p3_unequal"), synth.custom(1, 5, 16, 16, 2, 128, 1, "dense_p1"),
         synth.custom(1, 6, 24, 40, 2, 128, 2, "multi_tile"), synth.custom(1, 1, 1, 1, 1, 64, 2, "one_token"),
         synth.custom(1, 2, 26, 31, 1, 64, 5, "p5"), synth.custom(1, 1, 70, 65, 1, 32, 8, "p8")]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_backward_small_full(fps, w, mode):
    q, k, v = synth.qkv(w)
    dout = synth.randn_bf16(w.shape, 900 + w.family)
    dq_ref, dk_ref, dv_ref, lse_ref = oracle.attn_bwd(q, k, v, dout, w.P, mode)
    qd, kd, vd, gd = (t.cuda() for t in (q, k, v, dout))
    out, lse = fps.skiparse2d_attn_fwd_lse(qd, kd, vd, w.P, mode)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    fps.skiparse2d_attn_bwd(qd, kd, vd, out, gd, lse, w.P, mode, dq=dq, dk=dk, dv=dv)
    assert fps.get_device_status() == 0
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=0, atol=1e-3)
    check_grad(dq.double().cpu().numpy(), dq_ref, f"{w.name} dq")
    check_grad(dk.double().cpu().numpy(), dk_ref, f"{w.name} dk")
    check_grad(dv.double().cpu().numpy(), dv_ref, f"{w.name} dv")


@pytest.mark.parametrize("name,mode", [("480p", TOK), ("480p", GRP), ("720p", GRP)])
def test_backward_full_size_sampled(fps, name, mode):
    w = synth.WORKLOADS[name]
    q, k, v = synth.qkv(w)
    dout = synth.randn_bf16(w.shape, 900 + w.family)
    qd, kd, vd, gd = (t.cuda() for t in (q, k, v, dout))
    out, lse = fps.skiparse2d_attn_fwd_lse(qd, kd, vd, w.P, mode)
    dq, dk, dv = fps.skiparse2d_attn_bwd(qd, kd, vd, out, gd, lse, w.P, mode)
    assert fps.get_device_status() == 0
    rows = sample_rows_one_class(w, mode, 24, cls=w.P * w.P - 1, head=w.heads - 1, seed=w.family)
    rq, rk, rv = oracle.attn_bwd_rows(q, k, v, dout, rows, w.P, mode)
    idx = torch.from_numpy(rows).cuda()
    for got, want, what in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(got.reshape(-1, w.d).index_select(0, idx).double().cpu().numpy(), want, f"{name} {what}")


def test_autograd_function_matches_oracle(fps):
    w = synth.WORKLOADS["anyres"]
    q, k, v = synth.qkv(w)
    dout = synth.randn_bf16(w.shape, 990)
    qd, kd, vd = (t.cuda().requires_grad_(True) for t in (q, k, v))
    out = fps.skiparse_attention(qd, kd, vd, w.P, GRP)
    out.backward(dout.cuda())
    dq_ref, dk_ref, dv_ref, _ = oracle.attn_bwd(q, k, v, dout, w.P, GRP)
    check_grad(qd.grad.double().cpu().numpy(), dq_ref, "autograd dq")
    check_grad(kd.grad.double().cpu().numpy(), dk_ref, "autograd dk")
    check_grad(vd.grad.double().cpu().numpy(), dv_ref, "autograd dv")


def test_backward_is_deterministic(fps):
    w = synth.custom(1, 4, 12, 20, 2, 128, 2, "det")
    qd, kd, vd = (t.cuda() for t in synth.qkv(w))
    gd = synth.randn_bf16(w.shape, 991).cuda()
    out, lse = fps.skiparse2d_attn_fwd_lse(qd, kd, vd, w.P, TOK)
    a = fps.skiparse2d_attn_bwd(qd, kd, vd, out, gd, lse, w.P, TOK)
    b = fps.skiparse2d_attn_bwd(qd, kd, vd, out, gd, lse, w.P, TOK)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
