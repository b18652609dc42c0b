"""GPU parity of Skiparse-1D (the flattened-sequence variant) against the fp64 CPU oracle,
through the C ABI: rearrange, inverse and switch bit-exact; the forward within
max|err| <= 1e-2, mean|err| <= 1e-3; the backward within the tolerances of
test_gpu_backward.py. Small shapes element by element, full-size latents on sampled rows."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import skiparse_synth as synth
from parity_helpers import check_close, gpu_rows, sample_rows, sample_rows_one_class_1d
from test_gpu_backward import check_grad

pytestmark = pytest.mark.gpu

TOK, GRP = 0, 1


@pytest.fixture(scope="module")
def fps():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as m
    return m


SMALL = [
    synth.WORKLOADS["tiny"],                                   # L = 64: no padding
    synth.WORKLOADS["anyres"],                                 # L = 140 -> 144
    synth.custom(2, 3, 13, 22, 3, 64, 2, "b2_ragged"),         # L = 286 -> 288, B = 2
    synth.custom(1, 2, 20, 30, 2, 128, 3, "p3"),               # 9 classes, L = 600 -> 648
    synth.custom(1, 5, 16, 16, 2, 128, 1, "dense_p1"),         # P = 1: dense
    synth.custom(1, 3, 17, 19, 1, 32, 4, "p4"),                # 16 classes, L = 323 -> 512
    synth.custom(1, 2, 8, 9, 1, 32, 8, "p8"),                  # 64 classes, L = 72 -> 4096
    synth.custom(1, 1, 1, 1, 1, 64, 2, "one_token"),
    synth.custom(1, 6, 24, 40, 2, 128, 2, "multi_tile"),       # n_c = 1440: 12 tiles
]


def _dev(ts):
    return [t.cuda() for t in ts]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_attention_1d_small_full(fps, w, mode):
    q, k, v = synth.qkv(w)
    want = oracle.attn_fwd(q, k, v, w.P, mode, dims=1)
    qd, kd, vd = _dev((q, k, v))
    out = torch.full_like(qd, float("nan"))
    fps.skiparse1d_attn_fwd(qd, kd, vd, w.P, mode, out=out)
    assert fps.get_device_status() == 0
    check_close(out.to(torch.float64).cpu().numpy(), want, f"1d {w.name} mode={mode}")


@pytest.mark.parametrize("name", ["480p", "720p"])
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_attention_1d_full_size_sampled(fps, name, mode):
    w = synth.WORKLOADS[name]
    q, k, v = synth.qkv(w)
    qd, kd, vd = _dev((q, k, v))
    out = torch.full_like(qd, float("nan"))
    fps.skiparse1d_attn_fwd(qd, kd, vd, w.P, mode, out=out)
    assert fps.get_device_status() == 0
    assert not torch.isnan(out).any().item(), "a real token was left unwritten"
    rows = sample_rows(w, 320, seed=w.family * 10 + mode + 5)
    want = oracle.attn_fwd_rows(q, k, v, rows, w.P, mode, dims=1)
    check_close(gpu_rows(out, rows), want, f"1d {name} mode={mode}")


def test_1d_and_2d_are_different_patterns(fps):
    w = synth.WORKLOADS["anyres"]
    qd, kd, vd = _dev(synth.qkv(w))
    a = fps.skiparse1d_attn_fwd(qd, kd, vd, w.P, TOK)
    b = fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, TOK)
    assert not torch.equal(a, b)


@pytest.mark.parametrize("name", ["tiny", "anyres", "480p", "720p"])
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_rearrange_1d_bit_exact(fps, name, mode):
    w = synth.WORKLOADS[name]
    x, _, _ = synth.qkv(w)
    want = oracle.rearrange(x, w.P, mode, dims=1)
    xd = x.cuda()
    y = torch.empty(fps.rearranged_shape(x.shape, w.P, dims=1), dtype=torch.bfloat16, device="cuda")
    y.view(torch.int16).fill_(-1)
    fps.skiparse1d_rearrange(xd, w.P, mode, out=y)
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), want)
    back = torch.empty_like(xd)
    back.view(torch.int16).fill_(-1)
    fps.skiparse1d_unrearrange(y, x.shape, w.P, mode, out=back)
    assert torch.equal(back.view(torch.int16).cpu(), x.view(torch.int16))


@pytest.mark.parametrize("w", [synth.WORKLOADS["anyres"], synth.custom(2, 2, 5, 7, 3, 32, 3, "p3"),
                               synth.custom(1, 2, 8, 9, 2, 64, 8, "p8")], ids=lambda w: w.name)
@pytest.mark.parametrize("src", [TOK, GRP])
def test_switch_1d_bit_exact(fps, w, src):
    x, _, _ = synth.qkv(w)
    ysrc = oracle.rearrange(x, w.P, src, dims=1)
    want = oracle.switch_mode(ysrc, w.shape, w.P, src, dims=1)
    yd = torch.from_numpy(ysrc.view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty_like(yd)
    out.view(torch.int16).fill_(-1)
    fps.skiparse1d_switch_mode(yd, w.shape, w.P, src, out=out)
    assert fps.get_device_status() == 0
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
    # pad slots of the source are ignored: unrearrange of garbage pads gives the oracle's answer
    noisy = synth.randn_bf16(tuple(yd.shape), 78)
    got = fps.skiparse1d_unrearrange(noisy.cuda(), w.shape, w.P, src)
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16),
                          oracle.unrearrange(noisy, w.shape, w.P, src, dims=1))


BWD_SMALL = [synth.WORKLOADS["tiny"], synth.WORKLOADS["anyres"], synth.custom(1, 2, 20, 30, 2, 128, 3, "p3"),
             synth.custom(1, 6, 24, 40, 2, 128, 2, "multi_tile"), synth.custom(1, 2, 8, 9, 1, 64, 8, "p8")]


@pytest.mark.parametrize("w", BWD_SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_backward_1d_small_full(fps, w, mode):
    q, k, v = synth.qkv(w)
    dout = synth.randn_bf16(w.shape, 950 + w.family)
    dq_ref, dk_ref, dv_ref, lse_ref = oracle.attn_bwd(q, k, v, dout, w.P, mode, dims=1)
    qd, kd, vd, gd = (t.cuda() for t in (q, k, v, dout))
    out, lse = fps.skiparse1d_attn_fwd_lse(qd, kd, vd, w.P, mode)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    fps.skiparse1d_attn_bwd(qd, kd, vd, out, gd, lse, w.P, mode, dq=dq, dk=dk, dv=dv)
    assert fps.get_device_status() == 0
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=0, atol=1e-3)
    check_grad(dq.double().cpu().numpy(), dq_ref, f"1d {w.name} dq")
    check_grad(dk.double().cpu().numpy(), dk_ref, f"1d {w.name} dk")
    check_grad(dv.double().cpu().numpy(), dv_ref, f"1d {w.name} dv")


@pytest.mark.parametrize("name,mode", [("480p", GRP), ("720p", TOK)])
def test_backward_1d_full_size_sampled(fps, name, mode):
    w = synth.WORKLOADS[name]
    q, k, v = synth.qkv(w)
    dout = synth.randn_bf16(w.shape, 950 + w.family)
    qd, kd, vd, gd = (t.cuda() for t in (q, k, v, dout))
    out, lse = fps.skiparse1d_attn_fwd_lse(qd, kd, vd, w.P, mode)
    dq, dk, dv = fps.skiparse1d_attn_bwd(qd, kd, vd, out, gd, lse, w.P, mode)
    assert fps.get_device_status() == 0
    rows = sample_rows_one_class_1d(w, mode, 24, cls=w.P * w.P - 1, head=w.heads - 1, seed=w.family)
    rq, rk, rv = oracle.attn_bwd_rows(q, k, v, dout, rows, w.P, mode, dims=1)
    idx = torch.from_numpy(rows).cuda()
    for got, want, what in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        check_grad(got.reshape(-1, w.d).index_select(0, idx).double().cpu().numpy(), want, f"1d {name} {what}")


def test_autograd_1d_matches_oracle(fps):
    w = synth.WORKLOADS["anyres"]
    q, k, v = synth.qkv(w)
    dout = synth.randn_bf16(w.shape, 996)
    qd, kd, vd = (t.cuda().requires_grad_(True) for t in (q, k, v))
    out = fps.skiparse_attention(qd, kd, vd, w.P, GRP, dims=1)
    out.backward(dout.cuda())
    dq_ref, dk_ref, dv_ref, _ = oracle.attn_bwd(q, k, v, dout, w.P, GRP, dims=1)
    check_grad(qd.grad.double().cpu().numpy(), dq_ref, "1d autograd dq")
    check_grad(kd.grad.double().cpu().numpy(), dk_ref, "1d autograd dk")
    check_grad(vd.grad.double().cpu().numpy(), dv_ref, "1d autograd dv")
