"""GPU parity: the sm_100a kernels (through the C ABI) against the fp64 CPU oracle on the
same seeded inputs. Rearrange / unrearrange must be bit-exact; attention must meet
max|err| <= 1e-2 and mean|err| <= 1e-3 (bf16 in and out, N(0,1) inputs, scale 1/sqrt(d)).

Small shapes are compared element by element (they span several 128-row tiles and end in
ragged tails); the full-size latents are compared on sampled rows in the same launch
configuration the benchmark times."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import skiparse_synth as synth
from parity_helpers import check_close, gpu_rows, sample_rows, subsequence_rows

pytestmark = pytest.mark.gpu

TOK, GRP = 0, 1


@pytest.fixture(scope="module")
def fps():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as m
    return m


SMALL = [
    synth.WORKLOADS["tiny"],                                   # n = 32 < one tile, d = 32
    synth.WORKLOADS["anyres"],                                 # padded 12x16, n_c = 105 / 144 / 96
    synth.custom(2, 3, 13, 22, 3, 64, 2, "b2_ragged"),         # B = 2, two tiles, ragged tail
    synth.custom(1, 2, 20, 30, 2, 128, 3, "p3_unequal"),       # P = 3, classes of unequal size
    synth.custom(1, 5, 16, 16, 2, 128, 1, "dense_p1"),         # P = 1 dense, 10 full tiles
    synth.custom(1, 3, 17, 19, 1, 32, 4, "p4"),                # P = 4, 16 classes
    synth.custom(1, 1, 1, 1, 1, 64, 2, "one_token"),           # a single real token
    synth.custom(1, 6, 24, 40, 2, 128, 2, "multi_tile"),       # n_c = 1440: 12 tiles
    synth.custom(1, 4, 9, 33, 2, 128, 2, "thin"),              # W >> H, ragged both ways
    synth.custom(3, 2, 6, 10, 5, 64, 2, "b3_h5"),              # B = 3, 5 heads
    synth.custom(1, 2, 26, 31, 1, 64, 5, "p5"),                # P = 5: 25 classes, padded 50x50
    synth.custom(1, 2, 40, 45, 2, 128, 6, "p6"),               # P = 6: padded 72x72, 2 tiles
    synth.custom(1, 1, 50, 100, 1, 64, 7, "p7"),               # P = 7: padded 98x147, H != W
    synth.custom(1, 1, 70, 65, 1, 32, 8, "p8"),                # P = 8 (the maximum): 64 classes
]

LARGE = ["480p", "720p", "768p", "768p_p3", "768p_p1"]


def _dev(ts):
    return [t.cuda() for t in ts]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_attention_small_full(fps, w, mode):
    q, k, v = synth.qkv(w)
    want = oracle.attn_fwd(q, k, v, w.P, mode)
    qd, kd, vd = _dev((q, k, v))
    out = torch.full_like(qd, float("nan"))  # canary: every real token must be written
    fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, mode, out=out)
    assert fps.get_device_status() == 0
    got = out.to(torch.float64).cpu().numpy()
    check_close(got, want, f"{w.name} mode={mode}")


@pytest.mark.parametrize("name", LARGE)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_attention_full_size_sampled(fps, name, mode):
    w = synth.WORKLOADS[name]
    if w.P == 1 and mode == GRP:
        pytest.skip("P = 1 makes the modes identical")
    q, k, v = synth.qkv(w)
    qd, kd, vd = _dev((q, k, v))
    out = torch.full_like(qd, float("nan"))
    fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, mode, out=out)
    assert fps.get_device_status() == 0
    assert not torch.isnan(out).any().item(), "a real token was left unwritten"
    rows = sample_rows(w, 160 if w.P == 1 else 320, seed=w.family * 10 + mode)
    want = oracle.attn_fwd_rows(q, k, v, rows, w.P, mode)
    check_close(gpu_rows(out, rows), want, f"{name} mode={mode}")


# Whole subsequences at full size: every query of one (class, head), element by element, in the
# launch configuration the benchmark times. The last class and the last head are the raggedest in
# padded workloads (720p: 45 rows padded to 48; 768p P = 3: 48x84 padded to 54x90); group-wise
# classes differ from token-wise ones only through the row map, which these cover in full.
WHOLE = [("720p", TOK, -1), ("720p", GRP, -1), ("768p_p3", TOK, -1), ("768p_p3", GRP, -1),
         ("768p_p3", GRP, 4)]


@pytest.mark.parametrize("name,mode,cls", WHOLE, ids=[f"{n}-{'grp' if m else 'tok'}-c{c}" for n, m, c in WHOLE])
def test_attention_whole_subsequence(fps, name, mode, cls):
    w = synth.WORKLOADS[name]
    cls = cls % (w.P * w.P)
    head = w.heads - 1
    q, k, v = synth.qkv(w)
    qd, kd, vd = _dev((q, k, v))
    out = torch.full_like(qd, float("nan"))
    fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, mode, out=out)
    assert fps.get_device_status() == 0
    rows = subsequence_rows(w, mode, cls, head)
    assert len(rows) > 8000
    want = oracle.attn_fwd_rows(q, k, v, rows, w.P, mode)
    check_close(gpu_rows(out, rows), want, f"{name} mode={mode} class={cls} head={head} ({len(rows)} rows)")


def test_attention_is_deterministic_and_stream_ordered(fps):
    w = synth.WORKLOADS["anyres"]
    qd, kd, vd = _dev(synth.qkv(w))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, GRP)
        b = fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, GRP)
    s.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["tiny", "anyres", "480p", "720p", "768p", "768p_p3", "768p_p1"])
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_rearrange_bit_exact(fps, name, mode):
    w = synth.WORKLOADS[name]
    x, _, _ = synth.qkv(w)
    want = oracle.rearrange(x, w.P, mode)
    xd = x.cuda()
    y = torch.empty(fps.rearranged_shape(x.shape, w.P), dtype=torch.bfloat16, device="cuda")
    y.view(torch.int16).fill_(-1)  # canary: pad slots must become +0.0
    fps.skiparse_rearrange(xd, w.P, mode, out=y)
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want)
    # inverse: back to the original, bit for bit
    back = torch.empty_like(xd)
    back.view(torch.int16).fill_(-1)
    fps.skiparse_unrearrange(y, x.shape, w.P, mode, out=back)
    assert torch.equal(back.view(torch.int16).cpu(), x.view(torch.int16))


@pytest.mark.parametrize("w", [w for w in SMALL if w.P >= 5], ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_rearrange_bit_exact_large_p(fps, w, mode):
    """P = 5..8 (up to 64 classes, most of them holding pad slots) on small latents."""
    x, _, _ = synth.qkv(w)
    want = oracle.rearrange(x, w.P, mode)
    xd = x.cuda()
    y = torch.empty(fps.rearranged_shape(x.shape, w.P), dtype=torch.bfloat16, device="cuda")
    y.view(torch.int16).fill_(-1)
    fps.skiparse_rearrange(xd, w.P, mode, out=y)
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), want)
    back = torch.empty_like(xd)
    back.view(torch.int16).fill_(-1)
    fps.skiparse_unrearrange(y, x.shape, w.P, mode, out=back)
    assert torch.equal(back.view(torch.int16).cpu(), x.view(torch.int16))


@pytest.mark.parametrize("w", [synth.WORKLOADS["anyres"], synth.custom(2, 2, 5, 7, 3, 32, 3, "p3"),
                               synth.custom(1, 2, 9, 9, 2, 128, 4, "p4")], ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [TOK, GRP])
def test_unrearrange_ignores_pad_slots(fps, w, mode):
    shape = fps.rearranged_shape(w.shape, w.P)
    y = synth.randn_bf16(shape, 77)  # pad slots hold garbage on purpose
    want = oracle.unrearrange(y, w.shape, w.P, mode)
    got = fps.skiparse_unrearrange(y.cuda(), w.shape, w.P, mode)
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("name", ["tiny", "anyres", "480p", "720p", "768p", "768p_p3"])
@pytest.mark.parametrize("src", [TOK, GRP])
def test_switch_mode_bit_exact(fps, name, src):
    """Token-wise <-> group-wise re-layout in one pass, against the oracle."""
    w = synth.WORKLOADS[name]
    x, _, _ = synth.qkv(w)
    ysrc = oracle.rearrange(x, w.P, src)
    want = oracle.switch_mode(ysrc, w.shape, w.P, src)
    yd = torch.from_numpy(ysrc.view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty_like(yd)
    out.view(torch.int16).fill_(-1)  # canary: pad slots must become +0.0
    fps.skiparse_switch_mode(yd, w.shape, w.P, src, out=out)
    assert fps.get_device_status() == 0
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)


def test_switch_mode_equals_inverse_then_rearrange(fps):
    w = synth.custom(2, 3, 11, 17, 3, 64, 3, "p3_b2")
    x = synth.qkv(w)[0].cuda()
    for src in (TOK, GRP):
        y = fps.skiparse_rearrange(x, w.P, src)
        a = fps.skiparse_switch_mode(y, w.shape, w.P, src)
        b = fps.skiparse_rearrange(fps.skiparse_unrearrange(y, w.shape, w.P, src), w.P, 1 - src)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
