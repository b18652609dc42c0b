"""The host-buffer forward (skiparse2d_attn_fwd_host / skiparse1d_attn_fwd_host) through the C ABI:
identical, bit for bit, to the device-buffer forward on the same inputs (the same kernel runs on
each group of heads), for uneven head groups, both patterns and both modes; and ordered on the
caller's stream."""

from __future__ import annotations

import pytest
import torch

import skiparse_synth as synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fps():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as m
    return m


def _pinned(t):
    return t.contiguous().pin_memory()


@pytest.mark.parametrize("w,group", [(synth.custom(1, 3, 13, 22, 5, 64, 2, "h5"), 2),
                                     (synth.custom(2, 2, 10, 14, 4, 128, 2, "h4"), 4),
                                     (synth.custom(1, 2, 12, 16, 3, 32, 3, "h3"), 1),
                                     (synth.WORKLOADS["480p"], 5)],
                         ids=["h5g2", "h4g4", "h3g1", "480p_g5"])
@pytest.mark.parametrize("dims", [2, 1])
@pytest.mark.parametrize("mode", [0, 1])
def test_host_path_equals_device_path(fps, w, group, dims, mode):
    q, k, v = synth.qkv(w)
    want = fps._attn_fwd(dims, q.cuda(), k.cuda(), v.cuda(), w.P, mode, None, None).cpu()
    qh, kh, vh = (_pinned(t) for t in (q, k, v))
    out = torch.full(w.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
    fps.attn_fwd_host(qh, kh, vh, w.P, mode, out, heads_per_group=group, dims=dims)
    torch.cuda.current_stream().synchronize()
    assert fps.get_device_status() == 0
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))


def test_host_path_is_ordered_on_the_callers_stream(fps):
    w = synth.custom(1, 2, 16, 16, 6, 128, 2, "order")
    q, k, v = synth.qkv(w)
    qh, kh, vh = (_pinned(t) for t in (q, k, v))
    s = torch.cuda.Stream()
    outs = [torch.empty(w.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    ws = torch.empty(fps.host_workspace_bytes(w.shape, 2), dtype=torch.uint8, device="cuda")
    for o in outs:  # two calls back to back on one stream, one workspace
        fps.attn_fwd_host(qh, kh, vh, w.P, 1, o, heads_per_group=2, workspace=ws, stream=s)
    s.synchronize()
    want = fps.skiparse2d_attn_fwd(q.cuda(), k.cuda(), v.cuda(), w.P, 1).cpu()
    for o in outs:
        assert torch.equal(o.view(torch.int16), want.view(torch.int16))
