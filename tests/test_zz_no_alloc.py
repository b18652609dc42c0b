"""The allocation-free backward entry point, skiparse2d_attn_bwd_noalloc, called through the C ABI.

It is meant for callers that cannot allocate device memory themselves (a host framework that
owns every allocation, a loop that must not call the allocator): it keeps the backward's D
workspace in a fixed array inside the library. Here its results are checked against the
regular entry point, skiparse2d_attn_bwd (given a workspace allocated by torch), on two calls in
a row of different sizes, so the second call runs on a workspace that still holds the first
call's contents. Same tolerance as the other backward tests. This file is collected last and
also passes when run on its own in a fresh process."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import skiparse_synth as synth

pytestmark = pytest.mark.gpu


def _bwd_noalloc(L, qd, kd, vd, out, gd, lse, w, mode):
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    rc = L.skiparse2d_attn_bwd_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), out.data_ptr(), gd.data_ptr(),
                                       lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                       w.B, w.T, w.H, w.W, w.heads, w.d, w.P, mode,
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == 0, rc
    return dq, dk, dv


def _close(got, want, what):
    got, want = got.double().cpu().numpy(), want.double().cpu().numpy()
    assert np.all(np.isfinite(got)), what
    scale = max(np.abs(want).max(), 1e-3)
    err = np.abs(got - want)
    assert err.max() <= 2e-2 * scale and err.mean() <= 2e-3 * scale, what


def test_noalloc_backward_matches_regular_entry_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as fps
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    cases = [(synth.custom(1, 6, 24, 40, 2, 128, 2, "first"), 0),
             (synth.WORKLOADS["anyres"], 1)]  # smaller second call: stale workspace contents
    for w, mode in cases:
        q, k, v = (t.cuda() for t in synth.qkv(w))
        g = synth.randn_bf16(w.shape, 1234 + w.family).cuda()
        out, lse = fps.skiparse2d_attn_fwd_lse(q, k, v, w.P, mode)
        ref = fps.skiparse2d_attn_bwd(q, k, v, out, g, lse, w.P, mode)
        got = _bwd_noalloc(L, q, k, v, out, g, lse, w, mode)
        assert fps.get_device_status() == 0
        for a, b, what in zip(got, ref, ("dq", "dk", "dv")):
            _close(a, b, f"{w.name} {what}")


def test_noalloc_backward_rejects_sizes_beyond_its_workspace():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    fake = 0x10000  # never dereferenced: the size check comes first
    # 21 x 64 x 64 x 40 x 40 rows = 137,625,600 > 2^22
    rc = L.skiparse2d_attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                       1, 21, 64 * 8, 64 * 8, 40, 128, 2, 0, None)
    assert rc == 2  # SKIPARSE_ERR_UNSUPPORTED
