"""The allocation-free backward entry point, skiparse2d_attn_bwd_noalloc, called through the C ABI.

It is meant for callers that cannot allocate device memory themselves (a host framework that
owns every allocation, a loop that must not call the allocator): it keeps the backward's D
workspace in a fixed array inside the library. Its results are checked against the regular
entry point, skiparse2d_attn_bwd (given a workspace allocated by torch): both run the same
deterministic kernels (no atomics), so the gradients must be identical bit for bit. Two calls
in a row of different sizes make the second run on a workspace that still holds the first
call's contents; a call at exactly the workspace's capacity (2^22 rows) writes its last
element; one small case is also held to the fp64 oracle directly. This file is collected last
and also passes when run on its own in a fresh process."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import skiparse_synth as synth

pytestmark = pytest.mark.gpu

CAPACITY = 1 << 22  # rows (B*T*H*W*heads) the library's workspace holds


def _bwd_noalloc(L, qd, kd, vd, out, gd, lse, w, mode):
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    rc = L.skiparse2d_attn_bwd_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), out.data_ptr(), gd.data_ptr(),
                                       lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                       w.B, w.T, w.H, w.W, w.heads, w.d, w.P, mode,
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == 0, rc
    return dq, dk, dv


def _skip_without_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_noalloc_backward_matches_regular_entry_twice():
    _skip_without_cuda()
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
            assert torch.equal(a, b), f"{w.name} {what}"


def test_noalloc_backward_at_full_capacity():
    """B*T*H*W*heads = 2^22 exactly (16 x 64 x 64 frames, 64 heads): the workspace's last
    element is written and read; the result equals the regular entry's bit for bit."""
    _skip_without_cuda()
    import fixed_pattern_sparse_b200 as fps
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    w = synth.custom(1, 16, 64, 64, 64, 32, 2, "capacity")
    assert w.B * w.T * w.H * w.W * w.heads == CAPACITY
    q, k, v = (t.cuda() for t in synth.qkv(w))
    g = synth.randn_bf16(w.shape, 4321).cuda()
    for mode in (0, 1):
        out, lse = fps.skiparse2d_attn_fwd_lse(q, k, v, w.P, mode)
        ref = fps.skiparse2d_attn_bwd(q, k, v, out, g, lse, w.P, mode)
        got = _bwd_noalloc(L, q, k, v, out, g, lse, w, mode)
        assert fps.get_device_status() == 0
        for a, b, what in zip(got, ref, ("dq", "dk", "dv")):
            assert torch.equal(a, b), f"mode {mode} {what}"


def test_noalloc_backward_matches_the_oracle():
    """One small padded case held to the fp64 oracle directly, at the backward tests' tolerance
    (max|err| <= 2e-2 * max|ref|, mean|err| <= 2e-3 * max|ref|)."""
    _skip_without_cuda()
    import fixed_pattern_sparse_b200 as fps
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    w = synth.custom(1, 3, 13, 22, 3, 64, 2, "small_padded")
    q, k, v = synth.qkv(w)
    g = synth.randn_bf16(w.shape, 555)
    for mode in (0, 1):
        want = oracle.attn_bwd(q, k, v, g, w.P, mode)[:3]
        qd, kd, vd, gd = (t.cuda() for t in (q, k, v, g))
        out, lse = fps.skiparse2d_attn_fwd_lse(qd, kd, vd, w.P, mode)
        got = _bwd_noalloc(L, qd, kd, vd, out, gd, lse, w, mode)
        assert fps.get_device_status() == 0
        for a, ref, what in zip(got, want, ("dq", "dk", "dv")):
            a = a.double().cpu().numpy()
            assert np.all(np.isfinite(a)), what
            scale = max(np.abs(ref).max(), 1e-3)
            err = np.abs(a - ref)
            assert err.max() <= 2e-2 * scale and err.mean() <= 2e-3 * scale, f"mode {mode} {what}"


def test_noalloc_backward_rejects_sizes_beyond_its_workspace():
    _skip_without_cuda()
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    fake = 0x10000  # never dereferenced: the size check comes first
    # 1 x 21 x 512 x 512 frames x 40 heads = 220,200,960 rows > 2^22
    rc = L.skiparse2d_attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                       1, 21, 64 * 8, 64 * 8, 40, 128, 2, 0, None)
    assert rc == 2  # SKIPARSE_ERR_UNSUPPORTED
    # one row more than the capacity
    rc = L.skiparse2d_attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                       1, 1, 1, CAPACITY + 1, 1, 32, 2, 0, None)
    assert rc == 2
