"""Failure detection without a GPU fault: every wait in the attention kernels is bounded.

The test hook (skiparse_debug_inject_fault) makes one producer thread of the next launch skip
its cp.async arrival on the first K-tile barrier (forward) or on the first streamed tile's
barrier (backward, key-major kernel). That barrier then never completes -- a flag that nothing
sets -- so the MMA warp's bounded wait runs out. The kernel must record SKIPARSE_ERR_TIMEOUT in
the device status word, release its tensor memory and return; the context stays usable and the
next launch is correct."""

from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import oracle
import skiparse_synth as synth
from parity_helpers import check_close

pytestmark = pytest.mark.gpu


def test_lost_arrival_times_out_and_recovers():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as fps
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.qkv(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    assert fps.get_device_status() == 0
    prev = L.skiparse_set_wait_limit_ns(100_000_000)  # 0.1 s
    try:
        assert L.skiparse_debug_inject_fault(1) == 0
        t0 = time.time()
        fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, 0)
        status = fps.get_device_status()
        elapsed = time.time() - t0
        assert status == 5, f"expected SKIPARSE_ERR_TIMEOUT, got {status}"
        assert elapsed < 30
    finally:
        L.skiparse_debug_inject_fault(0)
        L.skiparse_set_wait_limit_ns(prev)
    # the context is still usable and the next launch is right
    out = fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, 0)
    assert fps.get_device_status() == 0
    check_close(out.to(torch.float64).cpu().numpy(), oracle.attn_fwd(q, k, v, w.P, 0), "after timeout")


def test_backward_lost_arrival_times_out_and_recovers():
    """The same for the backward pass: one producer thread of the key-major kernel never signals
    the first streamed tile; the call reports SKIPARSE_ERR_TIMEOUT, and the next call is right."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as fps
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.qkv(w)
    g = synth.randn_bf16(w.shape, 99)
    qd, kd, vd, gd = (t.cuda() for t in (q, k, v, g))
    out, lse = fps.skiparse2d_attn_fwd_lse(qd, kd, vd, w.P, 1)
    assert fps.get_device_status() == 0
    prev = L.skiparse_set_wait_limit_ns(100_000_000)  # 0.1 s
    try:
        assert L.skiparse_debug_inject_fault(2) == 0
        # a forward in between neither consumes nor triggers the backward's hook
        fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, 1)
        assert fps.get_device_status() == 0
        t0 = time.time()
        fps.skiparse2d_attn_bwd(qd, kd, vd, out, gd, lse, w.P, 1)
        status = fps.get_device_status()
        assert status == 5, f"expected SKIPARSE_ERR_TIMEOUT, got {status}"
        assert time.time() - t0 < 30
    finally:
        L.skiparse_debug_inject_fault(0)
        L.skiparse_set_wait_limit_ns(prev)
    dq, dk, dv = fps.skiparse2d_attn_bwd(qd, kd, vd, out, gd, lse, w.P, 1)
    assert fps.get_device_status() == 0
    refs = oracle.attn_bwd(q, k, v, g, w.P, 1)[:3]
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        scale = max(np.abs(want).max(), 1e-3)
        err = np.abs(got.to(torch.float64).cpu().numpy() - want)
        assert err.max() <= 2e-2 * scale and err.mean() <= 2e-3 * scale, name
