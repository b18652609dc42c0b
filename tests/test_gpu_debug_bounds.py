"""The bounds-checking debug build, libskiparse_debug.so, through the C ABI.

Its kernels check every token row index they compute for a global load or store against the
row count of the tensor and report an index outside as SKIPARSE_ERR_BOUNDS (skipping the access,
so the check never leaves a tensor). Here: (1) on real workloads it reports nothing, and its
results equal the release build's bit for bit -- the checks change no arithmetic; (2) with the
bounds declared a few rows smaller than the tensors (skiparse_debug_shrink_bounds) every entry
point reports SKIPARSE_ERR_BOUNDS, while every access it makes still lies inside the tensors."""

from __future__ import annotations

import pytest
import torch

import skiparse_synth as synth

pytestmark = pytest.mark.gpu

BOUNDS = 6  # SKIPARSE_ERR_BOUNDS

SHAPES = [synth.WORKLOADS["tiny"], synth.WORKLOADS["anyres"],
          synth.custom(2, 2, 11, 17, 3, 64, 3, "p3_b2"), synth.custom(1, 1, 70, 65, 1, 32, 8, "p8"),
          synth.custom(1, 3, 20, 30, 2, 128, 2, "multi_tile")]


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import os
    from fixed_pattern_sparse_b200 import _lib
    from fixed_pattern_sparse_b200 import build as libbuild
    if not os.path.exists(_lib.DEBUG_LIB_PATH):  # a checkout where only the release build was made
        libbuild.build(debug=True)
    return _lib.lib(), _lib.debug_lib()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _dims(w):
    return (w.B, w.T, w.H, w.W, w.heads, w.d, w.P)


def _run_all(L, w, mode, q, k, v, g):
    """Every entry point of library L on one workload; returns its outputs and the status."""
    st = _stream()
    dims = _dims(w)
    res = {}
    out = torch.empty_like(q)
    assert L.skiparse2d_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), *dims, mode, st) == 0
    res["fwd"] = out
    out2 = torch.empty_like(q)
    lse = torch.empty(q.shape[:5], dtype=torch.float32, device=q.device)
    assert L.skiparse2d_attn_fwd_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out2.data_ptr(), lse.data_ptr(),
                                     *dims, mode, st) == 0
    res["lse"] = lse
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    delta = torch.empty_like(lse)
    assert L.skiparse2d_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out2.data_ptr(), g.data_ptr(),
                                 lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), delta.data_ptr(),
                                 *dims, mode, st) == 0
    res.update(dq=dq, dk=dk, dv=dv)
    n = L.skiparse_rearranged_numel(w.B, w.T, w.H, w.W, w.heads, w.d, w.P)
    y = torch.empty(n, dtype=torch.bfloat16, device=q.device)
    assert L.skiparse_rearrange(q.data_ptr(), y.data_ptr(), *dims, mode, st) == 0
    res["rearrange"] = y
    y2 = torch.empty_like(y)
    assert L.skiparse_switch_mode(y.data_ptr(), y2.data_ptr(), *dims, mode, st) == 0
    res["switch"] = y2
    back = torch.empty_like(q)
    assert L.skiparse_unrearrange(y.data_ptr(), back.data_ptr(), *dims, mode, st) == 0
    res["unrearrange"] = back
    o1 = torch.empty_like(q)
    assert L.skiparse1d_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o1.data_ptr(), *dims, mode, st) == 0
    res["fwd1d"] = o1
    return res, L.skiparse_get_device_status(st)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_debug_build_reports_nothing_and_matches_release(libs, w, mode):
    R, D = libs
    q, k, v = (t.cuda() for t in synth.qkv(w))
    g = synth.randn_bf16(w.shape, 4321).cuda()
    want, st_r = _run_all(R, w, mode, q, k, v, g)
    got, st_d = _run_all(D, w, mode, q, k, v, g)
    assert st_r == 0 and st_d == 0, (st_r, st_d)
    for name in want:
        a, b = want[name], got[name]
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b), name


def test_debug_build_reports_rows_outside_declared_bounds(libs):
    R, D = libs
    w = synth.WORKLOADS["tiny"]  # no padding: every rearranged slot is a real token
    q, k, v = (t.cuda() for t in synth.qkv(w))
    g = synth.randn_bf16(w.shape, 4321).cuda()
    st = _stream()
    dims = _dims(w)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:5], dtype=torch.float32, device="cuda")
    assert D.skiparse2d_attn_fwd_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                     *dims, 0, st) == 0
    assert D.skiparse_get_device_status(st) == 0
    n = D.skiparse_rearranged_numel(*dims)
    y = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty_like(y)
    tmp = torch.empty_like(q)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    delta = torch.empty_like(lse)
    calls = {
        "fwd": lambda: D.skiparse2d_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), tmp.data_ptr(), *dims, 1, st),
        "bwd": lambda: D.skiparse2d_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), g.data_ptr(),
                                             lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                             delta.data_ptr(), *dims, 0, st),
        "rearrange": lambda: D.skiparse_rearrange(q.data_ptr(), y.data_ptr(), *dims, 0, st),
        "switch": lambda: D.skiparse_switch_mode(y.data_ptr(), y2.data_ptr(), *dims, 0, st),
        "unrearrange": lambda: D.skiparse_unrearrange(y.data_ptr(), tmp.data_ptr(), *dims, 0, st),
        "fwd1d": lambda: D.skiparse1d_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), tmp.data_ptr(), *dims, 0, st),
    }
    for name, call in calls.items():
        assert call() == 0, name                       # a clean launch first (y holds a rearrange)
        assert D.skiparse_get_device_status(st) == 0, name
        assert D.skiparse_debug_shrink_bounds(5) == 0
        assert call() == 0, name
        assert D.skiparse_get_device_status(st) == BOUNDS, name
    # the hook is consumed by one launch, and the release build is unaffected throughout
    assert calls["fwd"]() == 0 and D.skiparse_get_device_status(st) == 0
    assert R.skiparse_get_device_status(st) == 0
