"""CPU oracle for Skiparse-2D (and Skiparse-1D) attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg of
``bench.py`` may import this package. The product path (``fixed_pattern_sparse_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``skiparse_oracle.c`` (fp64, explicit index loops, one
function per step of the method as the OSP-Next summary page's 方法步骤详情 (method
step details) section orders them). This module only marshals numpy arrays.

Parity status of each function (what pins it is in tests/test_oracle_pins.py):
  padded_extent, axis_map, rearrange, unrearrange -- pinned (pixel_unshuffle library
      routine, hand-derived golden class maps, permutation/identity/local-equivalence
      invariants, two-hop property);
  switch_mode -- pinned (equals unrearrange of one mode followed by rearrange of the other;
      a switch there and back is the identity on real slots; pads are zero);
  attn_bwd, attn_bwd_rows -- pinned (torch autograd through an independent dense masked fp64
      attention; P=1 against autograd of fp64 scaled_dot_product_attention; central finite
      differences of the forward oracle; sampled rows equal the full result);
  attn_fwd, attn_fwd_rows, masked_attention -- pinned (P=1 against fp64
      scaled_dot_product_attention, numpy brute force with an explicit 2-D mask,
      closed forms, pad invariance).
Every function takes ``dims=2`` (Skiparse-2D, the default) or ``dims=1`` (Skiparse-1D, the
flattened-sequence variant, tests/test_oracle_1d_pins.py): numpy strided slicing and
reshape for the class rule, a brute force with an explicit 1-D class mask, P=1 against
scaled_dot_product_attention, torch autograd for the backward pass.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

TOKEN_WISE = 0
GROUP_WISE = 1

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        _LIB = load(_build.build())
    return _LIB


def load(path: str):
    """A ctypes handle on an oracle library at `path`, with every function's signature bound
    (lib() is the normal build; the oracle's mutation tests load planted-mistake builds)."""
    L = ctypes.CDLL(path)
    c_int, c_ll, vp = ctypes.c_int, ctypes.c_longlong, ctypes.c_void_p
    L.oracle_padded_extent.argtypes = [c_int, c_int]
    L.oracle_padded_extent.restype = c_int
    L.oracle_axis_map.argtypes = [c_int, c_int, c_int, ctypes.POINTER(c_int), ctypes.POINTER(c_int)]
    L.oracle_axis_map.restype = c_int
    L.oracle_subseq_len.argtypes = [c_int, c_int, c_int, c_int]
    L.oracle_subseq_len.restype = c_ll
    shape8 = [c_int] * 8  # B, T, H, W, heads, d, P, mode
    L.oracle_rearrange.argtypes = [vp, vp, vp] + shape8
    L.oracle_rearrange.restype = c_int
    L.oracle_unrearrange.argtypes = [vp, vp] + shape8
    L.oracle_unrearrange.restype = c_int
    L.oracle_switch_mode.argtypes = [vp, vp] + shape8
    L.oracle_switch_mode.restype = c_int
    L.oracle_unrearrange_f64.argtypes = [vp, vp] + shape8
    L.oracle_unrearrange_f64.restype = c_int
    L.oracle_masked_attention.argtypes = [vp, vp, vp, vp, vp, c_ll, c_ll, c_int, c_int, c_int]
    L.oracle_masked_attention.restype = c_int
    L.oracle_attn_fwd.argtypes = [vp, vp, vp, vp] + shape8 + [c_int]
    L.oracle_attn_fwd.restype = c_int
    L.oracle_attn_fwd_rows.argtypes = [vp, vp, vp, vp, c_ll, vp] + shape8 + [c_int]
    L.oracle_attn_fwd_rows.restype = c_int
    L.oracle_attn_bwd.argtypes = [vp] * 8 + shape8 + [c_int]
    L.oracle_attn_bwd.restype = c_int
    L.oracle_attn_bwd_rows.argtypes = [vp, vp, vp, vp, vp, c_ll, vp, vp, vp] + shape8 + [c_int]
    L.oracle_attn_bwd_rows.restype = c_int
    L.oracle1d_padded_length.argtypes = [c_int, c_int]
    L.oracle1d_padded_length.restype = c_int
    L.oracle1d_index_map.argtypes = L.oracle_axis_map.argtypes
    L.oracle1d_index_map.restype = c_int
    L.oracle1d_subseq_len.argtypes = L.oracle_subseq_len.argtypes
    L.oracle1d_subseq_len.restype = c_ll
    for name in ("rearrange", "unrearrange", "switch_mode", "unrearrange_f64", "attn_fwd",
                 "attn_fwd_rows", "attn_bwd", "attn_bwd_rows"):
        f1, f2 = getattr(L, "oracle1d_" + name), getattr(L, "oracle_" + name)
        f1.argtypes, f1.restype = f2.argtypes, f2.restype
    return L


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _bits(a) -> np.ndarray:
    """bf16 data as a contiguous uint16 numpy array of raw bit patterns."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch  # local: only for the dtype view
        return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    arr = np.ascontiguousarray(a)
    if arr.dtype != np.uint16:
        raise TypeError("expected bfloat16 torch tensor or uint16 bit-pattern array")
    return arr


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def _fn(name: str, dims: int):
    """The C function for Skiparse-2D (dims=2) or Skiparse-1D (dims=1)."""
    if dims not in (1, 2):
        raise ValueError("dims must be 1 or 2")
    return getattr(lib(), ("oracle1d_" if dims == 1 else "oracle_") + name)


def padded_extent(X: int, P: int) -> int:
    return lib().oracle_padded_extent(X, P)


def padded_length_1d(L: int, P: int) -> int:
    """Skiparse-1D: per-frame length H*W padded to the next multiple of P^4."""
    return lib().oracle1d_padded_length(L, P)


def index_map_1d(x: int, P: int, mode: int):
    """Skiparse-1D class and in-class position of flattened in-frame index x."""
    c, s = ctypes.c_int(), ctypes.c_int()
    _check(lib().oracle1d_index_map(x, P, mode, ctypes.byref(c), ctypes.byref(s)), "index_map_1d")
    return c.value, s.value


def axis_map(x: int, P: int, mode: int):
    c, s = ctypes.c_int(), ctypes.c_int()
    _check(lib().oracle_axis_map(x, P, mode, ctypes.byref(c), ctypes.byref(s)), "axis_map")
    return c.value, s.value


def subseq_len(T: int, H: int, W: int, P: int, dims: int = 2) -> int:
    return _fn("subseq_len", dims)(T, H, W, P)


def rearrange(x, P: int, mode: int, with_valid: bool = False, dims: int = 2):
    """x (B,T,H,W,heads,d) bf16 -> (B*P*P, n, heads, d) uint16 bit patterns."""
    xb = _bits(x)
    B, T, H, W, heads, d = xb.shape
    n = subseq_len(T, H, W, P, dims)
    y = np.empty((B * P * P, n, heads, d), dtype=np.uint16)
    valid = np.empty((B * P * P, n), dtype=np.uint8)
    _check(_fn("rearrange", dims)(_ptr(xb), _ptr(y), _ptr(valid), B, T, H, W, heads, d, P, mode),
           "rearrange")
    return (y, valid) if with_valid else y


def unrearrange(y, shape, P: int, mode: int, dims: int = 2):
    yb = _bits(y)
    B, T, H, W, heads, d = shape
    x = np.empty(shape, dtype=np.uint16)
    _check(_fn("unrearrange", dims)(_ptr(yb), _ptr(x), B, T, H, W, heads, d, P, mode),
           "unrearrange")
    return x


def switch_mode(y, shape, P: int, src_mode: int, dims: int = 2):
    """src_mode's rearranged layout -> the other mode's rearranged layout (bit patterns)."""
    yb = _bits(y)
    B, T, H, W, heads, d = shape
    out = np.empty_like(yb)
    _check(_fn("switch_mode", dims)(_ptr(yb), _ptr(out), B, T, H, W, heads, d, P, src_mode),
           "switch_mode")
    return out


def unrearrange_f64(y: np.ndarray, shape, P: int, mode: int, dims: int = 2):
    y = np.ascontiguousarray(y, dtype=np.float64)
    B, T, H, W, heads, d = shape
    x = np.empty(shape, dtype=np.float64)
    _check(_fn("unrearrange_f64", dims)(_ptr(y), _ptr(x), B, T, H, W, heads, d, P, mode),
           "unrearrange_f64")
    return x


def masked_attention(yq, yk, yv, valid, nthreads: int | None = None):
    yq, yk, yv = _bits(yq), _bits(yk), _bits(yv)
    valid = np.ascontiguousarray(valid, dtype=np.uint8)
    nseq, n, heads, d = yq.shape
    yo = np.zeros((nseq, n, heads, d), dtype=np.float64)
    _check(lib().oracle_masked_attention(_ptr(yq), _ptr(yk), _ptr(yv), _ptr(valid), _ptr(yo),
                                         nseq, n, heads, d, nthreads or default_threads()),
           "masked_attention")
    return yo


def attn_fwd(q, k, v, P: int, mode: int, nthreads: int | None = None, dims: int = 2) -> np.ndarray:
    """Full Skiparse-2D (dims=2) or Skiparse-1D (dims=1) forward in fp64; returns
    (B,T,H,W,heads,d) float64."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, T, H, W, heads, d = qb.shape
    out = np.empty(qb.shape, dtype=np.float64)
    _check(_fn("attn_fwd", dims)(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(out), B, T, H, W, heads, d,
                                 P, mode, nthreads or default_threads()), "attn_fwd")
    return out


def attn_fwd_rows(q, k, v, rows, P: int, mode: int, nthreads: int | None = None,
                  dims: int = 2) -> np.ndarray:
    """Forward for selected rows (token*heads + head of the original layout); (nrows, d)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, T, H, W, heads, d = qb.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.zeros((rows.shape[0], d), dtype=np.float64)
    _check(_fn("attn_fwd_rows", dims)(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(rows), rows.shape[0],
                                      _ptr(out), B, T, H, W, heads, d, P, mode,
                                      nthreads or default_threads()), "attn_fwd_rows")
    return out


def attn_bwd(q, k, v, dout, P: int, mode: int, nthreads: int | None = None, dims: int = 2):
    """Backward pass in fp64: returns (dq, dk, dv, lse); lse is the natural-log log-sum-exp of
    q.k/sqrt(d) over each token's class, shape (B,T,H,W,heads)."""
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, T, H, W, heads, d = qb.shape
    dq, dk, dv = (np.empty(qb.shape, dtype=np.float64) for _ in range(3))
    lse = np.empty((B, T, H, W, heads), dtype=np.float64)
    _check(_fn("attn_bwd", dims)(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gb), _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(lse), B, T, H, W, heads, d, P, mode, nthreads or default_threads()),
           "attn_bwd")
    return dq, dk, dv, lse


def attn_bwd_rows(q, k, v, dout, rows, P: int, mode: int, nthreads: int | None = None,
                  dims: int = 2):
    """Backward for selected rows (token*heads + head): (dq, dk, dv), each (nrows, d) fp64."""
    qb, kb, vb, gb = _bits(q), _bits(k), _bits(v), _bits(dout)
    B, T, H, W, heads, d = qb.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    dq, dk, dv = (np.zeros((rows.shape[0], d), dtype=np.float64) for _ in range(3))
    _check(_fn("attn_bwd_rows", dims)(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gb), _ptr(rows), rows.shape[0],
                                      _ptr(dq), _ptr(dk), _ptr(dv), B, T, H, W, heads, d, P, mode,
                                      nthreads or default_threads()), "attn_bwd_rows")
    return dq, dk, dv
