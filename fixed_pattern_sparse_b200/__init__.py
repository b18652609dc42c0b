"""Skiparse-2D (and Skiparse-1D) sparse attention on NVIDIA B200 -- Python binding of
libskiparse.so.

Every function here only marshals arguments (device pointers, sizes, the current CUDA
stream) into the C ABI declared in include/skiparse.h; all of the work runs in the
library's sm_100a kernels. PyTorch provides device memory and streams only. There is no
CPU fallback: without a CUDA device or without the built library these functions raise.
"""

from __future__ import annotations

import torch

from ._lib import STATUS, SkiparseError, check, lib

TOKEN_WISE = 0
GROUP_WISE = 1

__all__ = ["TOKEN_WISE", "GROUP_WISE", "SkiparseError", "skiparse2d_attn_fwd", "skiparse_rearrange",
           "skiparse_unrearrange", "skiparse_switch_mode", "rearranged_shape", "padded_extent", "subseq_len", "class_len",
           "get_device_status", "attn_fwd_from_host", "HostStaging", "attn_flops", "STATUS",
           "skiparse2d_attn_fwd_lse", "skiparse2d_attn_bwd", "SkiparseAttention", "skiparse_attention",
           "skiparse1d_attn_fwd", "skiparse1d_attn_fwd_lse", "skiparse1d_attn_bwd", "skiparse1d_rearrange",
           "skiparse1d_unrearrange", "skiparse1d_switch_mode", "padded_length_1d", "attn_fwd_host",
           "host_workspace_bytes"]


def _stream_ptr(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _need_cuda_bf16(name: str, t: torch.Tensor) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def padded_extent(X: int, P: int) -> int:
    return lib().skiparse_padded_extent(X, P)


def subseq_len(T: int, H: int, W: int, P: int) -> int:
    return lib().skiparse_subseq_len(T, H, W, P)


def class_len(T: int, H: int, W: int, P: int, mode: int, ci: int, cj: int) -> int:
    return lib().skiparse_class_len(T, H, W, P, mode, ci, cj)


def padded_length_1d(L: int, P: int) -> int:
    """Skiparse-1D: per-frame length H*W padded to the next multiple of P^4."""
    return lib().skiparse1d_padded_length(L, P)


def subseq_len_1d(T: int, H: int, W: int, P: int) -> int:
    return lib().skiparse1d_subseq_len(T, H, W, P)


def class_len_1d(T: int, H: int, W: int, P: int, mode: int, c: int) -> int:
    return lib().skiparse1d_class_len(T, H, W, P, mode, c)


def rearranged_shape(shape, P: int, dims: int = 2):
    B, T, H, W, heads, d = shape
    n = subseq_len(T, H, W, P) if dims == 2 else subseq_len_1d(T, H, W, P)
    return (B * P * P, n, heads, d)


def attn_flops(shape, P: int, dims: int = 2) -> float:
    """FLOPs of one call by the padded formula 4 * N * (N / P^2) * d * heads * B, N the padded
    token count: T * Hp * Wp (Skiparse-2D) or T * Lp (Skiparse-1D)."""
    B, T, H, W, heads, d = shape
    if dims == 2:
        N = T * padded_extent(H, P) * padded_extent(W, P)
    else:
        N = T * padded_length_1d(H * W, P)
    return 4.0 * N * (N / (P * P)) * d * heads * B


def _entry(name: str, dims: int):
    if dims not in (1, 2):
        raise ValueError("dims must be 1 (Skiparse-1D) or 2 (Skiparse-2D)")
    return getattr(lib(), name.replace("@", "1d" if dims == 1 else "2d"))


def _check_qkv(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda_bf16(name, t)
    if q.dim() != 6 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one (B,T,H,W,heads,d) shape")


def _attn_fwd(dims, q, k, v, P, mode, out, stream):
    _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    _need_cuda_bf16("out", out)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    B, T, H, W, heads, d = q.shape
    name = "skiparse@_attn_fwd"
    check(_entry(name, dims)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             B, T, H, W, heads, d, P, mode, _stream_ptr(stream)),
          name.replace("@", f"{dims}d"))
    return out


def _attn_fwd_lse(dims, q, k, v, P, mode, out, lse, stream):
    _check_qkv(q, k, v)
    out = torch.empty_like(q) if out is None else out
    _need_cuda_bf16("out", out)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    if lse is None:
        lse = torch.empty(q.shape[:5], dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or tuple(lse.shape) != tuple(q.shape[:5]) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 (B,T,H,W,heads) tensor")
    B, T, H, W, heads, d = q.shape
    name = "skiparse@_attn_fwd_lse"
    check(_entry(name, dims)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             B, T, H, W, heads, d, P, mode, _stream_ptr(stream)),
          name.replace("@", f"{dims}d"))
    return out, lse


def _attn_bwd(dims, q, k, v, out, dout, lse, P, mode, dq, dk, dv, delta, stream):
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        _need_cuda_bf16(name, t)
        if t.shape != q.shape:
            raise ValueError(f"{name} must have q's shape")
    if lse.dtype != torch.float32 or tuple(lse.shape) != tuple(q.shape[:5]) or not lse.is_cuda:
        raise ValueError("lse must be a CUDA fp32 (B,T,H,W,heads) tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    delta = torch.empty(q.shape[:5], dtype=torch.float32, device=q.device) if delta is None else delta
    B, T, H, W, heads, d = q.shape
    name = "skiparse@_attn_bwd"
    check(_entry(name, dims)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                             lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), delta.data_ptr(),
                             B, T, H, W, heads, d, P, mode, _stream_ptr(stream)),
          name.replace("@", f"{dims}d"))
    return dq, dk, dv


def skiparse2d_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, P: int, mode: int,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Fused Skiparse-2D attention forward; q/k/v/out are (B,T,H,W,heads,d) bf16 on CUDA."""
    return _attn_fwd(2, q, k, v, P, mode, out, stream)


def skiparse1d_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, P: int, mode: int,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Fused Skiparse-1D attention forward (class rule on the flattened in-frame index)."""
    return _attn_fwd(1, q, k, v, P, mode, out, stream)


def skiparse2d_attn_fwd_lse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, P: int, mode: int,
                            out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Forward that also returns lse (B,T,H,W,heads) fp32, the natural-log log-sum-exp of
    q.k/sqrt(d) over each token's class, for the backward pass."""
    return _attn_fwd_lse(2, q, k, v, P, mode, out, lse, stream)


def skiparse1d_attn_fwd_lse(q, k, v, P: int, mode: int, out=None, lse=None, stream=None):
    """Skiparse-1D forward that also returns lse, as skiparse2d_attn_fwd_lse."""
    return _attn_fwd_lse(1, q, k, v, P, mode, out, lse, stream)


def skiparse2d_attn_bwd(q, k, v, out, dout, lse, P: int, mode: int, dq=None, dk=None, dv=None, delta=None,
                        stream=None):
    """Backward pass: returns (dq, dk, dv), bf16 (B,T,H,W,heads,d). `delta` is an optional fp32
    (B,T,H,W,heads) workspace (allocated here when not given)."""
    return _attn_bwd(2, q, k, v, out, dout, lse, P, mode, dq, dk, dv, delta, stream)


def skiparse1d_attn_bwd(q, k, v, out, dout, lse, P: int, mode: int, dq=None, dk=None, dv=None, delta=None,
                        stream=None):
    """Skiparse-1D backward pass, as skiparse2d_attn_bwd."""
    return _attn_bwd(1, q, k, v, out, dout, lse, P, mode, dq, dk, dv, delta, stream)


class SkiparseAttention(torch.autograd.Function):
    """Differentiable Skiparse attention (dims=2: Skiparse-2D, dims=1: Skiparse-1D): forward and
    backward both run the sm_100a kernels."""

    @staticmethod
    def forward(ctx, q, k, v, P: int, mode: int, dims: int = 2):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        out, lse = _attn_fwd_lse(dims, q, k, v, P, mode, None, None, None)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.P, ctx.mode, ctx.dims = P, mode, dims
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = _attn_bwd(ctx.dims, q, k, v, out, dout.contiguous(), lse, ctx.P, ctx.mode,
                               None, None, None, None, None)
        return dq, dk, dv, None, None, None


def skiparse_attention(q, k, v, P: int, mode: int, dims: int = 2):
    """Autograd-aware Skiparse attention on (B,T,H,W,heads,d) bf16 CUDA tensors."""
    return SkiparseAttention.apply(q, k, v, P, mode, dims)


def _rearrange(dims, x, P, mode, out, stream):
    _need_cuda_bf16("x", x)
    if x.dim() != 6:
        raise ValueError("x must be (B,T,H,W,heads,d)")
    shape = rearranged_shape(x.shape, P, dims)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=x.device)
    _need_cuda_bf16("out", out)
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out must have shape {shape}")
    B, T, H, W, heads, d = x.shape
    name = "skiparse_rearrange" if dims == 2 else "skiparse1d_rearrange"
    check(getattr(lib(), name)(x.data_ptr(), out.data_ptr(), B, T, H, W, heads, d, P, mode,
                               _stream_ptr(stream)), name)
    return out


def _unrearrange(dims, y, shape, P, mode, out, stream):
    _need_cuda_bf16("y", y)
    shape = tuple(int(s) for s in shape)
    if tuple(y.shape) != tuple(rearranged_shape(shape, P, dims)):
        raise ValueError("y does not match the rearranged shape of `shape`")
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=y.device)
    _need_cuda_bf16("out", out)
    if tuple(out.shape) != shape:
        raise ValueError(f"out must have shape {shape}")
    B, T, H, W, heads, d = shape
    name = "skiparse_unrearrange" if dims == 2 else "skiparse1d_unrearrange"
    check(getattr(lib(), name)(y.data_ptr(), out.data_ptr(), B, T, H, W, heads, d, P, mode,
                               _stream_ptr(stream)), name)
    return out


def _switch_mode(dims, y, shape, P, src_mode, out, stream):
    _need_cuda_bf16("y", y)
    shape = tuple(int(s) for s in shape)
    rshape = tuple(rearranged_shape(shape, P, dims))
    if tuple(y.shape) != rshape:
        raise ValueError("y does not match the rearranged shape of `shape`")
    if out is None:
        out = torch.empty(rshape, dtype=torch.bfloat16, device=y.device)
    _need_cuda_bf16("out", out)
    if tuple(out.shape) != rshape:
        raise ValueError(f"out must have shape {rshape}")
    B, T, H, W, heads, d = shape
    name = "skiparse_switch_mode" if dims == 2 else "skiparse1d_switch_mode"
    check(getattr(lib(), name)(y.data_ptr(), out.data_ptr(), B, T, H, W, heads, d, P, src_mode,
                               _stream_ptr(stream)), name)
    return out


def skiparse_rearrange(x: torch.Tensor, P: int, mode: int, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """Skiparse-2D: (B,T,H,W,heads,d) -> (B*P*P, n, heads, d), pad slots zero."""
    return _rearrange(2, x, P, mode, out, stream)


def skiparse_unrearrange(y: torch.Tensor, shape, P: int, mode: int, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Skiparse-2D: (B*P*P, n, heads, d) -> (B,T,H,W,heads,d); pad slots are dropped."""
    return _unrearrange(2, y, shape, P, mode, out, stream)


def skiparse_switch_mode(y: torch.Tensor, shape, P: int, src_mode: int, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Skiparse-2D: src_mode's rearranged layout -> the other mode's rearranged layout (pads zero)."""
    return _switch_mode(2, y, shape, P, src_mode, out, stream)


def skiparse1d_rearrange(x: torch.Tensor, P: int, mode: int, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Skiparse-1D: (B,T,H,W,heads,d) -> (B*P*P, n, heads, d), n = T*Lp/P^2, pad slots zero."""
    return _rearrange(1, x, P, mode, out, stream)


def skiparse1d_unrearrange(y: torch.Tensor, shape, P: int, mode: int, out: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """Skiparse-1D inverse rearrange; pad slots are dropped."""
    return _unrearrange(1, y, shape, P, mode, out, stream)


def skiparse1d_switch_mode(y: torch.Tensor, shape, P: int, src_mode: int, out: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """Skiparse-1D: src_mode's rearranged layout -> the other mode's (pads zero)."""
    return _switch_mode(1, y, shape, P, src_mode, out, stream)


def get_device_status(stream=None) -> int:
    """Synchronizes the stream; returns and clears the device error word (0 = OK)."""
    return lib().skiparse_get_device_status(_stream_ptr(stream))


def host_workspace_bytes(shape, heads_per_group: int) -> int:
    B, T, H, W, heads, d = shape
    return lib().skiparse_attn_fwd_host_workspace_bytes(B, T, H, W, heads, d, heads_per_group)


def attn_fwd_host(q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor, P: int, mode: int,
                  out_host: torch.Tensor, heads_per_group: int = 8, workspace: torch.Tensor | None = None,
                  dims: int = 2, stream=None) -> torch.Tensor:
    """The forward with HOST buffers (skiparse2d_attn_fwd_host / skiparse1d_attn_fwd_host): q, k, v
    and out are CPU bf16 tensors of one (B,T,H,W,heads,d) shape (pinned memory lets the library
    overlap its copies with the kernel); `workspace` is a CUDA uint8 tensor of at least
    host_workspace_bytes(shape, heads_per_group) bytes (allocated here when not given).
    Asynchronous on `stream`: synchronize it before reading out_host."""
    for name, t in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host), ("out_host", out_host)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor")
        if t.shape != q_host.shape or t.dim() != 6:
            raise ValueError("q, k, v, out must share one (B,T,H,W,heads,d) shape")
    B, T, H, W, heads, d = q_host.shape
    need = host_workspace_bytes(q_host.shape, heads_per_group)
    if need < 0:
        raise ValueError("invalid shape or heads_per_group")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    if not workspace.is_cuda or workspace.dtype != torch.uint8 or workspace.numel() < need:
        raise ValueError(f"workspace must be a CUDA uint8 tensor of at least {need} bytes")
    name = "skiparse2d_attn_fwd_host" if dims == 2 else "skiparse1d_attn_fwd_host"
    check(getattr(lib(), name)(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), out_host.data_ptr(),
                               B, T, H, W, heads, d, P, mode, heads_per_group, workspace.data_ptr(),
                               workspace.numel(), _stream_ptr(stream)), name)
    return out_host


class HostStaging:
    """Device buffers reused by attn_fwd_from_host (allocated once, by torch)."""

    def __init__(self, shape, device="cuda"):
        self.shape = tuple(shape)
        self.q, self.k, self.v, self.out = (torch.empty(self.shape, dtype=torch.bfloat16, device=device)
                                            for _ in range(4))


def attn_fwd_from_host(q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor, P: int,
                       mode: int, out_host: torch.Tensor, staging: HostStaging, stream=None,
                       dims: int = 2) -> torch.Tensor:
    """End-to-end call from host memory: copy q/k/v (pinned CPU tensors) to the device, run the
    fused kernel, copy the output back into out_host (pinned). Asynchronous on `stream`."""
    s = torch.cuda.current_stream() if stream is None else stream
    with torch.cuda.stream(s):
        staging.q.copy_(q_host, non_blocking=True)
        staging.k.copy_(k_host, non_blocking=True)
        staging.v.copy_(v_host, non_blocking=True)
        _attn_fwd(dims, staging.q, staging.k, staging.v, P, mode, staging.out, s)
        out_host.copy_(staging.out, non_blocking=True)
    return out_host
