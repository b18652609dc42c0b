"""Skiparse-2D sparse attention on NVIDIA B200 -- Python binding of libskiparse.so.

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
           "skiparse2d_attn_fwd_lse", "skiparse2d_attn_bwd", "SkiparseAttention", "skiparse_attention"]


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


def rearranged_shape(shape, P: int):
    B, T, H, W, heads, d = shape
    return (B * P * P, subseq_len(T, H, W, P), heads, d)


def attn_flops(shape, P: int) -> float:
    """FLOPs of one call by the padded formula 4 * N * (N / P^2) * d * heads * B,
    N = T * Hp * Wp the padded token count."""
    B, T, H, W, heads, d = shape
    N = T * padded_extent(H, P) * padded_extent(W, P)
    return 4.0 * N * (N / (P * P)) * d * heads * B


def skiparse2d_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, P: int, mode: int,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Fused Skiparse-2D attention forward; q/k/v/out are (B,T,H,W,heads,d) bf16 on CUDA."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda_bf16(name, t)
    if q.dim() != 6 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one (B,T,H,W,heads,d) shape")
    if out is None:
        out = torch.empty_like(q)
    _need_cuda_bf16("out", out)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    B, T, H, W, heads, d = q.shape
    check(lib().skiparse2d_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    B, T, H, W, heads, d, P, mode, _stream_ptr(stream)),
          "skiparse2d_attn_fwd")
    return out


def skiparse2d_attn_fwd_lse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, P: int, mode: int,
                            out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
    """Forward that also returns lse (B,T,H,W,heads) fp32, the natural-log log-sum-exp of
    q.k/sqrt(d) over each token's class, for the backward pass."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda_bf16(name, t)
    if q.dim() != 6 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one (B,T,H,W,heads,d) shape")
    out = torch.empty_like(q) if out is None else out
    _need_cuda_bf16("out", out)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    if lse is None:
        lse = torch.empty(q.shape[:5], dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or tuple(lse.shape) != tuple(q.shape[:5]) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 (B,T,H,W,heads) tensor")
    B, T, H, W, heads, d = q.shape
    check(lib().skiparse2d_attn_fwd_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                        B, T, H, W, heads, d, P, mode, _stream_ptr(stream)),
          "skiparse2d_attn_fwd_lse")
    return out, lse


def skiparse2d_attn_bwd(q, k, v, out, dout, lse, P: int, mode: int, dq=None, dk=None, dv=None, delta=None,
                        stream=None):
    """Backward pass: returns (dq, dk, dv), bf16 (B,T,H,W,heads,d). `delta` is an optional fp32
    (B,T,H,W,heads) workspace (allocated here when not given)."""
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
    check(lib().skiparse2d_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                    lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), delta.data_ptr(),
                                    B, T, H, W, heads, d, P, mode, _stream_ptr(stream)), "skiparse2d_attn_bwd")
    return dq, dk, dv


class SkiparseAttention(torch.autograd.Function):
    """Differentiable Skiparse-2D attention: forward and backward both run the sm_100a kernels."""

    @staticmethod
    def forward(ctx, q, k, v, P: int, mode: int):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        out, lse = skiparse2d_attn_fwd_lse(q, k, v, P, mode)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.P, ctx.mode = P, mode
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = skiparse2d_attn_bwd(q, k, v, out, dout.contiguous(), lse, ctx.P, ctx.mode)
        return dq, dk, dv, None, None


def skiparse_attention(q, k, v, P: int, mode: int):
    """Autograd-aware Skiparse-2D attention on (B,T,H,W,heads,d) bf16 CUDA tensors."""
    return SkiparseAttention.apply(q, k, v, P, mode)


def skiparse_rearrange(x: torch.Tensor, P: int, mode: int, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """(B,T,H,W,heads,d) -> (B*P*P, n, heads, d), pad slots zero."""
    _need_cuda_bf16("x", x)
    if x.dim() != 6:
        raise ValueError("x must be (B,T,H,W,heads,d)")
    shape = rearranged_shape(x.shape, P)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=x.device)
    _need_cuda_bf16("out", out)
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out must have shape {shape}")
    B, T, H, W, heads, d = x.shape
    check(lib().skiparse_rearrange(x.data_ptr(), out.data_ptr(), B, T, H, W, heads, d, P, mode,
                                   _stream_ptr(stream)), "skiparse_rearrange")
    return out


def skiparse_unrearrange(y: torch.Tensor, shape, P: int, mode: int, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """(B*P*P, n, heads, d) -> (B,T,H,W,heads,d); pad slots are dropped."""
    _need_cuda_bf16("y", y)
    shape = tuple(int(s) for s in shape)
    if tuple(y.shape) != tuple(rearranged_shape(shape, P)):
        raise ValueError("y does not match the rearranged shape of `shape`")
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=y.device)
    _need_cuda_bf16("out", out)
    B, T, H, W, heads, d = shape
    check(lib().skiparse_unrearrange(y.data_ptr(), out.data_ptr(), B, T, H, W, heads, d, P, mode,
                                     _stream_ptr(stream)), "skiparse_unrearrange")
    return out


def skiparse_switch_mode(y: torch.Tensor, shape, P: int, src_mode: int, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """src_mode's rearranged layout -> the other mode's rearranged layout (pads zero)."""
    _need_cuda_bf16("y", y)
    shape = tuple(int(s) for s in shape)
    rshape = tuple(rearranged_shape(shape, P))
    if tuple(y.shape) != rshape:
        raise ValueError("y does not match the rearranged shape of `shape`")
    if out is None:
        out = torch.empty(rshape, dtype=torch.bfloat16, device=y.device)
    _need_cuda_bf16("out", out)
    if tuple(out.shape) != rshape:
        raise ValueError(f"out must have shape {rshape}")
    B, T, H, W, heads, d = shape
    check(lib().skiparse_switch_mode(y.data_ptr(), out.data_ptr(), B, T, H, W, heads, d, P, src_mode,
                                     _stream_ptr(stream)), "skiparse_switch_mode")
    return out


def get_device_status(stream=None) -> int:
    """Synchronizes the stream; returns and clears the device error word (0 = OK)."""
    return lib().skiparse_get_device_status(_stream_ptr(stream))


class HostStaging:
    """Device buffers reused by attn_fwd_from_host (allocated once, by torch)."""

    def __init__(self, shape, device="cuda"):
        self.shape = tuple(shape)
        self.q, self.k, self.v, self.out = (torch.empty(self.shape, dtype=torch.bfloat16, device=device)
                                            for _ in range(4))


def attn_fwd_from_host(q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor, P: int,
                       mode: int, out_host: torch.Tensor, staging: HostStaging, stream=None) -> torch.Tensor:
    """End-to-end call from host memory: copy q/k/v (pinned CPU tensors) to the device, run the
    fused kernel, copy the output back into out_host (pinned). Asynchronous on `stream`."""
    s = torch.cuda.current_stream() if stream is None else stream
    with torch.cuda.stream(s):
        staging.q.copy_(q_host, non_blocking=True)
        staging.k.copy_(k_host, non_blocking=True)
        staging.v.copy_(v_host, non_blocking=True)
        skiparse2d_attn_fwd(staging.q, staging.k, staging.v, P, mode, out=staging.out, stream=s)
        out_host.copy_(staging.out, non_blocking=True)
    return out_host
