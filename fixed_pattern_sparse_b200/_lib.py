"""ctypes loader for libskiparse.so (the C ABI in include/skiparse.h).

The library is built in-tree by ``python -m fixed_pattern_sparse_b200.build``. There is no
fallback: if the library is missing or fails to load, importing the binding raises.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libskiparse.so")
# The bounds-checking debug build of the same library (SKIPARSE_DEBUG=1), for tests and for
# hunting an out-of-range access: `python -m fixed_pattern_sparse_b200.build --debug`.
DEBUG_LIB_PATH = os.path.join(HERE, "libskiparse_debug.so")

# Every symbol include/skiparse.h declares, with (restype, argtypes).
_I, _LL, _ULL, _VP, _CP = ctypes.c_int, ctypes.c_longlong, ctypes.c_ulonglong, ctypes.c_void_p, ctypes.c_char_p
SIGNATURES = {
    "skiparse2d_attn_fwd": (_I, [_VP, _VP, _VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse2d_attn_fwd_lse": (_I, [_VP, _VP, _VP, _VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse2d_attn_bwd": (_I, [_VP] * 10 + [_I] * 8 + [_VP]),
    "skiparse2d_attn_bwd_noalloc": (_I, [_VP] * 9 + [_I] * 8 + [_VP]),
    "skiparse_rearrange": (_I, [_VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse_unrearrange": (_I, [_VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse_switch_mode": (_I, [_VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse_rearranged_numel": (_LL, [_I] * 7),
    "skiparse_padded_extent": (_I, [_I, _I]),
    "skiparse_subseq_len": (_LL, [_I] * 4),
    "skiparse_class_len": (_LL, [_I] * 7),
    "skiparse_get_device_status": (_I, [_VP]),
    "skiparse_status_string": (_CP, [_I]),
    "skiparse_version": (_CP, []),
    "skiparse_last_error_string": (_CP, []),
    "skiparse_set_wait_limit_ns": (_ULL, [_ULL]),
    "skiparse_debug_inject_fault": (_I, [_I]),
    "skiparse_debug_shrink_bounds": (_I, [_LL]),
    "skiparse_debug_exp2": (_I, [_VP, _VP, _LL, _I, _VP]),
    "skiparse_debug_mma_rate": (_I, [_I, _I, _VP, _I, _VP]),
    "skiparse_debug_softmax_rate": (_I, [_I, _I, _VP, _I, _VP]),
    "skiparse1d_attn_fwd": (_I, [_VP, _VP, _VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse1d_attn_fwd_lse": (_I, [_VP, _VP, _VP, _VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse1d_attn_bwd": (_I, [_VP] * 10 + [_I] * 8 + [_VP]),
    "skiparse1d_rearrange": (_I, [_VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse1d_unrearrange": (_I, [_VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse1d_switch_mode": (_I, [_VP, _VP] + [_I] * 8 + [_VP]),
    "skiparse1d_padded_length": (_LL, [_LL, _I]),
    "skiparse1d_subseq_len": (_LL, [_I] * 4),
    "skiparse1d_class_len": (_LL, [_I] * 6),
    "skiparse1d_rearranged_numel": (_LL, [_I] * 7),
    "skiparse2d_attn_fwd_host": (_I, [_VP] * 4 + [_I] * 9 + [_VP, ctypes.c_size_t, _VP]),
    "skiparse1d_attn_fwd_host": (_I, [_VP] * 4 + [_I] * 9 + [_VP, ctypes.c_size_t, _VP]),
    "skiparse_attn_fwd_host_workspace_bytes": (_LL, [_I] * 7),
}

STATUS = {0: "SKIPARSE_OK", 1: "SKIPARSE_ERR_INVALID_ARG", 2: "SKIPARSE_ERR_UNSUPPORTED",
          3: "SKIPARSE_ERR_MISALIGNED", 4: "SKIPARSE_ERR_CUDA", 5: "SKIPARSE_ERR_TIMEOUT",
          6: "SKIPARSE_ERR_BOUNDS"}


class SkiparseError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what} failed: {STATUS.get(code, code)}")
        self.code = code


_LIB = None


_DEBUG_LIB = None


def _load(path: str, how: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `{how}` (there is no CPU or library fallback)")
    L = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = _load(LIB_PATH, "python -m fixed_pattern_sparse_b200.build")
    return _LIB


def debug_lib() -> ctypes.CDLL:
    """The bounds-checking debug build, bound like lib() (separate library, separate state)."""
    global _DEBUG_LIB
    if _DEBUG_LIB is None:
        _DEBUG_LIB = _load(DEBUG_LIB_PATH, "python -m fixed_pattern_sparse_b200.build --debug")
    return _DEBUG_LIB


def check(code: int, what: str) -> None:
    if code != 0:
        err = SkiparseError(code, what)
        if code == 4:  # SKIPARSE_ERR_CUDA: add the CUDA message
            err.args = (f"{err.args[0]} ({lib().skiparse_last_error_string().decode()})",)
        raise err
