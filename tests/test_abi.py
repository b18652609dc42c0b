"""C-ABI checks that need no GPU: the library loads, exports every symbol the header
declares, computes the Skiparse geometry, and rejects bad arguments synchronously
(before any CUDA call)."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

import oracle
from fixed_pattern_sparse_b200 import _lib
from fixed_pattern_sparse_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "skiparse.h")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^SKIPARSE_API [^(]*?\b(skiparse\w*)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("skiparse2d_attn_fwd", "skiparse_rearrange", "skiparse_unrearrange",
                 "skiparse_get_device_status", "skiparse_status_string"):
        assert must in names
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_exports_are_only_the_c_abi():
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {n for n in exported if n.startswith("skiparse")}
    assert ours == set(declared_functions())


def test_status_strings(L):
    for code, name in _lib.STATUS.items():
        assert L.skiparse_status_string(code).decode() == name
    assert L.skiparse_status_string(99).decode() == "SKIPARSE_ERR_UNKNOWN"
    assert b"sm_100a" in L.skiparse_version()


@pytest.mark.parametrize("X,P", [(45, 2), (80, 2), (48, 3), (84, 3), (1, 2), (13, 4), (7, 1), (100, 8)])
def test_padded_extent_matches_oracle(L, X, P):
    assert L.skiparse_padded_extent(X, P) == oracle.padded_extent(X, P)


def test_geometry_matches_oracle(L):
    """Real per-class token counts of the product's geometry against the oracle's rearrange."""
    import numpy as np
    for (T, H, W, P) in [(2, 8, 8, 2), (3, 10, 14, 2), (1, 5, 7, 3), (2, 3, 20, 4), (1, 45, 80, 2),
                         (1, 48, 84, 3), (2, 6, 5, 1)]:
        assert L.skiparse_subseq_len(T, H, W, P) == oracle.subseq_len(T, H, W, P)
        for mode in (0, 1):
            x = (np.arange(T * H * W, dtype=np.uint16) + 1).reshape(1, T, H, W, 1, 1)
            y = oracle.rearrange(x, P, mode)
            for ci in range(P):
                for cj in range(P):
                    real = int((y[ci * P + cj, :, 0, 0] > 0).sum())
                    assert L.skiparse_class_len(T, H, W, P, mode, ci, cj) == real
        n = L.skiparse_rearranged_numel(2, T, H, W, 3, 64, P)
        assert n == 2 * P * P * oracle.subseq_len(T, H, W, P) * 3 * 64


def test_geometry_1d_matches_oracle(L):
    """Skiparse-1D: padded length, subsequence length and real per-class counts of the product's
    geometry against the oracle's 1D rearrange."""
    import numpy as np
    for L_, P in [(1, 2), (15, 2), (16, 2), (17, 2), (3600, 2), (1560, 2), (81, 3), (4032, 8), (5, 1)]:
        assert L.skiparse1d_padded_length(L_, P) == oracle.padded_length_1d(L_, P)
    for (T, H, W, P) in [(2, 8, 8, 2), (3, 10, 14, 2), (1, 5, 7, 3), (2, 3, 20, 4), (1, 45, 80, 2),
                         (1, 30, 52, 2), (2, 6, 5, 1), (1, 1, 1, 2)]:
        assert L.skiparse1d_subseq_len(T, H, W, P) == oracle.subseq_len(T, H, W, P, dims=1)
        for mode in (0, 1):
            x = (np.arange(T * H * W, dtype=np.uint16) + 1).reshape(1, T, H, W, 1, 1)
            y = oracle.rearrange(x, P, mode, dims=1)
            for c in range(P * P):
                real = int((y[c, :, 0, 0] > 0).sum())
                assert L.skiparse1d_class_len(T, H, W, P, mode, c) == real
            assert L.skiparse1d_class_len(T, H, W, P, mode, P * P) == -1
        n = L.skiparse1d_rearranged_numel(2, T, H, W, 3, 64, P)
        assert n == 2 * P * P * oracle.subseq_len(T, H, W, P, dims=1) * 3 * 64


def test_1d_entries_reject_bad_arguments_synchronously(L):
    assert L.skiparse1d_attn_fwd(0, FAKE, FAKE, FAKE + 4096, 1, 2, 8, 8, 2, 32, 2, 0, None) == 1
    assert L.skiparse1d_attn_fwd(FAKE, FAKE, FAKE, FAKE + (1 << 20), 1, 2, 8, 8, 2, 32, 9, 0, None) == 2
    assert L.skiparse1d_attn_fwd(FAKE, FAKE, FAKE, FAKE + (1 << 20), 1, 2, 8, 8, 2, 32, 2, 3, None) == 1
    assert L.skiparse1d_attn_fwd_lse(FAKE, FAKE, FAKE, FAKE + (1 << 20), 0, 1, 2, 8, 8, 2, 32, 2, 0,
                                     None) == 1
    assert L.skiparse1d_attn_bwd(*([FAKE] * 9), 0, 1, 2, 8, 8, 2, 32, 2, 0, None) == 1
    assert L.skiparse1d_rearrange(FAKE, FAKE + 4, 1, 2, 8, 8, 2, 32, 2, 0, None) == 3
    assert L.skiparse1d_unrearrange(FAKE, FAKE + 64, 1, 2, 8, 8, 2, 32, 2, 0, None) == 1
    assert L.skiparse1d_switch_mode(FAKE, FAKE, 1, 2, 8, 8, 2, 32, 2, 0, None) == 1
    # padded rows past 2^31: 1D pads each frame to a multiple of P^4 = 4096
    assert L.skiparse1d_rearrange(FAKE, FAKE + (1 << 40), 1, 1 << 16, 1, 1, 8192, 32, 8, 0, None) == 2


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case below fails before any CUDA call


@pytest.mark.parametrize("args,code", [
    ((0, FAKE, FAKE, FAKE + 4096, 1, 2, 8, 8, 2, 32, 2, 0), 1),          # null q
    ((FAKE, FAKE, FAKE, FAKE + (1 << 20), 1, 2, 8, 8, 2, 48, 2, 0), 2),   # d = 48 unsupported
    ((FAKE, FAKE, FAKE, FAKE + (1 << 20), 1, 2, 8, 8, 2, 32, 9, 0), 2),   # P = 9 unsupported
    ((FAKE, FAKE, FAKE, FAKE + (1 << 20), 1, 2, 8, 8, 2, 32, 2, 2), 1),   # bad mode
    ((FAKE, FAKE, FAKE, FAKE + (1 << 20), 0, 2, 8, 8, 2, 32, 2, 0), 1),   # B = 0
    ((FAKE, FAKE, FAKE, FAKE + (1 << 20), 1, 2, -8, 8, 2, 32, 2, 0), 1),  # negative H
    ((FAKE + 8, FAKE, FAKE, FAKE + (1 << 20), 1, 2, 8, 8, 2, 32, 2, 0), 3),  # misaligned q
    ((FAKE, FAKE, FAKE, FAKE + 2, 1, 2, 8, 8, 2, 32, 2, 0), 3),           # misaligned out
    ((FAKE, FAKE + (1 << 20), FAKE + (2 << 20), FAKE, 1, 2, 8, 8, 2, 32, 2, 0), 1),  # out aliases q
    ((FAKE, FAKE, FAKE, FAKE + 4096, 1, 2, 8, 8, 2, 32, 2, 0), 1),        # out overlaps q's range
    ((FAKE, FAKE, FAKE, FAKE + (1 << 30), 64, 21, 480, 840, 40, 128, 2, 0), 2),  # > 2^31 rows
])
def test_attn_fwd_rejects_bad_arguments_synchronously(L, args, code):
    assert L.skiparse2d_attn_fwd(*args, None) == code


def test_noalloc_backward_rejects_bad_arguments_before_any_cuda_call(L):
    """The allocation-free backward checks its arguments first, with the regular backward's
    codes, and its workspace capacity next; on this host (no GPU) any CUDA call would fail with
    SKIPARSE_ERR_CUDA instead."""
    f = L.skiparse2d_attn_bwd_noalloc
    good = (1, 2, 8, 8, 2, 32, 2, 0)
    assert f(0, *([FAKE] * 8), *good, None) == 1                       # null q
    assert f(*([FAKE] * 8), 0, *good, None) == 1                       # null dv
    assert f(*([FAKE] * 9), 1, 2, 8, 8, 2, 32, 2, 2, None) == 1        # bad mode
    assert f(*([FAKE] * 9), 0, 2, 8, 8, 2, 32, 2, 0, None) == 1        # B = 0
    assert f(*([FAKE] * 9), 1, 2, 8, 8, 2, 48, 2, 0, None) == 2        # d = 48
    assert f(*([FAKE] * 9), 1, 2, 8, 8, 2, 32, 9, 0, None) == 2        # P = 9
    assert f(*([FAKE] * 9), 1, 1, 1, (1 << 22) + 1, 1, 32, 2, 0, None) == 2  # beyond the workspace


def test_mma_rate_diagnostic_rejects_bad_arguments_synchronously(L):
    assert L.skiparse_debug_mma_rate(7, 8, FAKE, 148, None) == 1
    assert L.skiparse_debug_mma_rate(0, 0, FAKE, 148, None) == 1
    assert L.skiparse_debug_mma_rate(0, 8, 0, 148, None) == 1
    assert L.skiparse_debug_mma_rate(0, 1 << 20, FAKE, 148, None) == 2
    assert L.skiparse_debug_mma_rate(0, 8, FAKE + 4, 148, None) == 3


def test_rearrange_rejects_bad_arguments_synchronously(L):
    assert L.skiparse_rearrange(0, FAKE, 1, 2, 8, 8, 2, 32, 2, 0, None) == 1
    assert L.skiparse_rearrange(FAKE, FAKE + 4, 1, 2, 8, 8, 2, 32, 2, 0, None) == 3
    assert L.skiparse_rearrange(FAKE, FAKE, 1, 2, 8, 8, 2, 32, 2, 0, None) == 1  # in place
    assert L.skiparse_unrearrange(FAKE, FAKE + 64, 1, 2, 8, 8, 2, 32, 2, 0, None) == 1  # overlap
    assert L.skiparse_unrearrange(FAKE, FAKE + (1 << 20), 1, 2, 8, 8, 2, 40, 2, 0, None) == 2


def test_wait_limit_and_fault_hook(L):
    prev = L.skiparse_set_wait_limit_ns(123456)
    assert prev == 2_000_000_000
    assert L.skiparse_set_wait_limit_ns(0) == 123456
    assert L.skiparse_set_wait_limit_ns(0) == 2_000_000_000
    assert L.skiparse_debug_inject_fault(3) == 1
    assert L.skiparse_debug_inject_fault(2) == 0  # the backward's hook
    assert L.skiparse_debug_inject_fault(0) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    import fixed_pattern_sparse_b200 as fps
    x = torch.zeros((1, 1, 4, 4, 1, 32), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fps.skiparse2d_attn_fwd(x, x, x, 2, 0)
    with pytest.raises(ValueError):
        fps.skiparse_rearrange(x, 2, 0)


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "fixed_pattern_sparse_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower().replace("oracles", ""), f


def test_host_entry_rejects_bad_arguments_synchronously(L):
    """The host-buffer forward validates everything before it creates streams or enqueues."""
    need = L.skiparse_attn_fwd_host_workspace_bytes(1, 2, 8, 8, 4, 32, 2)
    assert need > 0
    assert L.skiparse_attn_fwd_host_workspace_bytes(1, 2, 8, 8, 4, 32, 5) == -1   # group > heads
    big = 1 << 40
    args = (FAKE, FAKE + big, FAKE + 2 * big, FAKE + 3 * big, 1, 2, 8, 8, 4, 32, 2, 0)
    assert L.skiparse2d_attn_fwd_host(*args, 2, FAKE + 4 * big, need - 1, None) == 1     # workspace small
    assert L.skiparse2d_attn_fwd_host(*args, 0, FAKE + 4 * big, need, None) == 1         # group 0
    assert L.skiparse2d_attn_fwd_host(*args, 2, FAKE + 4 * big + 16, need, None) == 3    # misaligned
    assert L.skiparse2d_attn_fwd_host(*args[:10], 2, 7, 2, FAKE + 4 * big, need, None) == 1  # bad mode
    assert L.skiparse2d_attn_fwd_host(*args[:9], 48, 2, 0, 2, FAKE + 4 * big, 1 << 40, None) == 2  # d = 48
    over = (FAKE, FAKE + big, FAKE + 2 * big, FAKE + 64, 1, 2, 8, 8, 4, 32, 2, 0)       # out overlaps q
    assert L.skiparse2d_attn_fwd_host(*over, 2, FAKE + 4 * big, need, None) == 1
    assert L.skiparse1d_attn_fwd_host(*args, 2, FAKE + 4 * big, need - 1, None) == 1


def test_debug_build_hook_and_exports(L):
    """The bounds-checking debug build exports the same C ABI; only it accepts the hook that
    declares the next launch's bounds smaller (the release build has no checks)."""
    from fixed_pattern_sparse_b200 import _lib
    libbuild.build(debug=True)  # no-op when up to date
    R = L
    assert R.skiparse_debug_shrink_bounds(3) == 2  # SKIPARSE_ERR_UNSUPPORTED
    assert b"debug" not in R.skiparse_version()
    D = _lib.debug_lib()
    for name in _lib.SIGNATURES:
        assert hasattr(D, name), name
    assert b"debug" in D.skiparse_version()
    assert D.skiparse_debug_shrink_bounds(-1) == 1
    assert D.skiparse_debug_shrink_bounds(0) == 0
    assert D.skiparse_status_string(6) == b"SKIPARSE_ERR_BOUNDS"


def test_header_is_plain_c_and_links(L, tmp_path):
    """include/skiparse.h is a C header: a C99 program that includes it compiles with gcc
    (-std=c99 -pedantic), links against libskiparse.so and calls its host-only entry points
    (geometry and status strings; nothing that needs a GPU)."""
    import shutil
    import subprocess
    from fixed_pattern_sparse_b200 import _lib
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "use_abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "skiparse.h"
int main(void) {
    printf("%d %lld %lld %s %s\n", skiparse_padded_extent(45, 2), skiparse_subseq_len(21, 45, 80, 2),
           skiparse_class_len(21, 45, 80, 2, SKIPARSE_GROUP_WISE, 1, 0),
           skiparse_status_string(SKIPARSE_ERR_TIMEOUT), skiparse_status_string(SKIPARSE_ERR_BOUNDS));
    return skiparse2d_attn_fwd(0, 0, 0, 0, 1, 1, 1, 1, 1, 32, 2, 0, 0) == SKIPARSE_ERR_INVALID_ARG ? 0 : 1;
}
''')
    exe = tmp_path / "use_abi"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Werror", str(src), "-I", os.path.dirname(HEADER),
                    "-L", libdir, "-lskiparse", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    # 720p latent, P = 2: H pads 45 -> 48; n = 21 * 24 * 40; group-wise class (1, 0) holds the
    # rows h with (h div 2) mod 2 = 1 below 45 (11 blocks of 4 rows x 2) and 40 of the 80 columns
    assert out[0] == "48" and out[1] == str(21 * 24 * 40) and out[2] == str(21 * 22 * 40)
    assert out[3] == "SKIPARSE_ERR_TIMEOUT" and out[4] == "SKIPARSE_ERR_BOUNDS"


def test_softmax_rate_diagnostic_rejects_bad_arguments_synchronously(L):
    assert L.skiparse_debug_softmax_rate(3, 8, FAKE, 148, None) == 1
    assert L.skiparse_debug_softmax_rate(0, 8, FAKE, 148, None) == 1
    assert L.skiparse_debug_softmax_rate(2, 0, FAKE, 148, None) == 1
    assert L.skiparse_debug_softmax_rate(2, 8, 0, 148, None) == 1
    assert L.skiparse_debug_softmax_rate(2, 8, FAKE, 0, None) == 1
    assert L.skiparse_debug_softmax_rate(2, 1 << 20, FAKE, 148, None) == 2
    assert L.skiparse_debug_softmax_rate(2, 8, FAKE, 2000, None) == 2
    assert L.skiparse_debug_softmax_rate(2, 8, FAKE + 4, 148, None) == 3
