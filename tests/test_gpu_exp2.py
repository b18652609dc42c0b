"""The two exp2 paths of the attention softmax against fp64 exp2 (through the C ABI).

Part of every 32-column chunk of scores takes exp2 as a degree-3 polynomial on the FMA pipe
instead of the MUFU unit. Its coefficients were fitted with the Remez exchange algorithm for
minimax relative error on [-1/2, 1/2]; the bound below is that fit's error (7.5e-5) with fp32
rounding headroom. Both paths are far inside half an ulp of bf16 (2^-9), the precision in
which the probabilities P enter the P*V product."""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def run(x: torch.Tensor, method: int) -> torch.Tensor:
    from fixed_pattern_sparse_b200 import _lib
    y = torch.empty_like(x)
    rc = _lib.lib().skiparse_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), method,
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    return y


def test_exp2_paths_match_fp64():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    xs = np.concatenate([np.linspace(-124.0, 9.0, 2_000_001), np.arange(-124, 10, dtype=np.float64),
                         np.arange(-124, 9, dtype=np.float64) + 0.5, [0.0, -0.0, 1e-7, -1e-7]])
    x = torch.from_numpy(xs.astype(np.float32)).cuda()
    want = np.exp2(x.cpu().numpy().astype(np.float64))
    for method, bound in ((0, 2e-6), (1, 8e-5)):
        got = run(x, method).cpu().numpy().astype(np.float64)
        rel = np.abs(got - want) / want
        assert rel.max() <= bound, (method, rel.max(), xs[np.argmax(rel)])


def test_exp2_polynomial_clamps_instead_of_wrapping():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    x = torch.tensor([-125.0, -125.4, -126.0, -200.0, -1e30, float("-inf")], device="cuda")
    got = run(x, 1).cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got <= 2.0 ** -124.9)
    assert run(x[-1:], 0).item() == 0.0  # the MUFU path, used on masked tiles, gives exact 0
