"""The exponential of the attention softmax against fp64 exp2 (through the C ABI).

The softmax evaluates p = 2^x with the MUFU ex2.approx instruction (flush-to-zero). Its
relative error must stay far inside half an ulp of bf16 (2^-9), the precision in which the
probabilities P enter the P*V product, over the whole range the softmax uses (x <= 8 after the
lazy-rescale threshold); -inf, which masked keys produce, must give exactly 0."""

from __future__ import annotations

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def run(x: torch.Tensor, method: int = 0) -> torch.Tensor:
    from fixed_pattern_sparse_b200 import _lib
    y = torch.empty_like(x)
    rc = _lib.lib().skiparse_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), method,
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    return y


def test_exp2_matches_fp64():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    xs = np.concatenate([np.linspace(-124.0, 9.0, 2_000_001), np.arange(-124, 10, dtype=np.float64),
                         np.arange(-124, 9, dtype=np.float64) + 0.5, [0.0, -0.0, 1e-7, -1e-7]])
    x = torch.from_numpy(xs.astype(np.float32)).cuda()
    want = np.exp2(x.cpu().numpy().astype(np.float64))
    got = run(x).cpu().numpy().astype(np.float64)
    rel = np.abs(got - want) / want
    assert rel.max() <= 2e-6, (rel.max(), xs[np.argmax(rel)])


def test_exp2_of_masked_scores_is_exactly_zero():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    x = torch.tensor([float("-inf"), -1e30, -200.0], device="cuda")
    assert run(x).cpu().tolist() == [0.0, 0.0, 0.0]


def test_exp2_rejects_other_methods():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fixed_pattern_sparse_b200 import _lib
    x = torch.zeros(4, device="cuda")
    assert _lib.lib().skiparse_debug_exp2(x.data_ptr(), x.data_ptr(), 4, 1, None) == 1
