"""The forward softmax's exponential loop alone, measured through the C ABI
(skiparse_debug_softmax_rate) on every SM at once.

The loop body is the attention softmax's (exponent by FFMA, ex2.approx, four running sums, bf16
pack) on distinct scores. The forward kernel's design reads its softmax as bound by the MUFU at
16 exponentials per clock per SM (2 x 128 x 128 per key step = 2048 clocks, beside 2067 clocks
of tensor-core work): with two warps per SM sub-partition, as the kernel runs them, the loop
reaches that rate, and more warps do not raise it."""

from __future__ import annotations

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

REPS = 256


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(wps: int):
    from fixed_pattern_sparse_b200 import _lib
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    warps = 4 * wps
    clocks = torch.full((sms * warps,), -2, dtype=torch.int64, device="cuda")
    rc = _lib.lib().skiparse_debug_softmax_rate(wps, REPS, clocks.data_ptr(), sms,
                                               torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    c = clocks.cpu().numpy()
    assert (c > 0).all(), "a warp did not report"
    med = float(np.median(c))
    per_warp_64 = med / REPS                              # clocks per 64 exponentials of one warp
    ex2_per_clk_sm = 64.0 * REPS * 32 * warps / med       # all warps of the SM run concurrently
    return per_warp_64, ex2_per_clk_sm


def test_the_loop_runs_at_sixteen_exponentials_per_clock(cuda):
    rates = {}
    for wps in (1, 2, 4):
        per_warp_64, rates[wps] = _run(wps)
        print(f"{wps} warp(s) / sub-partition: {per_warp_64:.0f} clocks per 64 exponentials, "
              f"{rates[wps]:.1f} ex2/clk/SM")
    # two warps per sub-partition (the kernel's softmax) reach the MUFU rate; four add nothing
    assert 14.0 <= rates[2] <= 17.0
    assert 14.0 <= rates[4] <= 17.0
    assert rates[4] < 1.1 * rates[2]
    # one warp alone stays close to it (its own dependency chains)
    assert rates[1] >= 12.0


def test_rejects_bad_arguments(cuda):
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    buf = torch.zeros(16, dtype=torch.int64, device="cuda")
    assert L.skiparse_debug_softmax_rate(3, 8, buf.data_ptr(), 1, None) == 1
    assert L.skiparse_debug_softmax_rate(1, 8, buf.data_ptr(), 2000, None) == 2
    assert L.skiparse_debug_softmax_rate(1, 8, buf.data_ptr() + 4, 1, None) == 3
