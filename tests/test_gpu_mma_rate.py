"""The tensor-core rate the attention kernels are designed around, measured through the C ABI
(skiparse_debug_mma_rate), on every SM at once.

A stream of tcgen05.mma instructions issued by one thread -- groups of 8 K-steps into one
accumulator, as the kernels' MMA warp issues them -- runs at the nominal dense bf16 rate of an SM
(8192 FLOP per clock) for M = 128 and N = 128, whether A comes from shared memory or from TMEM,
and for N = 256; a 128 x 128 x 16 step therefore takes 64 SM clocks. N = 64 runs well below it.
So the attention kernels' 128 x 128 tiles are not capped by the MMA shape: the time a kernel
spends above 64 clocks per step is idle tensor pipe."""

from __future__ import annotations

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

NOMINAL = 8192.0  # dense bf16 FLOP per clock per SM


def _rate(pattern: int, groups: int = 64):
    from fixed_pattern_sparse_b200 import _lib
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    clocks = torch.full((sms,), -2, dtype=torch.int64, device="cuda")
    rc = _lib.lib().skiparse_debug_mma_rate(pattern, groups, clocks.data_ptr(), sms,
                                           torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    c = clocks.cpu().numpy()
    assert (c > 0).all(), "a CTA did not finish its MMA stream"
    n = {0: 128, 1: 128, 2: 256, 3: 64, 4: 128, 5: 128, 6: 128}[pattern]
    flop = groups * 8 * 2.0 * 128 * n * 16
    return flop / np.median(c), np.median(c) / (groups * 8 * n / 128)


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("pattern", [0, 1, 2], ids=["ss_n128", "ts_n128", "ss_n256"])
def test_full_rate_shapes(cuda, pattern):
    per_clk, clk_per_128 = _rate(pattern)
    print(f"pattern {pattern}: {per_clk:.0f} FLOP/clk/SM ({per_clk / NOMINAL:.3f} of nominal), "
          f"{clk_per_128:.1f} clk per 128x128x16")
    assert per_clk >= 0.95 * NOMINAL


def test_n64_is_slower(cuda):
    per_clk, _ = _rate(3)
    print(f"N = 64: {per_clk:.0f} FLOP/clk/SM ({per_clk / NOMINAL:.3f} of nominal)")
    assert per_clk < 0.9 * NOMINAL


def test_issuer_starved_by_alu_bound_warps(cuda):
    """The issuing thread shares an SM sub-partition with other warps. Warps running the
    backward's dS arithmetic (FADD, FMUL, bf16 pack, no MUFU) leave it so few issue slots that
    the tensor pipe runs at a small fraction of its rate; warps running the forward softmax's
    exponential loop, which waits on the MUFU, cost it little. (Independent FFMA chains are
    printed for reference: whether they starve the issuer depends on how the loop compiles.)"""
    rates = {p: _rate(p)[0] / NOMINAL for p in (4, 5, 6)}
    print("beside FFMA chains / dS arithmetic / exponential loop:",
          " / ".join(f"{r:.3f}" for r in rates.values()), "of nominal")
    assert rates[5] < 0.5
    assert rates[6] >= 0.9


def test_rejects_bad_arguments(cuda):
    from fixed_pattern_sparse_b200 import _lib
    L = _lib.lib()
    buf = torch.zeros(4, dtype=torch.int64, device="cuda")
    assert L.skiparse_debug_mma_rate(7, 8, buf.data_ptr(), 4, None) == 1
    assert L.skiparse_debug_mma_rate(0, 0, buf.data_ptr(), 4, None) == 1
    assert L.skiparse_debug_mma_rate(0, 8, buf.data_ptr(), 5000, None) == 2
    assert L.skiparse_debug_mma_rate(0, 8, buf.data_ptr() + 4, 2, None) == 3
