"""The fused Skiparse-2D forward equals the pages' explicit three-step pipeline, bit for bit.

The method step details of the OSP-Next summary page describe Skiparse-2D attention as three
steps: rearrange the tokens into P^2 subsequences, run dense (FlashAttention) attention on each
subsequence, rearrange the result back. The fused kernel folds the two rearranges into its
loads and stores. Here the explicit pipeline is built from this library's own standalone
kernels -- skiparse_rearrange on q, k and v, the dense (P = 1) attention kernel over the
B*P^2 subsequences of length n, skiparse_unrearrange of the output -- and compared with the
fused call.

On shapes that need no padding (H and W multiples of P^2) every subsequence holds n real
tokens in the rearranged order (t, r, s), which is the order in which the fused kernel
enumerates a class; both paths therefore run the same tiles through the same arithmetic and
must agree exactly. (With padding the explicit pipeline would also need the pad-key mask of the
any-resolution rule, which dense attention over the padded subsequence does not apply; those
shapes are covered against the oracle elsewhere.)
"""

from __future__ import annotations

import pytest
import torch

import skiparse_synth as synth

pytestmark = pytest.mark.gpu

SHAPES = [
    synth.custom(1, 4, 16, 24, 2, 64, 2, "p2_three_tiles"),     # n = 384: three key tiles
    synth.custom(2, 3, 8, 12, 3, 128, 2, "p2_batch2"),           # n = 72: one ragged tile, B = 2
    synth.custom(1, 3, 36, 36, 1, 128, 3, "p3_four_tiles"),      # n = 432, nine classes
    synth.custom(1, 2, 16, 16, 2, 32, 4, "p4_d32"),              # P = 4: sixteen classes of 32
    synth.WORKLOADS["768p"],                                     # the unpadded benchmark latent
]


def _pipeline(fps, q, k, v, P, mode):
    B, T, H, W, heads, d = q.shape
    ys = [fps.skiparse_rearrange(x, P, mode) for x in (q, k, v)]
    n = ys[0].shape[1]
    # dense attention over each of the B*P^2 subsequences: a (B*P^2, 1, 1, n) token grid, P = 1
    as_grid = [y.view(B * P * P, 1, 1, n, heads, d) for y in ys]
    o = fps.skiparse2d_attn_fwd(*as_grid, 1, 0)
    return fps.skiparse_unrearrange(o.view(B * P * P, n, heads, d), q.shape, P, mode)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_fused_equals_rearrange_dense_unrearrange(w, mode):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as fps
    assert fps.padded_extent(w.H, w.P) == w.H and fps.padded_extent(w.W, w.P) == w.W
    q, k, v = (t.cuda() for t in synth.qkv(w))
    fused = fps.skiparse2d_attn_fwd(q, k, v, w.P, mode)
    explicit = _pipeline(fps, q, k, v, w.P, mode)
    assert fps.get_device_status() == 0
    assert torch.equal(fused.view(torch.int16), explicit.view(torch.int16))


SHAPES_1D = [
    synth.custom(1, 3, 4, 16, 2, 64, 2, "1d_p2"),        # frame of 64 = 4 * 2^4 tokens, n = 48
    synth.custom(1, 2, 9, 9, 1, 128, 3, "1d_p3"),        # frame of 81 = 3^4 tokens, n = 18
    synth.custom(2, 2, 16, 16, 2, 32, 4, "1d_p4_b2"),    # frame of 256 = 4^4 tokens, n = 32
    synth.WORKLOADS["720p"],                             # 3600 = 225 * 2^4 per frame: no padding
]


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("w", SHAPES_1D, ids=lambda w: w.name)
def test_fused_1d_equals_rearrange_dense_unrearrange(w, mode):
    """The same equivalence for Skiparse-1D on frames whose H*W needs no padding (a multiple
    of P^4): skiparse1d_rearrange, dense attention per subsequence, skiparse1d_unrearrange."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as fps
    assert fps.padded_length_1d(w.H * w.W, w.P) == w.H * w.W
    q, k, v = (t.cuda() for t in synth.qkv(w))
    fused = fps.skiparse1d_attn_fwd(q, k, v, w.P, mode)
    B, T, H, W, heads, d = q.shape
    ys = [fps.skiparse1d_rearrange(x, w.P, mode) for x in (q, k, v)]
    n = ys[0].shape[1]
    grid = [y.view(B * w.P * w.P, 1, 1, n, heads, d) for y in ys]
    o = fps.skiparse2d_attn_fwd(*grid, 1, 0)
    explicit = fps.skiparse1d_unrearrange(o.view(B * w.P * w.P, n, heads, d), q.shape, w.P, mode)
    assert fps.get_device_status() == 0
    assert torch.equal(fused.view(torch.int16), explicit.view(torch.int16))
