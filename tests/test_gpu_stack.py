"""GPU parity of a chained hybrid attention stack (through the C ABI) against the fp64 oracle.

The stack has the pages' shape (summary page, 核心方法 / 实验结果): dense (P = 1) layers at both
ends and Skiparse-2D layers in between with token-wise and group-wise layers alternating. Layers
are chained: layer l's output is layer l+1's q, and k and v are the same for every layer
(bench.py's stack rule). Every layer's output is compared with the oracle applied to that
layer's own GPU inputs (the previous layer's bf16 output), at the forward tolerance
(max|err| <= 1e-2, mean|err| <= 1e-3), so an error cannot hide behind the layers after it."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import bench
import oracle
import skiparse_synth as synth
from parity_helpers import check_close, gpu_rows, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fps():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fixed_pattern_sparse_b200 as m
    return m


def _run_stack(fps, w, layers, front, back):
    q, k, v = synth.qkv(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    sched = [(w.P if p is None else p, m) for p, m in bench.stack_schedule(layers, front, back)]
    outs = []
    bench.stack_pass(fps, qd, kd, vd, sched, (torch.empty_like(qd), torch.empty_like(qd)), keep=outs)
    assert fps.get_device_status() == 0
    return q, k, v, sched, outs


def test_stack_schedule_has_the_pages_shape():
    sched = bench.stack_schedule(6, 1, 1)
    assert sched == [(1, 0), (None, 0), (None, 1), (None, 0), (None, 1), (1, 0)]


def test_chained_stack_small_every_layer(fps):
    """Any-resolution latent (padded 12x16), 6 layers: 1 dense, 4 sparse alternating, 1 dense;
    every layer compared element by element."""
    w = synth.WORKLOADS["anyres"]
    q, k, v, sched, outs = _run_stack(fps, w, 6, 1, 1)
    x = q
    for layer, ((P, mode), out) in enumerate(zip(sched, outs)):
        want = oracle.attn_fwd(x, k, v, P, mode)
        check_close(out.double().cpu().numpy(), want, f"layer {layer} (P={P}, mode={mode})")
        x = out.cpu()  # the next layer's q is this layer's GPU output, bf16


def test_chained_stack_480p_sampled(fps):
    """480p latent, 8 layers: 2 dense, 4 sparse alternating, 2 dense; every layer on sampled
    rows (random tokens, frame corners, the last real row) of its own GPU inputs."""
    w = synth.WORKLOADS["480p"]
    q, k, v, sched, outs = _run_stack(fps, w, 8, 2, 2)
    x = q
    for layer, ((P, mode), out) in enumerate(zip(sched, outs)):
        rows = sample_rows(w, 96, seed=layer)
        want = oracle.attn_fwd_rows(x, k, v, rows, P, mode)
        check_close(gpu_rows(out, rows), want, f"layer {layer} (P={P}, mode={mode})")
        x = out.cpu()


def test_chained_stack_layers_differ(fps):
    """The chain is real: consecutive layers' outputs differ (each layer consumed the previous
    output), and the last output depends on the first layer's q."""
    w = synth.WORKLOADS["anyres"]
    _, _, _, _, outs = _run_stack(fps, w, 6, 1, 1)
    for a, b in zip(outs, outs[1:]):
        assert not torch.equal(a, b)
    q, k, v = (t.cuda() for t in synth.qkv(w))
    sched = [(w.P if p is None else p, m) for p, m in bench.stack_schedule(6, 1, 1)]
    bufs = (torch.empty_like(q), torch.empty_like(q))
    last_a = bench.stack_pass(fps, q, k, v, sched, bufs).clone()
    last_b = bench.stack_pass(fps, -q, k, v, sched, bufs).clone()
    assert not torch.equal(last_a, last_b)
    assert np.isfinite(last_a.double().cpu().numpy()).all()
