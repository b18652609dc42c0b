"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2): rank setup,
max-over-ranks timing, whole-job aggregation, and the reference arm's rank-0-only rule. The
data path has no collective (every rank runs an independent replica), so this is all the
multi-rank logic there is."""

from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_setup(world)
    bench.init_pg(w, "gloo")
    try:
        got = bench.max_over_ranks(100.0 + 7.0 * r, w, torch.device("cpu"))
        bench.barrier(w)
        out.put((r, local, got))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_with_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in results] == [0, 1]
    assert all(got == 107.0 for _, _, got in results)


def test_aggregation_is_total_work_over_slowest_rank():
    import bench
    # 2 ranks x 10 steps x 3.3e13 FLOP in 300 ms (the slower rank) -> 2200 TFLOP/s
    assert bench.aggregate_tflops(3.3e13, 10, 2, 300.0) == pytest.approx(2200.0)
    assert bench.aggregate_tflops(3.3e13, 10, 1, 300.0) == pytest.approx(1100.0)


def test_world_mismatch_is_rejected(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.dist_setup(2)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"])
    assert capsys.readouterr().out == ""


def test_hybrid_stack_schedule():
    """4 dense blocks at each end, alternating sparse modes in between (the pages' hybrid)."""
    import bench
    sched = bench.stack_schedule(40, 4, 4)
    assert len(sched) == 40
    assert all(p == 1 for p, _ in sched[:4] + sched[-4:])
    middle = sched[4:-4]
    assert all(p is None for p, _ in middle) and len(middle) == 32
    assert [m for _, m in middle] == [0, 1] * 16
