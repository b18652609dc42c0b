#!/usr/bin/env python3
"""Benchmark of the Skiparse-2D attention forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 720p] [--impl ours|reference]

One step = one fused skiparse2d_attn_fwd call (class rearrange + pad mask + per-class dense
attention + inverse rearrange, one kernel launch) over the whole synthetic workload; the
step alternates token-wise and group-wise mode, as the layers of the model do. Inputs are
seeded N(0,1) bf16 tensors larger than L2, resident in HBM when timing starts. `value` is
TFLOP/s by the padded formula 4*N*(N/P^2)*d*heads*B, N = T*Hp*Wp, summed over ranks.

Under torchrun (N > 1) every rank runs its own independent copy of the workload (the path
has no exchange step: (b, class, head) units are independent), timing is the max over
ranks, and `scaling` is "weak".

--impl reference times the CPU oracle (the only reference this method has: no reference
implementation is shipped) on a bounded sample of the same workload, on rank 0 only.
"""

from __future__ import annotations

import argparse
import datetime as _dt
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import skiparse_synth as synth  # noqa: E402

METRIC = "Skiparse-2D attn fwd TFLOP/s and % BF16 peak at 720p P=2; ms/layer vs P=1 dense"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the attention kernel (dram__bytes_read.sum + dram__bytes_write.sum,
# one-pass ncu capture of the 720p launch), keyed by the hash of the kernel sources it was
# captured on: a changed kernel reports null until it is captured again.
KNOWN_TRAFFIC = {
    # 2.33 GB read + 0.756 GB written (q, k, v read once, out written once)
    "e6281fdc8f37edc8": 3.086e9,
}

ATTN_SOURCES = ["fixed_pattern_sparse_b200/csrc/attn_fwd_sm100.cu",
                "fixed_pattern_sparse_b200/csrc/ptx_sm100.cuh",
                "fixed_pattern_sparse_b200/csrc/skiparse_internal.cuh",
                "fixed_pattern_sparse_b200/csrc/attn_common.cuh"]


def kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def padded(X, P):
    return -(-X // (P * P)) * (P * P)


def flops_padded(w) -> float:
    N = w.T * padded(w.H, w.P) * padded(w.W, w.P)
    return 4.0 * N * (N / (w.P * w.P)) * w.d * w.heads * w.B


def axis_real_counts(X: int, P: int, mode: int):
    """Real positions of each class along one frame axis of X real positions, counted one by one
    from the class rule (summary page, 核心方法: token-wise x mod P, group-wise (x div P) mod P).
    Padding only appends pad positions, so it never changes these counts. Written here, apart
    from both the library and the oracle, so that neither the timed oracle arm nor the FLOP
    counts depend on the code under test."""
    counts = [0] * P
    for x in range(X):
        counts[x % P if mode == 0 else (x // P) % P] += 1
    return counts


def class_lens(w, mode):
    """Real tokens of each class subsequence, class c = ci*P + cj, in class order."""
    rh, rw = axis_real_counts(w.H, w.P, mode), axis_real_counts(w.W, w.P, mode)
    return [w.T * rh[ci] * rw[cj] for ci in range(w.P) for cj in range(w.P)]


def flops_real(w, mode) -> float:
    return sum(4.0 * n * n * w.d * w.heads * w.B for n in class_lens(w, mode))


def describe(w) -> str:
    return (f"{w.name} latent B={w.B} T={w.T} H={w.H} W={w.W} heads={w.heads} d={w.d} P={w.P} "
            f"(padded {padded(w.H, w.P)}x{padded(w.W, w.P)})")


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        ident = None
        try:
            ident = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            pass
        if ident is None:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ident = vis.split(",")[device_index] if vis else str(device_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = []
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = _dt.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[4], parts[6:10]))
            except ValueError:
                continue
        os.unlink(self.file.name)
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[4]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "samples": len(inside), "power_w_max": max(float(r[3]) for r in inside if r[3].replace('.', '', 1).isdigit())
                if any(r[3].replace('.', '', 1).isdigit() for r in inside) else None,
                "reasons": reasons}


# ------------------------------------------------------------------------ distributed

def dist_setup(gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != gpus:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    return rank, world, local


def init_pg(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.distributed.init_process_group(backend, timeout=_dt.timedelta(seconds=300))


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def aggregate_tflops(flops_per_step: float, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job throughput: every rank ran `steps` steps of its own workload, timed as the
    maximum over ranks."""
    return flops_per_step * steps * world / (max_total_ms / 1e3) / 1e12


# ------------------------------------------------------------------------ CPU oracle

def subsequence_rows(w, mode, cls: int, head: int) -> np.ndarray:
    """Every query row (token*heads + head) of one (class, head) subsequence of batch element 0,
    in token order, with the class rule from the oracle."""
    import oracle
    toks = []
    for t in range(w.T):
        for h in range(w.H):
            ci, _ = oracle.axis_map(h, w.P, mode)
            for x in range(w.W):
                cj, _ = oracle.axis_map(x, w.P, mode)
                if ci * w.P + cj == cls:
                    toks.append((t * w.H + h) * w.W + x)
    return np.array(toks, dtype=np.int64) * w.heads + head


def oracle_sample_rows(w, mode, nrows: int, group: int = 0) -> np.ndarray:
    """`nrows` query rows (token*heads + head), evenly spaced over one (class, head) subsequence,
    for timing the oracle: class `group % P^2`, head `group // P^2`."""
    q2 = w.P * w.P
    rows = subsequence_rows(w, mode, group % q2, (group // q2) % w.heads)
    pick = np.linspace(0, len(rows) - 1, num=min(nrows, len(rows))).astype(np.int64)
    return rows[pick]


def time_oracle_subsequences(w, q, k, v, modes, nthreads: int):
    """Times the oracle on whole (class, head) subsequences: for each mode, every real query of
    the last class and the last head (in padded workloads the raggedest subsequence). Returns
    (TFLOP/s, seconds, description, {mode: (rows, fp64 output rows)}); the rows double as the
    benchmark's own parity check of the kernel."""
    import oracle
    q2 = w.P * w.P
    cls, head = q2 - 1, w.heads - 1
    flops, secs, per_mode = 0.0, 0.0, {}
    for m in modes:
        rows = subsequence_rows(w, m, cls, head)
        t = time.perf_counter()
        want = oracle.attn_fwd_rows(q, k, v, rows, w.P, m, nthreads)
        secs += time.perf_counter() - t
        n_c = class_lens(w, m)[cls]
        flops += 4.0 * n_c * w.d * len(rows)
        per_mode[m] = (rows, want)
    desc = ("; ".join(f"{MODE_NAME[m]}: all {len(per_mode[m][0])} query rows of the (class {cls}, head {head}) "
                      f"subsequence of the {w.name} workload over its {len(per_mode[m][0])} real keys"
                      for m in modes)
            + "; the oracle's per-subsequence gather included")
    return flops / secs / 1e12, secs, desc, per_mode


MODE_NAME = synth.MODE_NAMES


class nvtx_range:
    """An NVTX range around one leg of the benchmark (host-side annotation for a timeline tool;
    no effect on the device timings)."""

    def __init__(self, name: str):
        self.name = name

    def __enter__(self):
        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        torch.cuda.nvtx.range_pop()


# ------------------------------------------------------------- per-config table

TABLE_WORKLOADS = ("480p", "768p", "768p_p3")


def time_calls(fn, n, stream):
    """Mean ms per call of fn() over n calls after two untimed ones (CUDA events on `stream`)."""
    for _ in range(2):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def time_config_table(fps, dev, stream, peaks, args):
    """ms per call, TFLOP/s by the padded and the real-pair formulas and the fraction of the
    measured burst bf16 peak for every (workload, mode) of the measurement plan other than the
    headline one; the dense P = 1 call at 768p and the sparse speedups t(P=1) / t(P); the 768p
    backward at P = 2 and P = 3. Inputs are larger than L2 except at 480p (0.26 GB of q/k/v),
    whose calls are timed back to back."""
    peak = float(peaks["bf16_tflops"])
    rows = {}
    n = args.table_steps
    for name in TABLE_WORKLOADS:
        w = synth.WORKLOADS[name]
        q, k, v = (t.to(dev) for t in synth.qkv(w))
        out = torch.empty_like(q)
        fl = flops_padded(w)
        for m in (0, 1):
            ms = time_calls(lambda: fps.skiparse2d_attn_fwd(q, k, v, w.P, m, out=out), n, stream)
            rows[f"{name} {MODE_NAME[m]}"] = {
                "workload": describe(w), "ms_per_call": round(ms, 3),
                "tflops_padded": round(fl / (ms / 1e3) / 1e12, 1),
                "tflops_real_pairs": round(flops_real(w, m) / (ms / 1e3) / 1e12, 1),
                "frac_of_burst_peak": round(fl / (ms / 1e3) / 1e12 / peak, 4)}
        del q, k, v, out
    w1 = synth.WORKLOADS["768p_p1"]
    q, k, v = (t.to(dev) for t in synth.qkv(w1))
    out = torch.empty_like(q)
    ms1 = time_calls(lambda: fps.skiparse2d_attn_fwd(q, k, v, 1, 0, out=out), max(2, n // 2), stream)
    fl1 = flops_padded(w1)
    rows["768p_p1 dense"] = {"workload": describe(w1), "ms_per_call": round(ms1, 3),
                             "tflops_padded": round(fl1 / (ms1 / 1e3) / 1e12, 1),
                             "frac_of_burst_peak": round(fl1 / (ms1 / 1e3) / 1e12 / peak, 4)}
    speedup = {f"t(P=1)/t({name} {MODE_NAME[m]})": round(ms1 / rows[f"{name} {MODE_NAME[m]}"]["ms_per_call"], 3)
               for name in ("768p", "768p_p3") for m in (0, 1)}
    # backward at 768p: the inputs above (same latent), P = 2 and P = 3
    bwd = {}
    if not args.no_backward:
        g = synth.randn_bf16(w1.shape, 1000 * w1.family + 7).to(dev)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        delta = torch.empty(q.shape[:5], dtype=torch.float32, device=dev)
        for P in (2, 3):
            wP = synth.custom(w1.B, w1.T, w1.H, w1.W, w1.heads, w1.d, P)
            for m in (0, 1):
                o, lse = fps.skiparse2d_attn_fwd_lse(q, k, v, P, m)
                ms = time_calls(lambda: fps.skiparse2d_attn_bwd(q, k, v, o, g, lse, P, m, dq=dq, dk=dk, dv=dv,
                                                                delta=delta), max(2, n // 2), stream)
                bwd[f"768p P={P} {MODE_NAME[m]}"] = {"ms_per_call": round(ms, 3),
                                                     "tflops": round(2.5 * flops_padded(wP) / (ms / 1e3) / 1e12, 1)}
                del o, lse
        bwd["flop_formula"] = "2.5 x the forward's padded-formula FLOPs"
        del g, dq, dk, dv, delta
    del q, k, v, out
    if fps.get_device_status() != 0:
        raise SystemExit("device status error in the per-config timing")
    return {"forward": rows, "sparse_speedup_768p": speedup, "backward_768p": bwd or None,
            "steps_per_entry": n}


# --------------------------------------------------------------------------- our arm

def run_ours(args):
    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_pg(world, "nccl")
    import fixed_pattern_sparse_b200 as fps

    w = synth.WORKLOADS[args.workload]
    modes = [0, 1] if args.mode == "both" else [0 if args.mode == "token" else 1]
    if w.P == 1:
        modes = [0]
    q, k, v = synth.qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty_like(qd)
    fl = flops_padded(w)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, modes[i % len(modes)], out=out)

    for i in range(args.warmup):
        step(i)
    if fps.get_device_status() != 0:
        raise SystemExit("device status error during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    with nvtx_range("timed forward steps"):
        for i in range(args.steps):
            starts[i].record(stream)
            step(i)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier(world)
    clk = clocks.stop(t_wall0, t_wall1)
    if fps.get_device_status() != 0:
        raise SystemExit("device status error in the timed region")
    per_launch = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = starts[0].elapsed_time(ends[-1])
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_step = total_ms / args.steps
    value = aggregate_tflops(fl, args.steps, world, total_ms)
    by_mode = {MODE_NAME[m]: statistics.mean(per_launch[i] for i in range(args.steps) if i % len(modes) == j)
               for j, m in enumerate(modes) if j < args.steps}

    peaks, peak_src = load_peaks()
    mean_launch_s = statistics.mean(per_launch) / 1e3
    achieved = fl / mean_launch_s / 1e12
    peak = float(peaks["bf16_tflops"])
    roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": KNOWN_TRAFFIC.get(kernel_hash()),
            "kernel": "skiparse_attn_fwd_kernel<128>",
            "peak_source": f"{peak_src} burst cuBLAS bf16 (MEASURED_PEAKS.json bf16_tflops)",
            "frac_of_sustained": round(achieved / float(peaks.get("bf16_tflops_sustained", peak)), 4),
            "flop_per_launch": fl}

    # end to end through the public host API: pinned host in, pinned host out
    e2e = None
    if not args.no_e2e:
        # end to end through the C ABI with HOST buffers: skiparse2d_attn_fwd_host copies q, k, v
        # in from pinned host memory, runs the kernel and copies out back, overlapped per group
        # of heads; all of it inside the timed region
        qh, kh, vh = (t.pin_memory() for t in (q, k, v))
        oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        hg = min(args.e2e_heads_per_group, w.heads)
        ws = torch.empty(fps.host_workspace_bytes(q.shape, hg), dtype=torch.uint8, device=dev)
        for i in range(2):
            fps.attn_fwd_host(qh, kh, vh, w.P, modes[i % len(modes)], oh, heads_per_group=hg, workspace=ws,
                              stream=stream)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.nvtx.range_push("end-to-end host-buffer steps")
        e0.record(stream)
        for i in range(args.e2e_steps):
            fps.attn_fwd_host(qh, kh, vh, w.P, modes[i % len(modes)], oh, heads_per_group=hg, workspace=ws,
                              stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        torch.cuda.nvtx.range_pop()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        if fps.get_device_status() != 0:
            raise SystemExit("device status error in the end-to-end timing")
        # the transfer floor of the same bytes: plain pinned copies host -> device of q, k, v and
        # device -> host of the output, each direction timed alone (the two directions of the
        # link run concurrently in the pipelined call, so its floor is the slower of the two)
        scratch = torch.empty_like(qd)
        c0, c1, c2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        c0.record(stream)
        for t_h in (qh, kh, vh):
            scratch.copy_(t_h, non_blocking=True)
        c1.record(stream)
        oh.copy_(out, non_blocking=True)
        c2.record(stream)
        torch.cuda.synchronize(dev)
        h2d_ms, d2h_ms = c0.elapsed_time(c1), c1.elapsed_time(c2)
        del scratch
        e2e = {"value": round(aggregate_tflops(fl, args.e2e_steps, world, e_ms), 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": q.numel() * 2,
               "ms_per_step": round(e_ms / args.e2e_steps, 3), "steps": args.e2e_steps,
               "path": "skiparse2d_attn_fwd_host (C ABI, pinned host buffers, copies overlapped per head group)",
               "heads_per_group": hg,
               "copy_only_ms": {"h2d": round(h2d_ms, 3), "d2h": round(d2h_ms, 3),
                                "h2d_gbs": round(3 * q.numel() * 2 / (h2d_ms / 1e3) / 1e9, 1),
                                "d2h_gbs": round(q.numel() * 2 / (d2h_ms / 1e3) / 1e9, 1)},
               "frac_of_transfer_floor": round(max(h2d_ms, d2h_ms) / (e_ms / args.e2e_steps), 4)}
        del ws, qh, kh, vh, oh

    # P = 1 dense attention at the same shape on the same kernel: ms/layer and sparse speedup
    dense = None
    if not args.no_dense and w.P > 1:
        wd = synth.custom(w.B, w.T, w.H, w.W, w.heads, w.d, 1, name=w.name + "_p1")
        for _ in range(2):
            fps.skiparse2d_attn_fwd(qd, kd, vd, 1, 0, out=out)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with nvtx_range("dense P=1 steps"):
            d0.record(stream)
            for _ in range(args.dense_steps):
                fps.skiparse2d_attn_fwd(qd, kd, vd, 1, 0, out=out)
            d1.record(stream)
            torch.cuda.synchronize(dev)
        dms = d0.elapsed_time(d1) / args.dense_steps
        dense = {"ms_per_layer_p1": round(dms, 3), "tflops_p1": round(flops_padded(wd) / (dms / 1e3) / 1e12, 1),
                 "sparse_speedup": round(dms / statistics.mean(per_launch), 3)}
        if fps.get_device_status() != 0:
            raise SystemExit("device status error in the dense comparison")

    # The pages' explicit pipeline (方法步骤详情: rearrange into P^2 subsequences, dense attention on
    # each, rearrange back), built from this library's standalone kernels, against the fused
    # kernel on the unpadded 768p latent (P = 2), where the two give identical results: what
    # folding the rearranges into the attention kernel buys.
    mat = None
    if not args.no_materialized and rank == 0:
        wm = synth.WORKLOADS["768p"]
        qm, km, vm = (t.to(dev) for t in synth.qkv(wm))
        om = torch.empty_like(qm)
        ys = [torch.empty(fps.rearranged_shape(qm.shape, wm.P), dtype=torch.bfloat16, device=dev)
              for _ in range(4)]
        n = ys[0].shape[1]
        grid = (wm.B * wm.P * wm.P, 1, 1, n, wm.heads, wm.d)

        def explicit(m):
            for x, y in zip((qm, km, vm), ys):
                fps.skiparse_rearrange(x, wm.P, m, out=y)
            fps.skiparse2d_attn_fwd(*(y.view(grid) for y in ys[:3]), 1, 0, out=ys[3].view(grid))
            fps.skiparse_unrearrange(ys[3], qm.shape, wm.P, m, out=om)

        def fused(m):
            fps.skiparse2d_attn_fwd(qm, km, vm, wm.P, m, out=om)

        res = {}
        torch.cuda.nvtx.range_push("explicit pipeline vs fused, 768p")
        for name, fn in (("fused", fused), ("explicit", explicit)):
            for i in range(2):
                fn(modes[i % len(modes)])
            m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            m0.record(stream)
            for i in range(args.materialized_steps):
                fn(modes[i % len(modes)])
            m1.record(stream)
            torch.cuda.synchronize(dev)
            res[name] = m0.elapsed_time(m1) / args.materialized_steps
        torch.cuda.nvtx.range_pop()
        if fps.get_device_status() != 0:
            raise SystemExit("device status error in the explicit-pipeline timing")
        mat = {"workload": describe(wm) + ", no padding", "ms_fused": round(res["fused"], 3),
               "ms_explicit": round(res["explicit"], 3),
               "explicit_steps": "3 x skiparse_rearrange + dense (P=1) attention over B*P^2 "
                                 "subsequences + skiparse_unrearrange",
               "fusion_speedup": round(res["explicit"] / res["fused"], 3),
               "hbm_bytes_saved_per_call": 2 * (4 * qm.numel() + 4 * ys[0].numel())}
        del qm, km, vm, om, ys

    # Skiparse-1D (the flattened-sequence variant) at the same shape on the same kernels: the
    # 1D-vs-2D comparison, by the same padded FLOP formula with N = T * Lp
    one_d = None
    if not args.no_1d and w.P > 1:
        fl1 = fps.attn_flops(q.shape, w.P, dims=1)
        for i in range(3):
            fps.skiparse1d_attn_fwd(qd, kd, vd, w.P, modes[i % len(modes)], out=out)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.one_d_steps):
            fps.skiparse1d_attn_fwd(qd, kd, vd, w.P, modes[i % len(modes)], out=out)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms1 = e0.elapsed_time(e1) / args.one_d_steps
        yshape1 = fps.rearranged_shape(q.shape, w.P, dims=1)
        y1 = torch.empty(yshape1, dtype=torch.bfloat16, device=dev)
        for i in range(3):
            fps.skiparse1d_rearrange(qd, w.P, modes[i % len(modes)], out=y1)
        e0.record(stream)
        for i in range(args.rearrange_steps):
            fps.skiparse1d_rearrange(qd, w.P, modes[i % len(modes)], out=y1)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        rms1 = e0.elapsed_time(e1) / args.rearrange_steps
        rbytes1 = (qd.numel() + y1.numel()) * 2
        del y1
        if fps.get_device_status() != 0:
            raise SystemExit("device status error in the Skiparse-1D timing")
        one_d = {"ms_per_layer": round(ms1, 3), "tflops": round(fl1 / (ms1 / 1e3) / 1e12, 1),
                 "frac_of_bf16_peak": round(fl1 / (ms1 / 1e3) / 1e12 / float(peaks["bf16_tflops"]), 4),
                 "padded_tokens_per_frame": fps.padded_length_1d(w.H * w.W, w.P),
                 "vs_2d_ms": round(ms1 / statistics.mean(per_launch), 3),
                 "rearrange_gbs": round(rbytes1 / (rms1 / 1e3) / 1e9, 1),
                 "modes": "alternating " + " / ".join(MODE_NAME[m] for m in modes)}

    # backward pass (fine-tuning): 3 launches per call, FLOPs counted as 2.5x the forward's
    # (dV, dP, dQ, dK and the recomputed S: the standard accounting of attention backward)
    bwd = None
    if not args.no_backward:
        gd = synth.randn_bf16(w.shape, 1000 * w.family + 7).to(dev)
        outs, lses = [], []
        for m in modes:
            o_m, l_m = fps.skiparse2d_attn_fwd_lse(qd, kd, vd, w.P, m)
            outs.append(o_m)
            lses.append(l_m)
        dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
        delta = torch.empty(qd.shape[:5], dtype=torch.float32, device=dev)

        def bstep(i):
            j = i % len(modes)
            fps.skiparse2d_attn_bwd(qd, kd, vd, outs[j], gd, lses[j], w.P, modes[j], dq=dq, dk=dk, dv=dv, delta=delta)

        for i in range(3):
            bstep(i)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with nvtx_range("backward steps"):
            b0.record(stream)
            for i in range(args.backward_steps):
                bstep(i)
            b1.record(stream)
            torch.cuda.synchronize(dev)
        bms = b0.elapsed_time(b1) / args.backward_steps
        if fps.get_device_status() != 0:
            raise SystemExit("device status error in the backward timing")
        bwd = {"ms_per_call": round(bms, 3), "tflops": round(2.5 * fl / (bms / 1e3) / 1e12, 1),
               "flop_formula": "2.5 x the forward's padded-formula FLOPs",
               "launches_per_call": 3, "forward_plus_backward_ms": round(bms + statistics.mean(per_launch), 3)}
        del gd, outs, lses, dq, dk, dv, delta

    # standalone rearrange / unrearrange bandwidth (HBM-bound permutation of token rows)
    rearr = None
    if not args.no_rearrange:
        yshape = fps.rearranged_shape(q.shape, w.P)
        y = torch.empty(yshape, dtype=torch.bfloat16, device=dev)
        back = torch.empty_like(qd)
        bytes_fwd = (qd.numel() + y.numel()) * 2  # read real rows, write all slots
        bytes_inv = 2 * qd.numel() * 2            # read real slots, write all rows
        res = {}
        y2 = torch.empty_like(y)
        for name, fn, nbytes in (("rearrange", lambda m: fps.skiparse_rearrange(qd, w.P, m, out=y), bytes_fwd),
                                 ("unrearrange", lambda m: fps.skiparse_unrearrange(y, q.shape, w.P, m, out=back), bytes_inv),
                                 ("switch_mode", lambda m: fps.skiparse_switch_mode(y, q.shape, w.P, m, out=y2), bytes_fwd)):
            for i in range(3):
                fn(modes[i % len(modes)])
            r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            r0.record(stream)
            for i in range(args.rearrange_steps):
                fn(modes[i % len(modes)])
            r1.record(stream)
            torch.cuda.synchronize(dev)
            ms = r0.elapsed_time(r1) / args.rearrange_steps
            gbs = nbytes / (ms / 1e3) / 1e9
            res[name] = {"ms": round(ms, 4), "bytes": nbytes, "gbs": round(gbs, 1),
                         "frac_of_hbm": round(gbs / float(peaks["hbm_gbs"]), 4)}
        res["hbm_peak_gbs"] = float(peaks["hbm_gbs"])
        res["note"] = "algorithmic bytes (read + write) per call / CUDA-event time; inputs > L2"
        rearr = res
        del y, y2, back
        if fps.get_device_status() != 0:
            raise SystemExit("device status error in the rearrange timing")

    # the measurement plan's other workloads (480p, 768p at P = 2 and P = 3, 768p P = 1 dense), each
    # mode timed on its own, the sparse speedups against dense at 768p, and the 768p backward
    configs = None
    if not args.no_configs:
        configs = time_config_table(fps, dev, stream, peaks, args)

    stack = None
    if not args.no_stack:
        stack = time_stack(fps, w, qd, kd, vd, args.layers, args.dense_front, args.dense_back, 1, world, dev, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        nth = oracle.default_threads()
        val, dt, desc, per_mode = time_oracle_subsequences(w, q, k, v, modes, nth)
        # the same rows from the kernel (outside every timed region): the bench's own parity
        # check against the oracle, whole subsequences in every mode, at the parity tests' tolerance
        parity = {}
        for m in modes:
            orows, want = per_mode[m]
            fps.skiparse2d_attn_fwd(qd, kd, vd, w.P, m, out=out)
            got = out.reshape(-1, w.d).index_select(0, torch.from_numpy(orows).to(dev)).double().cpu().numpy()
            err = np.abs(got - want)
            parity[MODE_NAME[m]] = {
                "rows": int(len(orows)), "subsequence": f"class {w.P * w.P - 1}, head {w.heads - 1} (whole)",
                "max_abs_err": float(err.max()), "mean_abs_err": float(err.mean()),
                "ok": bool(np.isfinite(got).all() and err.max() <= 1e-2 and err.mean() <= 1e-3)}
        parity["tolerance"] = "max <= 1e-2, mean <= 1e-3 against the fp64 oracle"
        cpu = {"value": round(val, 6), "unit": "TFLOP/s", "cores": nth, "kind": "oracle",
               "sample": desc, "seconds": round(dt, 2),
               # labelled extrapolation: the whole workload's real-pair FLOPs at the sample's rate
               "extrapolated_seconds_per_call": round(flops_real(w, modes[0]) / (val * 1e12), 1),
               "parity": parity}

    if rank == 0:
        real = {MODE_NAME[m]: round(flops_real(w, m) / (by_mode[MODE_NAME[m]] / 1e3) / 1e12, 1)
                for m in modes if MODE_NAME[m] in by_mode}
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) q/k/v rounded to bf16 (no dataset)",
            "config": {"workload": describe(w),
                       "modes": "alternating " + " / ".join(MODE_NAME[m] for m in modes) + " per step",
                       "flop_formula": "4*N*(N/P^2)*d*heads*B with N = T*Hp*Wp (padded)",
                       "l2": f"inputs larger than L2 ({3 * q.numel() * 2 / 1e9:.2f} GB of q/k/v per step), no flush",
                       "parallelism": f"{world} independent replica(s), one per GPU, no collective"},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": clk,
            "ms_per_layer": {k_: round(v_, 3) for k_, v_ in by_mode.items()},
            "ms_per_launch": {"median": round(statistics.median(per_launch), 3),
                              "min": round(min(per_launch), 3)},
            "tflops_real_pairs": real,
            "dense_p1": dense,
            "explicit_pipeline": mat,
            "skiparse1d": one_d,
            "rearrange_kernels": rearr,
            "backward": bwd,
            "configs": configs,
            "stack": stack,
            "kernel_hash": kernel_hash(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------- hybrid stack harness

STACK_RULE = "layer l's output is layer l+1's q; k and v are the same for every layer"


def stack_schedule(layers: int, dense_front: int, dense_back: int):
    """(P, mode) per layer of a hybrid stack: dense (P=1) blocks at both ends, Skiparse-2D in
    the middle with token-wise and group-wise layers alternating (summary page 核心方法 /
    实验结果: 4 full-attention blocks at the front and 4 at the back, the rest sparse).
    P is None for the sparse layers (the workload's P)."""
    sched, k = [], 0
    for i in range(layers):
        if i < dense_front or i >= layers - dense_back:
            sched.append((1, 0))
        else:
            sched.append((None, k % 2))
            k += 1
    return sched


def stack_pass(fps, x0, k, v, sched, bufs, keep=None):
    """One pass of a chained attention stack: layer l attends with q = x_l (x_0 = x0) over the
    fixed k and v, and its output is x_{l+1}. Outputs alternate between the two buffers of
    `bufs`, so no layer's output aliases its own q. `keep` collects every layer's output (a
    copy) when given. Returns the last layer's output."""
    x = x0
    for layer, (P, mode) in enumerate(sched):
        out = bufs[layer % 2]
        fps.skiparse2d_attn_fwd(x, k, v, P, mode, out=out)
        if keep is not None:
            keep.append(out.clone())
        x = out
    return x


def time_stack(fps, w, q, k, v, layers, dense_front, dense_back, steps, world, dev, stream):
    """Times the chained hybrid stack and the all-dense stack of the same depth (one pass = all
    layers in order, each layer's launch reading the previous layer's output from HBM)."""
    hybrid = [(w.P if p is None else p, m) for p, m in stack_schedule(layers, dense_front, dense_back)]
    dense = [(1, 0)] * layers
    bufs = (torch.empty_like(q), torch.empty_like(q))

    def timed(sched, n):
        stack_pass(fps, q, k, v, sched, bufs)
        torch.cuda.synchronize(dev)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            stack_pass(fps, q, k, v, sched, bufs)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return max_over_ranks(e0.elapsed_time(e1) / n, world, dev)

    with nvtx_range("chained hybrid stack"):
        h_ms = timed(hybrid, steps)
    with nvtx_range("chained dense stack"):
        d_ms = timed(dense, steps)
    if fps.get_device_status() != 0:
        raise SystemExit("device status error in the stack timing")
    fl_h = sum(flops_padded(synth.custom(w.B, w.T, w.H, w.W, w.heads, w.d, P)) for P, _ in hybrid)
    return {"layers": layers, "dense_front": dense_front, "dense_back": dense_back,
            "sparse_layers": layers - dense_front - dense_back,
            "sparse_modes": "alternating token-wise / group-wise", "chaining": STACK_RULE,
            "ms_per_pass": round(h_ms, 2), "dense_stack_ms": round(d_ms, 2),
            "attention_speedup": round(d_ms / h_ms, 3), "hybrid_tflops": round(fl_h / (h_ms / 1e3) / 1e12, 1),
            "gpu_launches_per_pass": layers, "passes_timed": steps}


def run_stack(args):
    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_pg(world, "nccl")
    import fixed_pattern_sparse_b200 as fps
    w = synth.WORKLOADS[args.workload]
    q, k, v = (t.to(dev) for t in synth.qkv(w))
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        stack_pass(fps, q, k, v, [(w.P if p is None else p, m) for p, m in
                                   stack_schedule(args.layers, args.dense_front, args.dense_back)],
                   (torch.empty_like(q), torch.empty_like(q)))
    st = time_stack(fps, w, q, k, v, args.layers, args.dense_front, args.dense_back, args.steps, world, dev,
                    stream)
    if rank == 0:
        print(json.dumps({
            "metric": "chained hybrid attention stack: ms per pass vs an all-dense stack (attention layers only)",
            "value": st["ms_per_pass"], "unit": "ms", "higher_is_better": False, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "scaling": "weak", "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) q/k/v rounded to bf16",
            "config": {"workload": describe(w), **{k_: st[k_] for k_ in ("layers", "dense_front", "dense_back",
                                                                        "sparse_layers", "sparse_modes", "chaining")}},
            "dense_stack_ms": st["dense_stack_ms"], "attention_speedup": st["attention_speedup"],
            "hybrid_tflops": st["hybrid_tflops"], "gpu_launches_per_pass": args.layers,
        }), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# --------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = synth.WORKLOADS[args.workload]
    modes = [0, 1] if args.mode == "both" else [0 if args.mode == "token" else 1]
    if w.P == 1:
        modes = [0]
    q, k, v = synth.qkv(w)
    nth = oracle.default_threads()
    n_c = {m: max(class_lens(w, m)) for m in modes}
    # size one step's sample so that all warm-up + timed steps take a few minutes
    budget_per_step = min(6.0, 150.0 / max(1, args.steps + args.warmup))
    rows = {}
    for m in modes:
        probe = oracle_sample_rows(w, m, max(nth, 8))
        t = time.perf_counter()
        oracle.attn_fwd_rows(q, k, v, probe, w.P, m, nth)
        dt = time.perf_counter() - t
        rows[m] = oracle_sample_rows(w, m, int(max(nth, len(probe) * budget_per_step / max(dt, 1e-3))))
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        m = modes[i % len(modes)]
        t = time.perf_counter()
        oracle.attn_fwd_rows(q, k, v, rows[m], w.P, m, nth)
        dt = time.perf_counter() - t
        if i >= args.warmup:
            times.append(dt)
            flops.append(4.0 * n_c[m] * w.d * len(rows[m]))
    value = sum(flops) / sum(times) / 1e12
    sample = (f"per step: {len(rows[modes[0]])} query rows of one (class, head) subsequence of the "
              f"{w.name} workload, each over its class's ~{n_c[modes[0]]} real keys (fp64 oracle)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * sum(times) / len(times), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: seeded N(0,1) q/k/v rounded to bf16 (no dataset)",
            "config": {"workload": describe(w),
                       "modes": "alternating " + " / ".join(MODE_NAME[m] for m in modes) + " per step",
                       "flop_formula": "4 * (real keys of the class) * d per sampled query row"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": nth, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="720p", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--mode", choices=["both", "token", "group"], default="both")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-heads-per-group", type=int, default=2)
    ap.add_argument("--dense-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rearrange", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-1d", action="store_true", help="skip the Skiparse-1D comparison")
    ap.add_argument("--no-materialized", action="store_true",
                    help="skip the explicit rearrange / dense / unrearrange pipeline comparison")
    ap.add_argument("--materialized-steps", type=int, default=4)
    ap.add_argument("--one-d-steps", type=int, default=4)
    ap.add_argument("--backward-steps", type=int, default=4)
    ap.add_argument("--rearrange-steps", type=int, default=10)
    ap.add_argument("--stack", action="store_true",
                    help="time only the chained hybrid stack of dense and alternating Skiparse-2D layers")
    ap.add_argument("--no-stack", action="store_true", help="skip the chained hybrid stack in the default run")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-config table (480p, 768p P=2/3, 768p dense, 768p backward)")
    ap.add_argument("--table-steps", type=int, default=4)
    ap.add_argument("--layers", type=int, default=40)
    ap.add_argument("--dense-front", type=int, default=4)
    ap.add_argument("--dense-back", type=int, default=4)
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.stack:
        run_stack(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
