"""Host-side pieces of bench.py that define the reported numbers, checked on CPU: the FLOP
count behind `value` (4*N*(N/P^2)*d*heads*B with N = T*Hp*Wp, the padded token count) and the
real-pair count reported beside it (sum over classes of 4*n_c^2*d*heads*B), for every
benchmark workload of the measurement plan."""

from __future__ import annotations

import pytest

import bench
import skiparse_synth as synth

# (workload, padded-formula FLOPs, real-pair FLOPs token-wise / group-wise), to 4 digits
TABLE = [
    ("tiny", 1.049e6, 1.049e6, 1.049e6),
    ("anyres", 8.493e7, 4.516e7, 4.792e7),
    ("480p", 1.876e12, 1.649e12, 1.656e12),
    ("720p", 3.329e13, 2.928e13, 2.928e13),
    ("768p", 3.671e13, 3.671e13, 3.671e13),
    ("768p_p3", 2.370e13, 1.631e13, 1.648e13),
    ("768p_p1", 1.468e14, 1.468e14, 1.468e14),
]


@pytest.mark.parametrize("name,padded,real_tok,real_grp", TABLE, ids=[t[0] for t in TABLE])
def test_flop_counts(name, padded, real_tok, real_grp):
    w = synth.WORKLOADS[name]
    assert bench.flops_padded(w) == pytest.approx(padded, rel=5e-4)
    assert bench.flops_real(w, 0) == pytest.approx(real_tok, rel=5e-4)
    assert bench.flops_real(w, 1) == pytest.approx(real_grp, rel=5e-4)


def test_720p_formula_by_hand():
    # N = 21 * 48 * 80 padded tokens, n = N / 4 per class, d = 128, 40 heads
    N = 21 * 48 * 80
    assert bench.flops_padded(synth.WORKLOADS["720p"]) == 4.0 * N * (N / 4) * 128 * 40


@pytest.mark.parametrize("name", ["tiny", "anyres", "480p", "720p", "768p", "768p_p3"])
def test_class_lens_match_the_library_geometry(name):
    """bench.py counts class sizes itself (so that its oracle arm never loads the library); the
    counts must still agree with the library's host geometry."""
    import fixed_pattern_sparse_b200 as fps
    w = synth.WORKLOADS[name]
    for mode in (0, 1):
        want = [fps.class_len(w.T, w.H, w.W, w.P, mode, ci, cj) for ci in range(w.P) for cj in range(w.P)]
        assert bench.class_lens(w, mode) == want


def test_reference_arm_loads_only_the_oracle():
    """`bench.py --impl reference` times the oracle; nothing of the product may be imported or
    loaded on that path."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, json, bench; bench.main(['--impl', 'reference', '--workload', 'tiny', '--steps', '1', "
            "'--warmup', '0']); mods = [m for m in sys.modules if m.startswith('fixed_pattern_sparse_b200')]; "
            "maps = open('/proc/self/maps').read(); print(json.dumps({'mods': mods, 'lib': 'libskiparse' in maps}))")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
    check = json.loads(lines[-1])
    assert check == {"mods": [], "lib": False}


def test_dram_traffic_entry_matches_the_current_forward_sources():
    """bench.py reports `roofline.traffic` only for the forward kernel sources it was captured on
    (keyed by their hash). An edit to those sources must come with a new one-pass capture of the
    720p launch (dram__bytes_read.sum + dram__bytes_write.sum) and a new key; this test makes a
    missing re-capture fail loudly instead of leaving the field silently null."""
    h = bench.kernel_hash()
    assert h in bench.KNOWN_TRAFFIC, (
        f"forward sources hash {h} has no captured DRAM traffic: re-capture the 720p launch and key it")
    # the captured bytes are the algorithmic ones: q, k, v read once and out written once (720p)
    w = synth.WORKLOADS["720p"]
    algorithmic = 4 * w.B * w.T * w.H * w.W * w.heads * w.d * 2
    assert abs(bench.KNOWN_TRAFFIC[h] - algorithmic) / algorithmic < 0.01
