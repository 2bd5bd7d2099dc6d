"""The benchmark's contract on the host (no GPU): the reference arm (the oracle
timed on the host cores) prints one JSON line with the keys the driver reads, and
the algorithmic byte counts behind every roofline fraction are the per-unit
figures the design notes state.
"""
from __future__ import annotations

import json
import subprocess
import sys
from pathlib import Path

import bench

ROOT = Path(__file__).resolve().parents[1]


def test_reference_arm_prints_one_json_line_with_the_contract_keys():
    r = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-tokens", "64"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["metric"] == bench.METRIC
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["unit"] == "tok/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tok/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_algorithmic_bytes_per_unit():
    """Prefill: q, k, v, o bf16 + g fp32 + beta fp32 = 1540 B per token-head, plus 64 KB
    per (snapshot or state, head). Decode: 64 KB read + 64 KB written + 1540 B per
    state-step. Verify: the state read once per sequence-head, then per token-head a
    state written plus the vectors. Commit: a state read and a state written."""
    H, D = bench.H, bench.D
    state = H * D * D * 4
    assert bench.prefill_bytes(1, 0, 0, False) == 1540 * H
    assert bench.prefill_bytes(8192, 1, 32, False) == 8192 * 1540 * H + 33 * state == 945815552
    assert bench.prefill_bytes(10, 2, 3, True) == 10 * 1540 * H + (3 + 4) * state
    assert bench.decode_bytes(1) == H * (2 * D * D * 4 + 1540)
    assert bench.verify_bytes(2, 5) == 2 * state + 5 * H * (D * D * 4 + 1540)
    assert bench.commit_bytes(3) == 3 * 2 * state


def test_end_to_end_windows_cover_the_call_and_its_snapshot_rows():
    """The end-to-end leg runs the 8192-token prefill as windows with start positions: the
    windows tile the call, and each window's snapshot rows (the host plan with its start
    position) are the slice of the whole call's rows that the bench hands it."""
    import numpy as np
    from hybrid_linear_attention_04_b200 import kda as K
    T, W, snap = bench.PREFILL_T, bench.E2E_WIN, bench.SNAP
    assert W % snap == 0 and W % 64 == 0
    offs, pos = K.kda_snapshot_plan(np.array([0, T], np.int32), None, snap)
    wins = [(a, min(T, a + W)) for a in range(0, T, W)]
    assert wins[0][0] == 0 and wins[-1][1] == T
    assert all(b == c for (_, b), (c, _) in zip(wins, wins[1:]))
    rows = []
    for a, b in wins:
        o, p = K.kda_snapshot_plan(np.array([0, b - a], np.int32), np.array([a], np.int64), snap)
        assert list(p) == list(pos[a // snap:b // snap])
        rows += list(range(a // snap, a // snap + int(o[-1])))
    assert rows == list(range(int(offs[-1])))
