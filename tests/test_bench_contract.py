"""CPU checks of the benchmark's contract pieces: the reference arm's JSON line
(the oracle on the host cores) and the counting rules the GPU line reports."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny")


def test_launch_counts_per_step():
    # short heads: one prep kernel (relative-position tables ride along) + the fused kernel
    assert bench.launches_per_step(197, 2, "u8i8", True) == 2
    # a dense bias matrix adds its range and table kernels
    assert bench.launches_per_step(197, 2, "u8i8", True, dense_bias=True) == 4
    # long heads: statistics + their finalization + pack (+ bias range and table fill) + the fused kernel
    assert bench.launches_per_step(16384, 2, "float", True) == 6
    assert bench.launches_per_step(16384, 2, "float", False) == 4
    # fp32 V in float mode adds the hi/lo split
    assert bench.launches_per_step(128, 4, "float", False) == 3


@pytest.mark.parametrize("mode,N,n,bias,ops", [
    ("u8i8", 0, 197, True, 9.25),    # DeiT: 2 lookups + mul + add, then 2 lookups + mul + FFMA + convert + 1/4 pack
    ("float", 120, 1024, False, 4.5),
    ("float", 1920, 16384, True, 13.625),   # sampled level pass: 1/8 increment + 6 + 7.5
    ("float", 128, 1024, True, 14.5),       # 16 tiles: the level pass counts every key
])
def test_alu_ops_per_score(mode, N, n, bias, ops):
    assert bench.alu_ops_per_score(mode, N, n, bias) == ops
