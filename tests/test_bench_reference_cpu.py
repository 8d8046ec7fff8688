"""bench.py's reference arm (the fp64 oracle on the host cores) runs without a
GPU and prints one JSON line with impl "reference", for a plain, a grouped,
a windowed and an ALiBi workload (small budgets: a few seconds each)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", ["attn_B1_H1_N128_d64_noncausal", "attn_B2_H8_N1024_d64_causal",
                                      "mqa_B4_H16_Hkv1_N4096_d128_causal", "alibi_B4_H16_N4096_d128_causal"])
def test_reference_arm_prints_one_line(workload):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1", "--ref-seconds", "0.2", "--workload", workload],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["value"] > 0 and j["config"]["workload"] == workload
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["h2d_bytes_per_step"] == 0
