"""The benchmark's reference arm (the CPU oracle timed on the host) runs without
a GPU and prints the one JSON line of the bench contract."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "1", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, check=True).stdout
    lines = [ln for ln in out.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e",
                "cpu_baseline"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == "dsa_decode_steps_per_s"
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("decode_")
    # the same workload description as the GPU arm prints, and a per-step time
    # that is the work actually timed (one sequence per step)
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    assert d["config"] == bench.bench_config(workloads.WORKLOADS[1], 1)
    assert abs(d["value"] * workloads.WORKLOADS[1].B * d["ms_per_step"] * 1e-3 - 1) < 1e-6
