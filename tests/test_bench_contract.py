"""The benchmark's JSON line keeps its contract: one line with the keys the
harness reads, typed as it expects.  The reference arm (the fp64 oracle on the
host cores) runs without a GPU, so its line is checked here end to end on the
tiny workload; the GPU arm's line is produced by the same helpers."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

BASE_KEYS = {
    "metric": str, "value": (int, float), "unit": str, "n_gpus": int, "steps": int, "warmup": int,
    "ms_per_step": (int, float), "higher_is_better": bool, "scaling": str, "dtype": str, "data": str,
    "config": dict,
}


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key, typ in BASE_KEYS.items():
        assert isinstance(line[key], typ), key
    assert line["impl"] == "reference"
    assert "vs_baseline" in line and line["vs_baseline"] is None
    assert line["steps"] == 1 and line["warmup"] >= 3 and line["n_gpus"] == 1
    assert line["scaling"] == "weak" and line["higher_is_better"] is True
    assert line["config"]["workload"].startswith("tiny")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    one = cb["single_thread"]  # reported for the tiny and 7B workloads
    assert one["cores"] == 1 and one["value"] > 0 and one["unit"] == "GB/s"
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert line["value"] > 0 and line["ms_per_step"] > 0
