"""bench.py's reference arm (the CPU oracle timed on a bounded sample) runs
without a GPU and prints the one JSON line of the benchmark contract."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny",
                        "--steps", "2", "--warmup", "1"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "us/step" and d["higher_is_better"] is False
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and abs(d["ms_per_step"] * 1e3 - d["value"]) < 1e-6 * d["value"]
    assert d["config"]["workload"] == "tiny"
    # the same config keys as the GPU arm's line
    assert set(d["config"]) == {"workload", "batch", "h_q", "h_k", "h_v", "head_dim", "v_head_dim",
                                "l_kv", "N", "n", "parallelism", "l2", "timing"}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"]
    assert cb["cores"] == len(os.sched_getaffinity(0))
    assert cb["sample"].startswith("oracle steps 1..2 ")  # the timed steps follow the warm-up
    e = d["e2e"]
    assert e["value"] == d["value"] and e["h2d_bytes_per_step"] == 0 == e["d2h_bytes_per_step"]
