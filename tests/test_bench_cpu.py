"""bench.py's reference arm and JSON contract, on the CPU (the reference arm
times the oracle on host cores and needs no GPU)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, timeout=600):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       timeout=timeout, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    j = _bench("--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1")
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in j, k
    assert j["impl"] == "reference" and j["steps"] == 2 and j["warmup"] == 1 and j["n_gpus"] == 1
    assert j["unit"] == "tokens/s" and j["higher_is_better"] is True and j["value"] > 0
    assert j["config"]["workload"] == "tiny" and j["config"]["batch"] == 1 and j["config"]["seq_len"] == 256
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"] and cb["sample"]
    e = j["e2e"]
    assert e["value"] == j["value"] and e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_arms_share_the_workload_config():
    sys.path.insert(0, ROOT)
    import bench
    for name, cfgd in bench.CONFIGS.items():
        c = bench.workload_config(name, cfgd, cfgd["layers"], 1)
        assert c["workload"] == name and c["batch"] == cfgd["B"] and c["seq_len"] == cfgd["T"]
        assert c["parallelism"] == "replicas x1"
