"""bench.py's reference arm (the fp64 oracle on the host cores) prints the line the driver
reads: the base keys, impl, a cpu_baseline describing the run and an e2e with no copies."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*extra):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *extra],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_reference_line_has_the_contract_keys():
    line = _run("--workload", "bf16_n256_tail10", "--steps", "2", "--warmup", "0")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["n_gpus"] == 1
    assert line["unit"] == "ms/layer" and line["higher_is_better"] is False and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert "workload" in line["config"] and "N=256" in line["config"]["workload"]


def test_reference_declines_the_workload_it_cannot_finish():
    line = _run("--workload", "bf16_n2048", "--steps", "1", "--warmup", "0")
    assert line["impl"] == "reference" and "unavailable" in line
