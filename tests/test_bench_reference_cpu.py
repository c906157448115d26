"""bench.py's reference arm (the fp64 oracle on the host cores) on CPU: one JSON line with the
keys of the benchmark contract, and silence on ranks other than 0."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = run_bench({"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr
    lines = [s for s in r.stdout.splitlines() if s.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["dtype"] == "f64" and line["data"] == "synthetic"
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["steps"] == 1 and line["warmup"] == 1 and line["value"] > 0
    # value = tokens per step / seconds per step, each step a bounded sample of the long_bf16
    # step: the first `tok` tokens of the sequence plus one decode token
    import re
    cb = line["cpu_baseline"]
    tok = int(re.search(r"first (\d+) tokens", cb["sample"]).group(1))
    assert 64 <= tok <= 2048
    assert abs(line["value"] - (tok + 1) / (line["ms_per_step"] * 1e-3)) <= 1e-6 * line["value"]
    assert line["config"]["workload"].startswith("long_bf16")
    assert line["config"]["seq_len"] == 32768
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
