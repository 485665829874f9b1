"""bench.py's reference arm (the CPU fp64 oracle on the host cores): the JSON
line it prints carries the keys of the bench contract, and under a launcher
only rank 0 runs it.  No GPU is needed: the arm never touches the device."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=600)


def test_reference_line_has_the_contract_keys():
    r = _run(["--impl", "reference", "--steps", "2", "--warmup", "1", "--cpu-seconds", "0.6",
              "--config", "pr1_b1_h4_n1024_f32"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "outputs_per_step"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "elems/s" and d["higher_is_better"] is True
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 2, 1)
    assert d["vs_baseline"] is None and d["data"] == "synthetic" and d["dtype"] == "f64"
    assert d["config"]["workload"] == "pr1_b1_h4_n1024_f32"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
    # the line's time is the sample it ran, consistent with its own rate
    assert abs(d["outputs_per_step"] / (d["ms_per_step"] * 1e-3) - d["value"]) <= 1e-6 * d["value"]


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.3",
              "--config", "pr1_b1_h4_n1024_f32"], {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
