"""The bench's reference arm (the CPU oracle) on the CPU: one JSON line with
the contract's keys for each workload; under torchrun only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.join(os.path.dirname(__file__), "..")
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference"] + args,
                       capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return [l for l in r.stdout.splitlines() if l.startswith("{")]


def _check(line):
    d = json.loads(line)
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]
    return d


def test_reference_arm_decode_line():
    lines = _run(["--steps", "1", "--warmup", "3"])
    assert len(lines) == 1
    d = _check(lines[0])
    assert d["config"]["workload"].startswith("decode_linear_4096")


def test_reference_arm_sweep_line():
    lines = _run(["--workload", "sweep", "--steps", "1", "--warmup", "3"])
    assert len(lines) == 1
    d = _check(lines[0])
    assert d["config"]["workload"] == "denoise_sweep_52"


def test_reference_arm_other_ranks_print_nothing():
    assert _run(["--steps", "1", "--warmup", "3"], {"RANK": "1", "WORLD_SIZE": "2"}) == []
