"""bench.py's JSON contract on CPU: the reference arm (the oracle timed on the
host) prints one line with every required key, only on rank 0, and carries
the key-cache width and base selector in its config."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [l for l in r.stdout.splitlines() if l.strip()]


def test_reference_arm_line_has_the_contract_keys():
    import bench
    lines = _run(["--impl", "reference", "--steps", "2", "--warmup", "1", "--config", "tiny"])
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is False
    assert d["value"] > 0 and d["ms_per_step"] == pytest.approx(d["value"] / 1e3)
    assert d["config"]["workload"] == "tiny_1h_4k"
    assert d["config"]["key_bits"] == 4 and d["config"]["selector"] == "quest"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["h2d_bytes_per_step"] == 0 and \
        e["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_on_other_ranks():
    assert _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--config", "tiny"],
                {"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_reference_arm_two_bit_keys():
    d = json.loads(_run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--config",
                         "tiny", "--key-bits", "2"])[0])
    assert d["config"]["key_bits"] == 2 and d["value"] > 0
