"""Host-side contract of bench.py (CPU): the reference arm's JSON line, the
non-zero ranks of the reference arm, and workload selection."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def _run(args, env_extra=None, timeout=240):
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    env.pop("RANK", None)
    env.pop("LOCAL_RANK", None)
    if env_extra:
        env.update(env_extra)
    return subprocess.run([sys.executable, BENCH] + args, cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=timeout)


def test_reference_arm_json_line():
    p = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--batch", "1"])
    assert p.returncode == 0, p.stderr
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["unit"] == "samples/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "fno2d_f32_b16_w32_256sq_m16"
    assert d["config"]["batch_per_gpu"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    p = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--gpus", "2"],
             env_extra={"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


@pytest.mark.parametrize("args,msg", [
    (["--workload", "no_such_workload"], "unknown workload"),
    (["--workload", "block2d_f32_b4_w20_64sq_m12"], "single-block parity case"),
    (["--batch", "0"], "--batch must be >= 1"),
])
def test_workload_selection_errors(args, msg):
    p = _run(["--impl", "reference", "--steps", "1", "--warmup", "0"] + args, timeout=120)
    assert p.returncode != 0
    assert msg in p.stderr
