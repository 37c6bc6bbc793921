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


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", BENCH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_roofline_alu_for_cuda_core_backward():
    from fourier_neural_spectral_fno_b200 import synth
    bench = _bench_module()
    wl = synth.WORKLOADS["fno2d_bf16_train_b32_w64_256sq_m24"]
    rec = bench.roofline_record("epi_block_bwd", 2.5, wl, 148)
    # per point: 4 m_L C (inverse of dxhat) + 4 C^2 (dx and dW) FLOPs over B N points
    flops = 32 * 65536 * (4 * 24 * 64 + 4 * 64 * 64)
    assert rec["bound"] == "alu" and rec["unit"] == "TFLOP/s"
    assert rec["algorithmic_flops_per_launch"] == flops
    assert rec["achieved"] == pytest.approx(flops / 2.5e-3 / 1e12)
    assert rec["peak"] == pytest.approx(2 * 128 * 148 * 1965e6 / 1e12)
    assert rec["frac"] == pytest.approx(rec["achieved"] / rec["peak"])
    assert rec["hbm_view"]["unit"] == "GB/s" and rec["hbm_view"]["achieved"] > 0


def test_roofline_hbm_for_the_forward_pipeline():
    from fourier_neural_spectral_fno_b200 import synth
    bench = _bench_module()
    wl = synth.WORKLOADS["fno2d_f32_b16_w32_256sq_m16"]
    rec = bench.roofline_record("epi_block_fwd_pipe", 0.1, wl, 148)
    act = 16 * 32 * 65536 * 4
    spec = 16 * 32 * 16 * 32 * 8
    assert rec["bound"] == "hbm" and rec["unit"] == "GB/s"
    assert rec["algorithmic_bytes_per_launch"] == 2 * act + spec
    assert rec["achieved"] == pytest.approx((2 * act + spec) / 0.1e-3 / 1e9)
    assert rec["peak"] == pytest.approx(bench.hbm_peak()[0])   # measured copy peak, else fallback


def test_traffic_records_and_bench_name_the_same_source():
    """A traffic record is keyed by (timing tag, hash of the kernel's source file); bench.py
    looks the hash up through its own tag -> file table, so the two tables must agree for
    every kernel the recorder knows, or a fresh record would never be used."""
    import importlib.util
    from fourier_neural_spectral_fno_b200 import profile_traffic as pt
    spec = importlib.util.spec_from_file_location("bench_mod", BENCH)
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    pairs = set(pt.KERNELS.values()) | {(t, "epilogue.cu") for t in pt.EPILOGUE_TAGS.values()}
    pairs |= {("fwd_plane_dz", "transform_plane.cu"), ("mix_fwd_tc", "mix_tc.cu"),
              ("mix_bwd_dx_tc", "mix_tc.cu"), ("mix_bwd_dr_tc", "mix_tc.cu")}
    for tag, src in sorted(pairs):
        path = os.path.join(ROOT, "fourier_neural_spectral_fno_b200", "csrc", src)
        assert os.path.isfile(path), src
        assert bench.kernel_source_sha(tag) == pt.source_sha(src), (tag, src)
