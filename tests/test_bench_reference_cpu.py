"""The reference arm of bench.py runs on the CPU (it times the oracle), so its contract
is checked here: one JSON line on rank 0 with the fields the driver reads, and a quiet
exit 0 on the other ranks."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(env_extra):
    env = dict(os.environ)
    env.update(env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "3"], capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    res = run_bench({"RANK": "0", "WORLD_SIZE": "1", "LOCAL_RANK": "0"})
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["config"]["workload"] and "model" not in line["config"]


def test_reference_arm_other_ranks_exit_quietly():
    res = run_bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.strip() == ""


def test_gpus_flag_launches_the_ranks_itself():
    """`bench.py --gpus 2` started as one process runs two ranks (torch.distributed.run on
    this node); the reference arm needs no GPU, so the launcher is checked here: one
    contract line, from rank 0, that counts both ranks."""
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                             "MASTER_PORT")}
    env["OMP_NUM_THREADS"] = "2"
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env, timeout=900,
                         cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"]["parallelism"] == "dp2"


def test_gpus_flag_must_match_the_launched_world():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT,
                         env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"))
    assert res.returncode != 0
    assert "WORLD_SIZE is 1" in res.stderr


def test_peaks_file_forms(tmp_path):
    """MEASURED_PEAKS.json may hold plain numbers or records; anything unusable falls
    back per key, and the source names it."""
    import json
    import bench
    p = tmp_path / "peaks.json"
    assert bench.load_peaks(str(tmp_path / "absent.json")) == (bench.FALLBACK_PEAKS, "fallback")
    p.write_text(json.dumps({"hbm_gbs": 6538.0, "bf16_tflops": 1638, "bf16_tflops_sustained": 1372.5}))
    peaks, src = bench.load_peaks(str(p))
    assert src == "measured" and peaks == {"hbm_gbs": 6538.0, "bf16_tflops": 1638.0, "bf16_tflops_sustained": 1372.5}
    p.write_text(json.dumps({"hbm_gbs": {"value": 6500}, "bf16_tflops": "n/a", "clocks": {"sm": 1965}}))
    peaks, src = bench.load_peaks(str(p))
    assert peaks["hbm_gbs"] == 6500.0 and peaks["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert src == "measured (fallback for bf16_tflops, bf16_tflops_sustained)"
    p.write_text("not json")
    assert bench.load_peaks(str(p))[1] == "fallback"
