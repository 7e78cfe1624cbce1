"""The bench's reference arm runs on CPU and prints the contract's JSON line;
the GPU arm's line is checked on the GPU machine."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config"}


def _run(args, timeout=600):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=timeout, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--config", "tiny", "--warmup", "3", "--steps", "1"])
    assert KEYS <= set(d)
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "Mtokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_gpus_two_starts_two_ranks():
    """`--gpus 2` without an outside launcher starts two ranks itself; they
    meet over a gloo group and rank 0 alone prints, labelled with both."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--config", "tiny", "--warmup", "3", "--steps", "1"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT, env={k: v for k, v in os.environ.items()
                                                     if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["ranks_joined"] == 2
    assert "rank 1/2: reference arm runs on rank 0 only" in out.stderr


def test_gpus_mismatch_is_refused():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--config", "tiny"], capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert out.returncode != 0 and "WORLD_SIZE=1" in out.stderr


def test_gpu_arm_refuses_more_gpus_than_visible():
    import torch

    if torch.cuda.device_count() >= 64:
        pytest.skip("64 devices visible")
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "64"], capture_output=True,
                         text=True, timeout=300, cwd=ROOT, env=env)
    assert out.returncode != 0 and "needs 64 CUDA devices" in out.stderr


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "1"], capture_output=True,
                         text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0


@pytest.mark.gpu
def test_gpu_arm_line():
    d = _run(["--config", "512p-17s", "--steps", "3", "--warmup", "3", "--e2e-steps", "1", "--no-cpu-baseline"])
    assert KEYS <= set(d)
    assert d["value"] > 0 and d["gpu_launches"] > 0
    assert d["roofline"]["unit"] == "GB/s" and 0 < d["roofline"]["frac"] < 2
    assert 0 < d["roofline"]["tensor_frac"] < 2 and 0 < d["roofline"]["path_frac"] < 2
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert set(d["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
