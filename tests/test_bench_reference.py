"""bench.py --impl reference on the CPU: the oracle arm's JSON line and its multi-rank behaviour.

The reference arm times the fp64 oracle on the host; under torchrun only rank 0
runs and prints, the other ranks exit 0 without work.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(rank, *extra):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "1",
                           "--reference-seconds", "2", *extra],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_line_on_rank0():
    r = _run(0)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "GB/s" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["warmup"] >= 3  # at least three warm-up steps, whatever is asked
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_other_ranks_exit_quietly():
    r = _run(1)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""



def test_reference_config_is_the_workload_config_of_our_arm():
    """Both arms describe the same workload: the reference line's config is what our arm's line carries
    for the same workload and arguments (the bounded sample is named in cpu_baseline.sample)."""
    sys.path.insert(0, ROOT)
    import bench

    r = _run(0, "--gpus", "2")
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    ours = bench.workload_config("llama_decode", bench.make_workload("llama_decode", 16), "auto", 2)
    assert line["config"] == ours
    assert "sequences per step" in line["cpu_baseline"]["sample"]
