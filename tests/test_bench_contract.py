"""The bench.py contract, checked without a GPU.

* The reference arm (the float64 oracle on host cores) prints one JSON line
  with the contract keys, a cpu_baseline and an e2e object.
* The GPU arm refuses to run without CUDA instead of falling back to a CPU
  path.
* Under a multi-rank launch the reference arm runs on rank 0 alone; the other
  ranks exit 0 without work or output.
* Argument checks: at least 3 warm-up steps; the reference arm is forward only.
* The kernel-source hash that ties the committed DRAM counters to the code
  ignores comments and whitespace and changes with any code edit.
"""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def _run(*args, env=None, timeout=600):
    e = dict(os.environ)
    e.pop("RANK", None)
    e.pop("WORLD_SIZE", None)
    e.pop("LOCAL_RANK", None)
    if env:
        e.update(env)
    return subprocess.run([sys.executable, BENCH, *args], capture_output=True, text=True, env=e,
                          timeout=timeout, cwd=ROOT)


def test_reference_arm_prints_the_contract_line():
    r = _run("--impl", "reference", "--workload", "small", "--steps", "2", "--warmup", "3",
             "--reference-rows", "64")
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("small")


def test_reference_arm_runs_on_rank_zero_only():
    args = ("--impl", "reference", "--gpus", "2", "--workload", "small", "--steps", "1",
            "--warmup", "3", "--reference-rows", "32")
    other = _run(*args, env={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert other.returncode == 0, other.stderr
    assert other.stdout.strip() == ""
    root = _run(*args, env={"RANK": "0", "LOCAL_RANK": "0", "WORLD_SIZE": "2"})
    assert root.returncode == 0, root.stderr
    lines = [ln for ln in root.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU refusal")
def test_gpu_arm_refuses_without_cuda():
    r = _run("--steps", "3", "--warmup", "3", "--no-cpu-baseline", timeout=300)
    assert r.returncode != 0
    assert "CUDA" in r.stderr


def test_argument_checks():
    r = _run("--warmup", "2", timeout=120)
    assert r.returncode != 0 and "--warmup must be >= 3" in r.stderr
    r = _run("--impl", "reference", "--pass", "bwd", timeout=120)
    assert r.returncode != 0 and "forward oracle only" in r.stderr


def test_kernel_hash_ignores_comments_but_not_code(tmp_path):
    """The committed DRAM counters stay attached to the kernel across comment
    edits and are dropped by any code change."""
    sys.path.insert(0, ROOT)
    import bench

    base = "__global__ void k(int* p) {\n  p[0] = 1;  // store\n}\n"
    variants = {
        "same": base,
        "comments": "/* header\n   text */\n__global__ void k(int* p) {\n  // new note\n  p[0] = 1;\n}\n",
        "spacing": "__global__   void k(int* p)\n{ p[0] = 1; }",
        "code": "__global__ void k(int* p) {\n  p[0] = 2;  // store\n}\n",
    }
    hashes = {}
    for name, text in variants.items():
        f = tmp_path / f"{name}.cuh"
        f.write_text(text)
        hashes[name] = bench.kernel_hash((str(f),))
    assert hashes["same"] == hashes["comments"] == hashes["spacing"]
    assert hashes["code"] != hashes["same"]
