"""bench.py on the CPU: the reference arm (the oracle timed on the host cores)
prints one JSON line with the keys the benchmark contract names, ranks other
than 0 exit quietly, and the GPU arm refuses to run without a CUDA device
instead of falling back to anything."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(args, env=None):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, timeout=600, env=env, cwd=ROOT)


def _json_lines(out):
    return [json.loads(x) for x in out.splitlines() if x.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    r = _bench(["--impl", "reference", "--config", "1", "--steps", "3", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    j = lines[0]
    assert j["impl"] == "reference"
    assert j["value"] > 0 and j["ms_per_step"] > 0
    assert (j["n_gpus"], j["steps"], j["warmup"]) == (1, 3, 3)
    assert j["higher_is_better"] is True and j["scaling"] == "weak" and j["vs_baseline"] is None
    assert j["data"] == "synthetic" and j["config"]["workload"] == "tiny-fp32-3x48"
    assert isinstance(j["metric"], str) and j["unit"] == "token·heads/s"
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == j["value"] and cb["unit"] == j["unit"]
    e = j["e2e"]
    assert e["value"] == j["value"] and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = _bench(["--impl", "reference", "--config", "1", "--steps", "3", "--warmup", "3"], env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    assert _json_lines(r.stdout) == []


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a CUDA device")
def test_gpu_arm_fails_loudly_without_a_device():
    r = _bench(["--config", "1", "--steps", "3", "--warmup", "3"])
    assert r.returncode != 0
    assert "needs a CUDA device" in r.stderr
    assert _json_lines(r.stdout) == []
