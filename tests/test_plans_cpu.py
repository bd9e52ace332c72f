"""The launch plans that the stream-K tensor-core kernels index memory with,
checked on the host without a GPU.

`tests/plan_check.cu` is linked against the library's own objects and walks,
for 1,360 call shapes (B, N, H, tokens per block), every CTA range of the
reduce's and the apply's stream-K plans the way the kernels do.  It checks
that each granule is taken once, that every split-sum slot written is below
the workspace's slot count and is read once by the combine, that the
workspace size the C ABI reports holds those slots, that every cos/sin record
the transform can read lies inside the table, and that the multiply-shift
divisors divide exactly.  A plan error here would be an out-of-bounds write
on the GPU, so it is caught before any kernel runs.
"""
import os
import subprocess

import pytest

from block_causal_linear_b200 import build as la_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _library_objects():
    la_build.build()
    objdir = os.path.join(ROOT, "block_causal_linear_b200", "_build")
    objs = [os.path.join(objdir, s.replace(".cu", ".o")) for s in la_build.SOURCES]
    if not all(os.path.exists(o) for o in objs):
        # the shared library came without its objects: build them here
        la_build.build(force=True)
    return objs


def test_stream_k_plans_tables_and_divisors(tmp_path):
    if not os.path.exists(la_build.NVCC):
        pytest.skip("nvcc not found")
    objs = _library_objects()
    exe = tmp_path / "plan_check"
    subprocess.check_call([la_build.NVCC, "-std=c++17", "-O2", "--expt-relaxed-constexpr",
                           "-gencode", "arch=compute_100a,code=sm_100a",
                           os.path.join(ROOT, "tests", "plan_check.cu"), *objs,
                           "-cudart", "static", "-o", str(exe)])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok 1360 cases"), r.stdout
