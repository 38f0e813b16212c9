"""Launch plans of the batched-decode stream kernel, checked on the host.

`stream_plan_check.cu` includes the kernel's translation unit (the kernel is
compiled, never launched) and runs its planning code for every routed shape
over a range of SM counts, checking the conditions the kernel relies on for
memory safety: shared-memory bounds (including the A operand's rows read past
the X box), B-operand reads inside their stage, TMEM columns within the SM's
share, TMA box dimensions, the epilogue's staging chunk and the MMA shapes."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


def test_stream_plans_keep_memory_bounds():
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "stream_plan_check")
        cmd = [nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
               "-I" + os.path.join(ROOT, "include"),
               "-I" + os.path.join(ROOT, "up_projection_b200", "csrc"),
               os.path.join(ROOT, "tests", "stream_plan_check.cu"),
               os.path.join(ROOT, "up_projection_b200", "csrc", "tmap.cu"), "-o", exe]
        p = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
        assert p.returncode == 0, p.stdout + p.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr
        assert int(r.stdout.split()[1]) > 100000
