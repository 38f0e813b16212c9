"""Launch plans, geometries and schedules of the kernels, checked on the host
(each checker includes the kernel's translation unit and calls its own
planning code; nothing is launched).

Launch plans of the batched-decode stream kernel:

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


def _build_and_run(sources, min_checked):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "check")
        cmd = [nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
               "-I" + os.path.join(ROOT, "include"),
               "-I" + os.path.join(ROOT, "up_projection_b200", "csrc"),
               *[os.path.join(ROOT, s) for s in sources], "-o", exe]
        p = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
        assert p.returncode == 0, p.stdout + p.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr
        assert int(r.stdout.split()[1]) >= min_checked


def test_stream_plans_keep_memory_bounds():
    _build_and_run(["tests/stream_plan_check.cu", "up_projection_b200/csrc/tmap.cu"], 100000)


def test_backward_schedule_is_an_exact_partition():
    """The backward GEMMs' static schedule (dX tiles round-robin, then dW
    tiles in the order the CTAs free up) covers every dX and dW tile exactly
    once, dX before dW within each CTA, for tile counts, grids and cost
    ratios including the edge cases (bwd_sched_check.cu)."""
    _build_and_run(["tests/bwd_sched_check.cu"], 8000)


def test_dx_split_tail_is_an_exact_partition():
    """fp32 dX alone: the tail tiles split along the reduction are covered
    chunk by chunk exactly once, the whole tiles round-robin exactly once, at
    most one part per CTA after its whole tiles, never more parts than CTAs
    (dx_split_check.cu)."""
    _build_and_run(["tests/dx_split_check.cu"], 1000)


def test_decode_geometry_for_every_supported_k():
    """Decode kernel: for every K it accepts, both launch forms and M <= 8,
    the shared-memory layout fits (two CTAs per SM on the small budget), the
    TMA boxes and regions are legal and aligned, and the transaction counts
    stay below the mbarrier limit (decode_geometry_check.cu)."""
    _build_and_run(["tests/decode_geometry_check.cu", "up_projection_b200/csrc/tmap.cu"], 20000)
