"""Host logic of the tensor-core scan without a GPU: the launch plan (output
segments, state parts, the carry's segment starts, workspace regions) is
checked over a grid of batch sizes, head counts and lengths by compiling the
planner with a small host program (tests/scan_plan_check.cu) and running it."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    return None


def test_scan_plan_geometry_and_workspace():
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not found")
    csrc = os.path.join(ROOT, "selective_ssm_sequence_b200", "csrc")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "scan_plan_check")
        cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
               "-I", os.path.join(ROOT, "include"), "-I", csrc,
               os.path.join(ROOT, "tests", "scan_plan_check.cu"), os.path.join(csrc, "tc_host.cu"), "-o", exe]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stdout + r.stderr
        # no device: the planner's SM count falls back to 148
        env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
        r = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=120)
        assert r.returncode == 0, r.stdout + r.stderr
        assert " 0 failures" in r.stdout, r.stdout
