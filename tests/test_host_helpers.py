"""Host-side logic of the CUDA path, checked on the CPU: the visible-range helpers that every
kernel masks with (compiled with nvcc as a host program, no GPU needed)."""

import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_window_ranges_agree_with_the_visibility_rule():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "window_ranges_check")
        src = os.path.join(ROOT, "tests", "host", "window_ranges_check.cu")
        build = subprocess.run([nvcc, "-std=c++17", "-O1", "-Wno-deprecated-gpu-targets",
                                "-I", os.path.join(ROOT, "exact_io_aware_91_b200", "csrc"),
                                "-I", os.path.join(ROOT, "include"), src, "-o", exe],
                               capture_output=True, text=True)
        assert build.returncode == 0, build.stderr
        run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert run.returncode == 0, run.stdout + run.stderr
        assert run.stdout.startswith("ok ")
