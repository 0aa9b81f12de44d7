"""Host-side logic of the library that runs without a GPU: the once-only per-device set-up under concurrent
first calls (compiled with nvcc as a plain host program against the library's internal header)."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for c in (os.environ.get("CUDA_HOME", "") + "/bin/nvcc", "/usr/local/cuda/bin/nvcc"):
        if os.path.exists(c):
            return c
    return shutil.which("nvcc")


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not available")
def test_setup_once_runs_once_under_racing_threads():
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "setup_once")
        subprocess.run([_nvcc(), "-std=c++17", "-O2", "-Wno-deprecated-gpu-targets",
                        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "ball_tree_sparse_b200", "csrc"),
                        os.path.join(ROOT, "tests", "host", "setup_once.cu"), "-o", exe],
                       check=True, capture_output=True, timeout=300)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert r.returncode == 0, r.stdout + r.stderr
