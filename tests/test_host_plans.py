"""The kernels' host-side planning arithmetic (tests/host_plans.cu): compiled
from the library's headers with nvcc as a host program and run on the CPU."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_host_plans(tmp_path):
    exe = str(tmp_path / "host_plans")
    subprocess.check_call([NVCC if os.path.exists(NVCC) else "nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-std=c++17", "--expt-relaxed-constexpr", "-O1", "-o", exe,
                           os.path.join(HERE, "host_plans.cu")])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout + out.stderr
