"""Host-side checks of the mask/code bit tricks in csrc/quant_mask.cuh (no GPU needed).

The helpers are __host__ __device__; tests/host/qm_helpers_host.cu compiles them for the
host and checks them against their definitions (ternary code by IEEE division and
rint, keep bits by ranking, 2-bit packing, the PTX byte-permute semantics).
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"


@pytest.mark.skipif(not os.path.exists(NVCC), reason="nvcc not installed")
def test_quant_mask_helpers_host(tmp_path):
    exe = tmp_path / "qm_helpers_host"
    src = os.path.join(HERE, "host", "qm_helpers_host.cu")
    subprocess.run([NVCC, "-std=c++17", "-O1", "--expt-relaxed-constexpr", "-gencode",
                    "arch=compute_100a,code=sm_100a", "-o", str(exe), src], check=True,
                   capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.startswith("OK"), r.stdout + r.stderr
