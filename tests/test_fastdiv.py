"""The unit-index division of the attention kernel (make_fastdiv in csrc/sm100_ptx.cuh): its
magic numbers give n / d exactly for 31-bit dividends. A host program (tests/native/
fastdiv_check.cu, compiled here with nvcc, run on the CPU) checks every n < 2^31 for d = 48 and
boundary / sampled dividends for every d <= 5000 and some large d."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_fastdiv_exact(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "fastdiv_check")
    subprocess.run([nvcc, "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-o", exe, os.path.join(HERE, "native", "fastdiv_check.cu")], check=True)
    out = subprocess.run([exe, "48"], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout
