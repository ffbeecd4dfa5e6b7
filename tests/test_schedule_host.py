"""The decode kernel's host-and-device schedule arithmetic (decode_kernels.cuh)
checked on the CPU: tests/host/decode_schedule_check.cu is compiled with nvcc
and run without a GPU."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not on PATH")
def test_decode_schedule_arithmetic():
    src = os.path.join(ROOT, "tests", "host", "decode_schedule_check.cu")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "check")
        subprocess.run(["nvcc", "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                        "--expt-relaxed-constexpr", src, "-o", exe], check=True, capture_output=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr
