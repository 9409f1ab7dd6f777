"""The step kernel's fast square root equals CUDA's correctly rounded
__fsqrt_rn on every float in the range the kernel sends to it (exhaustive,
about 1.9e9 inputs; a second on a B200)."""
import os
import re
import subprocess

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_fast_sqrt_is_exact_on_its_whole_range(tmp_path):
    exe = tmp_path / "fastmath_check"
    subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
                           "-I", os.path.join(ROOT, "ragged_bucket_layout_b200", "csrc"),
                           "-o", str(exe), os.path.join(ROOT, "tests", "fastmath_check.cu")])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    m = re.search(r"checked=(\d+) mismatches=(\d+)", out.stdout)
    assert m, out.stdout
    assert int(m.group(1)) > 1_800_000_000
    assert int(m.group(2)) == 0, out.stdout
