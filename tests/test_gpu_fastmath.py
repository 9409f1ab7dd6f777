"""The step kernel's fast square root and division equal CUDA's correctly
rounded __fsqrt_rn and __fdiv_rn on the ranges the kernel sends to them:
the square root and the reciprocal exhaustively (about 1.9e9 and 1.0e9
inputs), the quotient on 1.7e10 random and 1.4e11 structured pairs, and the
per-block code factors on every 32-bit pattern (a few seconds on a B200)."""
import os
import re
import subprocess

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def report(tmp_path_factory):
    exe = tmp_path_factory.mktemp("fastmath") / "fastmath_check"
    subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
                           "-I", os.path.join(ROOT, "ragged_bucket_layout_b200", "csrc"),
                           "-o", str(exe), os.path.join(ROOT, "tests", "fastmath_check.cu")])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout + out.stderr
    res = {}
    for name, n, bad in re.findall(r"(\w+) checked=(\d+) mismatches=(\d+)", out.stdout):
        res[name] = (int(n), int(bad))
    return res, out.stdout


@pytest.mark.parametrize("name,min_checked", [("sqrt", 1_800_000_000), ("rcp", 1_000_000_000),
                                              ("div_random", 17_000_000_000), ("div_grid", 137_000_000_000),
                                              ("block_factors", 8_589_934_592)])
def test_fast_path_is_exact_on_its_range(report, name, min_checked):
    res, text = report
    assert name in res, text
    checked, bad = res[name]
    assert checked >= min_checked, text
    assert bad == 0, text
