"""The C-ABI from plain C99: tests/c_abi_check.c includes only include/dbuf.h,
links libdbuf.so, and calls the host-only entry points (planner, shards,
rank buckets, work table, required bytes, row-wise layout, error path).  Its numbers must
equal what the Python binding reports (CPU only)."""
import os
import re
import subprocess

import ragged_bucket_layout_b200 as rb
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c99_caller(tmp_path):
    exe = tmp_path / "c_abi_check"
    libdir = os.path.dirname(rb.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                           "-o", str(exe), os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", libdir, "-ldbuf",
                           f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    w = synth.workload("tiny_m4")
    r, c, k = w.arrays()
    p = rb.dbuf_plan(r, c, k, w.m, 16)
    info = rb.dbuf_plan_info(p)
    m = re.search(r"slice=(\d+) bucket=(\d+) padding=(\d+) n_blocks=(\d+) offsets=(\d+),(\d+),(\d+)", out.stdout)
    assert m, out.stdout
    assert [int(x) for x in m.groups()] == [info["slice"], info["bucket"], info["padding"], info["n_blocks"],
                                            *info["offsets"]]
    m = re.search(r"entries=(\d+) covered=(\d+) required_bytes=(\d+)", out.stdout)
    assert int(m.group(1)) == len(rb.dbuf_work_table(p))
    assert int(m.group(2)) == info["bucket"]
    assert int(m.group(3)) == rb.dbuf_required_bytes(p)
    assert re.search(r"bad=%d msg_nonempty=1" % rb.DBUF_EINVAL, out.stdout), out.stdout
    chunk, q, _ = rb.dbuf_rowwise_layout(r, c, 4)
    assert f"rowwise chunk={chunk} q={q[0]},{q[1]},{q[2]}" in out.stdout
    ends = [b for a, b in rb.dbuf_plan_shards(p, w.m)[0]]
    assert "shards_w=" + ",".join(map(str, ends)) in out.stdout, out.stdout
    R = rb.dbuf_plan_rank(p, 3)
    ri = rb.dbuf_plan_info(R)
    assert f"rank3 first_block={R.first_block} padding={ri['padding']} n_blocks={ri['n_blocks']}" in out.stdout
    assert f"rank_bad={rb.DBUF_EINVAL} null_out=1" in out.stdout, out.stdout
    assert f"dims=3,4 rank3_dims={R.n},1" in out.stdout, out.stdout


import pytest  # noqa: E402


@pytest.mark.gpu
def test_c99_caller_on_the_device(tmp_path):
    """Plain C99 drives the whole device path: library-allocated bucket,
    resident step, host-buffer step, status word."""
    exe = tmp_path / "c_abi_gpu"
    libdir = os.path.dirname(rb.LIB_PATH)
    cuda = "/usr/local/cuda"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(cuda, "include"), "-o", str(exe),
                           os.path.join(ROOT, "tests", "c_abi_gpu.c"), "-L", libdir, "-ldbuf",
                           "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm", f"-Wl,-rpath,{libdir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    m = re.search(r"first_step_worst_abs_err=(\S+) second_step_param=(\S+) status=(\d+)", out.stdout)
    assert m and float(m.group(1)) < 1e-6 and int(m.group(3)) == 0, out.stdout
    assert 0.0075 < float(m.group(2)) < 0.0085     # two steps of about lr each from 0.01
