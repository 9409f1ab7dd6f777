"""Multi-rank host logic of the bench on CPU (gloo, world size 2).

Each rank steps its own bucket (weak scaling, no data-path collective); the
only collective is the all-reduce that takes the slowest rank's time.  This
checks that logic with two real processes and the gloo backend.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local_ms = [10.0, 25.0][rank]            # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        value, per_step = bench.job_throughput(ms, 5, world, 1_000_000_000)
        dist.barrier()
        out[rank] = (ms, value, per_step)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for r in range(world):
        ms, value, per_step = res[r]
        assert ms == 25.0                        # max over ranks on every rank
        assert per_step == pytest.approx(5.0)
        # two ranks x 1 GB per step in 5 ms
        assert value == pytest.approx(2 * 1e9 / 5e-3 / 1e9)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    v, per = bench.job_throughput(10.0, 10, 1, 2_000_000_000)
    assert per == 1.0 and v == pytest.approx(2000.0)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the CPU oracle arm) prints one JSON line
    with the contract's keys and its own metric, unit and e2e block."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1"], capture_output=True, text=True, timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1


def test_algorithmic_bytes_of_the_tiny_and_llama_buckets():
    """16 B per parameter, 16 B per block, 2 B per padding element: the tiny
    bucket (131,840 parameters, 34 blocks, 15,616 padding) moves 2,141,216 B
    per step, the Llama bucket 3,490,693,152 B; copy-in moves 4 B per
    parameter."""
    import ragged_bucket_layout_b200 as rb
    import synth
    expect = {"tiny_m4": (131840, 34, 15616, 2141216), "llama_layer_m8": (218112000, 53250, 24576, 3490693152)}
    for name, (P, B, pad, total) in expect.items():
        w = synth.workload(name)
        r, c, k = w.arrays()
        info = rb.dbuf_plan_info(rb.dbuf_plan(r, c, k, w.m, 16))
        st = bench.workload_stats(w, info)
        assert (st["params"], st["blocks"], st["padding"], st["step_bytes"]) == (P, B, pad, total)
        assert st["copy_in_bytes"] == 4 * P


def test_reference_arm_on_other_ranks_exits_without_work():
    """Under torchrun with N > 1 only rank 0 runs and prints the reference
    arm; another rank exits 0 at once and prints no JSON line."""
    import subprocess
    import sys
    import time
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    t0 = time.monotonic()
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "1"], capture_output=True, text=True, timeout=300, cwd=root,
                         env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    assert not [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert time.monotonic() - t0 < 120
