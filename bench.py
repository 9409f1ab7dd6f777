"""Benchmark of the fused ragged-bucket 8-bit Adam step on B200.

Metric: bucket step GB/s (algorithmic bytes 16*P + 16*B + 2*Pad per step:
P parameters, B quantisation blocks, Pad padding elements), params/s and the
fraction of measured HBM bandwidth; copy-in GB/s of the per-tensor gradient
gather (4 bytes per parameter) beside it.

Default workload: one Llama-style layer (hidden 4096, GQA 32q/8kv, SwiGLU
14336; 218,112,000 fp32 parameters, 1-row blocks) in a bucket of m=8 slices.

Usage (one process per GPU; N>1 under torch.distributed.run):
    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N>1 every rank steps its own bucket of the same shape (one layer per
rank): no data-path collective, weak scaling; the timing is the max over
ranks of device time.  ``--impl reference`` times the CPU oracle instead (the
only other place this script runs it) on a bounded sample of the workload.
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth.rng import STREAM_GRAD, STREAM_PARAM  # noqa: E402
from synth.workloads import GRAD_SIGMA, PARAM_SIGMA  # noqa: E402

METRIC = "fused 8-bit Adam bucket step GB/s & params/s vs HBM roofline; copy-in GB/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama_layer_m8", choices=synth.WORKLOAD_NAMES)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-copy-in", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--graph-steps", type=int, default=10,
                    help="steps per CUDA graph for the launch-overhead-free figure (0: skip)")
    return ap.parse_args()


def workload_stats(w, info):
    P, B, pad = w.numel, info["n_blocks"], info["padding"]
    return dict(params=P, blocks=B, padding=pad, bucket=info["bucket"],
                step_bytes=16 * P + 16 * B + 2 * pad, copy_in_bytes=4 * P)


NOMINAL_HBM_GBS = 8000.0   # B200 nominal HBM3e bandwidth (8 TB/s, the DGX figure)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, burst copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def measured_bf16_peak():
    """Burst cuBLAS bf16 TFLOP/s from MEASURED_PEAKS.json, else the fallback 1590."""
    try:
        return float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"])
    except Exception:
        return 1590.0


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("dbuf.cu", "internal.h", "step_kernel.cuh", "fastmath.cuh", "tma.cuh", "tables.h"):
        h.update(open(os.path.join(ROOT, "ragged_bucket_layout_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, stats):
    """DRAM bytes per launch of the step kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"adam8_step_kernel_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m_src = re.search(r"kernel source hash: `([0-9a-f]+)`", txt)
    m_b = re.search(r"dram bytes per launch: ([0-9.eE+]+)", txt)
    if not m_src or not m_b or m_src.group(1) != kernel_source_hash():
        return None
    return float(m_b.group(1))


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index, period=0.005):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def host_inputs(w, seed_offset=0):
    """Per-tensor fp32 parameters and bf16 gradient bits from the generator."""
    r, c, _ = w.arrays()
    n = r * c
    cum = np.concatenate([[0], np.cumsum(n)])
    kp = synth.stream_key(w.seed + seed_offset, STREAM_PARAM)
    kg = synth.stream_key(w.seed + seed_offset, STREAM_GRAD * 1000 + 1)
    params = [synth.normal_f32(kp, int(cum[i]), int(n[i]), PARAM_SIGMA) for i in range(len(n))]
    grads = [synth.normal_bf16(kg, int(cum[i]), int(n[i]), GRAD_SIGMA) for i in range(len(n))]
    return params, grads


def hp_at(t):
    return dict(synth.HPARAMS, step=t)


# ------------------------------------------------------------ ranks

def max_over_ranks(x, dist=None, device="cpu"):
    """Max of a per-rank float over all ranks (one all-reduce; identity on one rank)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ms_total_max, steps, world, bytes_per_step):
    """Whole-job GB/s: every rank moves bytes_per_step per step (weak
    scaling); time is the slowest rank's."""
    per_step_ms = ms_total_max / steps
    return world * bytes_per_step / (per_step_ms * 1e-3) / 1e9, per_step_ms


# ------------------------------------------------------------ CPU oracle

def oracle_sample(w, info, offsets, fraction_blocks):
    """Blocks of the first slice (rank 0's shard) of the planned bucket, as
    compact host arrays for the oracle."""
    import oracle
    r, c, k = w.arrays()
    start, length = oracle.blocks(r, c, k, offsets)
    s = info["slice"]
    sel = np.nonzero(start < s)[0]
    if fraction_blocks < 1.0:
        sel = sel[: max(1, int(len(sel) * fraction_blocks))]
    lens = length[sel]
    st = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    tot = int(lens.sum())
    arr = dict(p=synth.normal_f32(synth.stream_key(w.seed, STREAM_PARAM), 0, tot, PARAM_SIGMA),
               g=synth.normal_bf16(synth.stream_key(w.seed, STREAM_GRAD * 1000 + 1), 0, tot, GRAD_SIGMA),
               mq=np.zeros(tot, np.int8), vq=np.zeros(tot, np.uint8), pb=np.zeros(tot, np.uint16),
               sm=np.zeros(len(sel), np.float32), sv=np.zeros(len(sel), np.float32))
    return st, lens, arr


def oracle_step(st, lens, arr, t, gscale, threads):
    import oracle
    oracle.adam8_step(st, lens, np.arange(lens.size), arr["p"], arr["g"], arr["mq"], arr["vq"], arr["sm"],
                      arr["sv"], arr["pb"], hp_at(t), t, gscale, threads)


def cpu_baseline(w, info, offsets, seconds):
    threads = os.cpu_count() or 1
    st, lens, arr = oracle_sample(w, info, offsets, 1.0)
    P, B = int(lens.sum()), int(lens.size)
    t0 = time.perf_counter()
    oracle_step(st, lens, arr, 1, 1.0 / w.m, threads)
    one = time.perf_counter() - t0
    reps = max(1, min(200, int(seconds / max(one, 1e-6))))
    t0 = time.perf_counter()
    for t in range(2, 2 + reps):
        oracle_step(st, lens, arr, t, 1.0 / w.m, threads)
    dt = time.perf_counter() - t0
    nbytes = (16 * P + 16 * B) * reps
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"slice 0 of {w.m} ({P} params, {B} blocks) of {w.name}, {reps} steps, "
                      f"{dt:.1f} s, OpenMP over blocks",
            "params_per_s": P * reps / dt}


def run_reference(args):
    """The CPU oracle as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = synth.workload(args.workload)
    r, c, k = w.arrays()
    st_, offsets, s = oracle.plan(r, c, k, w.m, w.align)
    info = dict(slice=s, bucket=s * w.m)
    threads = os.cpu_count() or 1
    # each step: the oracle on 1/4 of rank 0's slice (bounded CPU time)
    st, lens, arr = oracle_sample(w, info, offsets, 0.25)
    P, B = int(lens.sum()), int(lens.size)
    for t in range(1, args.warmup + 1):
        oracle_step(st, lens, arr, t, 1.0 / w.m, threads)
    t0 = time.perf_counter()
    for t in range(args.warmup + 1, args.warmup + args.steps + 1):
        oracle_step(st, lens, arr, t, 1.0 / w.m, threads)
    dt = time.perf_counter() - t0
    value = (16 * P + 16 * B) * args.steps / dt / 1e9
    sample = f"1/4 of slice 0 of {w.m} ({P} params, {B} blocks) of {w.name} per step, OpenMP over blocks"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": {"workload": w.name, "params": P, "blocks": B, "m": w.m},
            "params_per_s": P * args.steps / dt,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ GPU arm

def _ensure_library():
    """Compile libdbuf.so with nvcc if this checkout has not built it yet (the
    package itself refuses to load without it)."""
    if os.path.exists(os.path.join(ROOT, "ragged_bucket_layout_b200", "libdbuf.so")):
        return
    import importlib.util
    spec = importlib.util.spec_from_file_location("_dbuf_build", os.path.join(ROOT, "ragged_bucket_layout_b200",
                                                                              "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def run_ours(args):
    import torch
    _ensure_library()
    import ragged_bucket_layout_b200 as rb

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    w = synth.workload(args.workload)
    r, c, k = w.arrays()
    t_plan = time.perf_counter()
    plan = rb.dbuf_plan(r, c, k, w.m, w.align)
    planner_ms = (time.perf_counter() - t_plan) * 1e3       # host, once at init
    info = rb.dbuf_plan_info(plan)
    stats = workload_stats(w, info)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        D = rb.DBuffer(plan, stream=stream)
        params, grads = host_inputs(w, seed_offset=rank)
        for v, x in zip(D.views(rb.DBUF_MASTER_F32), params):
            v.copy_(torch.from_numpy(x).view(v.shape), non_blocking=False)
        for v, x in zip(D.views(rb.DBUF_GRAD_BF16), grads):
            v.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).view(v.shape))
    stream.synchronize()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    gscale = 1.0 / w.m
    step_no = 0
    for _ in range(args.warmup):
        step_no += 1
        D.step(hp_at(step_no), gscale)
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step_no += 1
            D.step(hp_at(step_no), gscale)
        ev1.record(stream)
        ev1.synchronize()
        barrier()
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, dist, "cuda")
    status = D.device_status()
    if status != 0:
        raise RuntimeError(f"device status word {status}")
    value, per_step_ms = job_throughput(ms, args.steps, world, stats["step_bytes"])
    kernel_gbs = stats["step_bytes"] / (ms_local / args.steps * 1e-3) / 1e9

    # ---- the same steps replayed from a CUDA graph (no per-launch host
    # overhead; matters for small buckets).  The graph holds steps
    # t+1..t+G with their hyper-parameters fixed at capture.
    graph = None
    if args.graph_steps > 0:
        G = args.graph_steps
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(G):
                D.step(hp_at(step_no + 1 + i), gscale)
        step_no += G
        for _ in range(3):
            g.replay()
        reps = max(3, min(100, args.steps // G))
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g0.record(stream)
            for _ in range(reps):
                g.replay()
            g1.record(stream)
        g1.synchronize()
        gms = max_over_ranks(g0.elapsed_time(g1), dist, "cuda") / (reps * G)
        graph = {"steps_per_graph": G, "replays": reps, "ms_per_step": gms,
                 "value": world * stats["step_bytes"] / (gms * 1e-3) / 1e9, "unit": UNIT}
        del g

    # ---- end to end through the host-buffer entry point
    S = info["bucket"]
    e2e = None
    if args.e2e_steps > 0:
        g_host = D.array(rb.DBUF_GRAD_BF16).view(torch.int16).cpu().pin_memory()
        p_host = torch.empty(S, dtype=torch.int16).pin_memory()
        for _ in range(3):
            step_no += 1
            D.step_host(hp_at(step_no), gscale, g_host.data_ptr(), p_host.data_ptr())
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            step_no += 1
            D.step_host(hp_at(step_no), gscale, g_host.data_ptr(), p_host.data_ptr())
        e1.record(stream)
        e1.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1), dist, "cuda") / args.e2e_steps
        # The PCIe bound of this path: the same bytes copied in and out at
        # once, pinned, with nothing else running.
        d_in = torch.empty(S, dtype=torch.int16, device="cuda")
        d_out = torch.empty(S, dtype=torch.int16, device="cuda")
        h_back = torch.empty(S, dtype=torch.int16).pin_memory()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

        def both_ways():
            with torch.cuda.stream(s_in):
                d_in.copy_(g_host, non_blocking=True)
            with torch.cuda.stream(s_out):
                h_back.copy_(d_out, non_blocking=True)
            s_in.synchronize()
            s_out.synchronize()
        both_ways()
        t0 = time.perf_counter()
        for _ in range(3):
            both_ways()
        pcie_ms = (time.perf_counter() - t0) / 3 * 1e3
        ceiling = stats["step_bytes"] / (pcie_ms * 1e-3) / 1e9
        e2e = {"value": world * stats["step_bytes"] / (ems * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": 2 * S, "d2h_bytes_per_step": 2 * S, "ms_per_step": ems,
               "path": "dbuf_adam8_step_host (pinned host grads in, bf16 params out)",
               "pcie_bound": {"copy_in_and_out_ms": pcie_ms, "ceiling_gbs": ceiling,
                              "frac": (stats["step_bytes"] / (ems * 1e-3) / 1e9) / ceiling}}
        del d_in, d_out, h_back

    # ---- copy-in baseline on the same workload (rank-local, informative)
    copy_in = None
    if not args.no_copy_in:
        sep = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda().view(int(rr), int(cc))
               for x, rr, cc in zip(grads, r, c)]
        torch.cuda.synchronize()
        reps = max(5, min(200, args.steps // 5))
        with torch.cuda.stream(stream):
            for _ in range(3):
                D.pack(sep, gscale)
            a0, a1, a2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a0.record(stream)
            for _ in range(reps):
                D.pack(sep, gscale)
            a1.record(stream)
            for _ in range(reps):
                D.pack(sep, gscale)
                step_no += 1
                D.step(hp_at(step_no), 1.0)
            a2.record(stream)
        a2.synchronize()
        pack_ms = a0.elapsed_time(a1) / reps
        path_ms = a1.elapsed_time(a2) / reps
        copy_in = {"gbs": stats["copy_in_bytes"] / (pack_ms * 1e-3) / 1e9, "pack_ms": pack_ms,
                   "copy_in_path_ms": path_ms, "zero_copy_path_ms": ms_local / args.steps,
                   "copy_bytes": stats["copy_in_bytes"], "tensors": len(sep),
                   "saved_ms": path_ms - ms_local / args.steps}
        # DBuffer group operations beyond scale/zero on the same bucket:
        # accumulate (6 B/param), norm (2 B/bucket element), clipped step.
        norm_out = torch.zeros(1, dtype=torch.float64, device="cuda")
        with torch.cuda.stream(stream):
            b0, b1, b2, b3 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
            D.accumulate(sep, gscale)
            D.grad_norm(gscale, norm_out)
            b0.record(stream)
            for _ in range(reps):
                D.accumulate(sep, gscale)
            b1.record(stream)
            for _ in range(reps):
                D.grad_norm(gscale, norm_out)
            b2.record(stream)
            for _ in range(reps):
                step_no += 1
                D.step_clipped(hp_at(step_no), gscale, 1.0, norm_out)
            b3.record(stream)
        b3.synchronize()
        acc_ms, norm_ms, clip_ms = b0.elapsed_time(b1) / reps, b1.elapsed_time(b2) / reps, b2.elapsed_time(b3) / reps
        copy_in["group_ops"] = {
            "accumulate_gbs": 6 * stats["params"] / (acc_ms * 1e-3) / 1e9, "accumulate_ms": acc_ms,
            "grad_norm_gbs": 2 * stats["bucket"] / (norm_ms * 1e-3) / 1e9, "grad_norm_ms": norm_ms,
            "clipped_step_ms": clip_ms, "clipped_step_gbs": (stats["step_bytes"] + 2 * stats["bucket"]) / (clip_ms * 1e-3) / 1e9}
        # Row-wise (FSDP2-style) baseline: the interleaved copy-in before the
        # ReduceScatter and copy-out after the AllGather that the bucket
        # layout does without, on the same tensors and m.
        R = rb.Rowwise(r, c, w.m, stream=stream)
        flat = torch.empty(w.m * R.chunk, dtype=torch.bfloat16, device="cuda")
        outs = [torch.empty_like(x) for x in sep]
        with torch.cuda.stream(stream):
            R.copy_in(sep, gscale, flat, stream=stream)
            R.copy_out(flat, outs, stream=stream)
            r0, r1, r2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            r0.record(stream)
            for _ in range(reps):
                R.copy_in(sep, gscale, flat, stream=stream)
            r1.record(stream)
            for _ in range(reps):
                R.copy_out(flat, outs, stream=stream)
            r2.record(stream)
        r2.synchronize()
        if R.status(stream=stream) != 0:
            raise RuntimeError("row-wise copy status word set")
        in_ms, out_ms = r0.elapsed_time(r1) / reps, r1.elapsed_time(r2) / reps
        copy_in["rowwise_baseline"] = {
            "copy_in_gbs": stats["copy_in_bytes"] / (in_ms * 1e-3) / 1e9, "copy_in_ms": in_ms,
            "copy_out_gbs": stats["copy_in_bytes"] / (out_ms * 1e-3) / 1e9, "copy_out_ms": out_ms,
            "gathered_elems": w.m * R.chunk,
            "copies_vs_step": (in_ms + out_ms) / (ms_local / args.steps)}
        R.close()
        del sep, flat, outs

        # Distributed Muon on the bucket's matrices (the pages' other case
        # study): momentum, bf16 Newton-Schulz on the tensor cores (cuBLAS
        # GEMMs, fp32 accumulation), update; timed per step over all of them.
        ids = [i for i, t in enumerate(w.tensors) if t.rows >= 2 and t.cols >= 2]
        if ids:
            M = rb.Muon(D, ids)
            hpm = dict(rb.MUON_DEFAULTS)
            M.step(hpm, gscale)
            mreps = 5
            with torch.cuda.stream(stream):
                m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                m0.record(stream)
                for _ in range(mreps):
                    M.step(hpm, gscale)
                m1.record(stream)
            m1.synchronize()
            muon_ms = m0.elapsed_time(m1) / mreps
            flops = 0
            for i in ids:
                sm, lg = min(int(r[i]), int(c[i])), max(int(r[i]), int(c[i]))
                flops += hpm["ns_steps"] * (4 * sm * sm * lg + 2 * sm ** 3)
            bf16_peak = measured_bf16_peak()
            copy_in["muon"] = {"tensors": len(ids), "ns_steps": hpm["ns_steps"], "ms_per_step": muon_ms,
                               "ns_flops_per_step": flops, "tflops": flops / (muon_ms * 1e-3) / 1e12,
                               "bf16_peak_tflops": bf16_peak,
                               "frac_of_bf16_peak": flops / (muon_ms * 1e-3) / 1e12 / bf16_peak,
                               "gemm": "cuBLAS bf16, fp32 accumulate"}
            M.close()

    peak, peak_src = measured_peak()
    roof = {"bound": "hbm", "achieved": kernel_gbs, "peak": peak, "unit": "GB/s", "frac": kernel_gbs / peak,
            "traffic": profiled_traffic(w.name, stats), "peak_source": peak_src,
            "frac_of_nominal_8tbs": kernel_gbs / NOMINAL_HBM_GBS,
            "kernel": "adam8_step_kernel", "algorithmic_bytes_per_launch": stats["step_bytes"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, info, np.array(info["offsets"]), args.cpu_seconds)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "params": stats["params"], "blocks": stats["blocks"],
                   "padding": stats["padding"], "padding_frac": stats["padding"] / stats["bucket"],
                   "planner_ms": planner_ms, "bucket_elems": stats["bucket"], "m": w.m,
                   "bytes_per_step": stats["step_bytes"],
                   "l2": f"inputs larger than L2 ({stats['step_bytes'] / 1e9:.2f} GB moved per step)",
                   "parallelism": f"dp{world} (one bucket per rank, no data-path collective)"},
        "params_per_s": world * stats["params"] / (per_step_ms * 1e-3),
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
        "clocks": clk.summary(), "cuda_graph": graph, "copy_in": copy_in,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    D.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
