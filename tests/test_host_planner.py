"""Host-side logic of the product library (CPU only, no device calls).

* libdbuf.so loads and exports every entry point include/dbuf.h declares;
* the C++ planner (dbuf_plan) gives the oracle's layout bit for bit: on every
  workload bucket and on thousands of random small buckets;
* invalid descriptors and caps come back as status codes, not crashes;
* dbuf_required_bytes covers every bucket array.
"""
import os
import random
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle
import ragged_bucket_layout_b200 as rb
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    hdr = open(os.path.join(ROOT, "include", "dbuf.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    return sorted(set(re.findall(r"\b(dbuf_[a-z0-9_]+)\s*\(", hdr)))


def test_library_exports_every_declared_symbol():
    names = declared_entry_points()
    assert len(names) >= 15
    out = subprocess.run(["nm", "-D", "--defined-only", rb.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(rb.EXPORTED) == set(names)


def test_oracle_and_library_share_nothing():
    """The oracle library exports none of the product's symbols and the
    product none of the oracle's."""
    prod = subprocess.run(["nm", "-D", "--defined-only", rb.LIB_PATH], capture_output=True, text=True).stdout
    orc = subprocess.run(["nm", "-D", "--defined-only", oracle.build()], capture_output=True, text=True).stdout
    assert "orc_" not in prod
    assert "dbuf_" not in orc


def _plans_equal(r, c, k, m, A, cap=0):
    st, off, s = oracle.plan(r, c, k, m, A, max_bucket=cap)
    try:
        p = rb.dbuf_plan(r, c, k, m, A, cap)
    except rb.DbufError as e:
        assert st != oracle.OK and e.status == rb.DBUF_EINFEASIBLE, (st, e)
        return None
    assert st == oracle.OK
    info = rb.dbuf_plan_info(p)
    assert info["slice"] == s, (r, c, k, m, A)
    assert info["offsets"] == off.tolist(), (r, c, k, m, A)
    assert info["bucket"] == s * m
    assert info["padding"] == s * m - int(np.sum(np.asarray(r) * np.asarray(c)))
    assert info["n_blocks"] == int(sum(-(-int(x) // int(y)) for x, y in zip(r, k)))
    return info


@pytest.mark.parametrize("name", [n for n in synth.WORKLOAD_NAMES])
def test_planner_matches_oracle_on_workloads(name):
    w = synth.workload(name)
    r, c, k = w.arrays()
    _plans_equal(r, c, k, w.m, w.align)


def test_planner_matches_oracle_random():
    rng = random.Random(2024)
    for _ in range(3000):
        n = rng.randint(1, 12)
        rows = [rng.randint(1, 200) for _ in range(n)]
        cols = [rng.choice([1, 2, 3, 7, 16, 48, 64]) for _ in range(n)]
        k = [rng.randint(1, r) for r in rows]
        m = rng.choice([1, 2, 3, 4, 8, 16, 64])
        A = rng.choice([1, 2, 16, 32])
        _plans_equal(rows, cols, k, m, A)


def test_planner_matches_oracle_large_random():
    """Buckets shaped like the stress workload, many m."""
    rng = random.Random(77)
    for _ in range(60):
        n = rng.randint(5, 80)
        rows = [int(np.exp(rng.uniform(np.log(64), np.log(16384)))) for _ in range(n)]
        cols = [rng.choice(synth.workloads.STRESS_COLS) for _ in range(n)]
        k = [min(rng.choice(synth.workloads.STRESS_KS), r) for r in rows]
        _plans_equal(rows, cols, k, rng.choice([8, 64, 128, 1024]), 16)


def test_planner_cap():
    w = synth.workload("tiny_m4")
    r, c, k = w.arrays()
    assert _plans_equal(r, c, k, 4, 16, cap=147456) is not None
    with pytest.raises(rb.DbufError) as e:
        rb.dbuf_plan(r, c, k, 4, 16, 147455)
    assert e.value.status == rb.DBUF_EINFEASIBLE


@pytest.mark.parametrize("rows,cols,k,m,A", [
    ([4], [4], [5], 2, 16),     # k > rows
    ([0], [4], [1], 2, 16),     # rows < 1
    ([4], [-1], [1], 2, 16),    # cols < 1
    ([4], [4], [0], 2, 16),     # k < 1
    ([4], [4], [1], 0, 16),     # m < 1
    ([4], [4], [1], 2, 0),      # align < 1
])
def test_planner_rejects_invalid(rows, cols, k, m, A):
    with pytest.raises(rb.DbufError) as e:
        rb.dbuf_plan(rows, cols, k, m, A)
    assert e.value.status == rb.DBUF_EINVAL
    assert rb.dbuf_last_error()


def test_empty_plan():
    p = rb.dbuf_plan([], [], [], 8, 16)
    info = rb.dbuf_plan_info(p)
    assert info["slice"] == 0 and info["bucket"] == 0 and info["n_blocks"] == 0
    assert rb.dbuf_required_bytes(p) > 0


def test_required_bytes_cover_arrays():
    for name in ("tiny_m4", "ragged_mix_m4", "llama_layer_m8"):
        w = synth.workload(name)
        r, c, k = w.arrays()
        p = rb.dbuf_plan(r, c, k, w.m, 16)
        info = rb.dbuf_plan_info(p)
        need = rb.dbuf_required_bytes(p)
        S, B = info["bucket"], info["n_blocks"]
        assert need >= S * (4 + 2 + 2 + 1 + 1) + B * 8
        assert need % 256 == 0
        assert need < S * 10 + B * 8 + 64 * S // 100 + (1 << 20)


def test_planner_time_budget():
    """The pages report under 0.3 s of planning at init; time ours."""
    import time
    for name in ("moe_layer_m64", "ragged_stress_m8", "ragged_stress_m128", "ragged_stress_m1024"):
        w = synth.workload(name)
        r, c, k = w.arrays()
        t = time.perf_counter()
        rb.dbuf_plan(r, c, k, w.m, 16)
        assert time.perf_counter() - t < 0.3


@pytest.mark.parametrize("name", ["tiny_m4", "ragged_mix_m4", "ragged_mix_m8", "llama_layer_m8",
                                  "moe_layer_m64", "ragged_stress_m8", "ragged_stress_m128"])
def test_work_table_covers_bucket_once(name):
    """Every element of the bucket is in exactly one work item; items respect
    the kernel's limits; block numbers follow bucket order."""
    w = synth.workload(name)
    r, c, k = w.arrays()
    p = rb.dbuf_plan(r, c, k, w.m, 16)
    info = rb.dbuf_plan_info(p)
    S = info["bucket"]
    tab = rb.dbuf_work_table(p)
    start, length = oracle.blocks(r, c, k, info["offsets"])   # bucket-order blocks
    blk_of_start = {int(s): j for j, s in enumerate(start)}
    cover = np.zeros(S + 1, np.int64)
    seen_blocks = np.zeros(start.size, np.int64)
    for t in tab:
        e0, n = t["first_elem"], t["n_elems"]
        assert 0 <= e0 and e0 + n <= S and n > 0
        cover[e0] += 1
        cover[e0 + n] -= 1
        if t["kind"] == 2:
            continue
        j = blk_of_start[e0]                     # starts on a block edge
        assert t["first_block"] == j
        if t["kind"] == 0:
            b = t["block_elems"]
            assert 1 <= b <= 4096 and 1 <= t["n_blocks"] <= 254
            assert (e0 % 16) + n <= 4096
            assert np.all(length[j:j + t["n_blocks"] - 1] == b)
            assert int(length[j:j + t["n_blocks"]].sum()) == n
            seen_blocks[j:j + t["n_blocks"]] += 1
        else:
            assert t["kind"] == 1 and t["n_blocks"] == 1 and n == length[j]
            seen_blocks[j] += 1
    assert np.all(np.cumsum(cover)[:S] == 1)
    assert np.all(seen_blocks == 1)
    # padding items are exactly the padding
    pad = oracle.padding_mask(r, c, info["offsets"], S)
    zmask = np.zeros(S, bool)
    for t in tab:
        if t["kind"] == 2:
            zmask[t["first_elem"]:t["first_elem"] + t["n_elems"]] = True
    assert np.array_equal(zmask, pad)


def test_block_index_reciprocal_is_exact():
    """Whole-block tiles find a vector's block as umulhi(x, ceil(2^32/b)):
    exact for every block size 2..4096 and every offset x < 4096 in a tile."""
    x = np.arange(4096, dtype=np.uint64)
    for b in range(2, 4097):
        magic = np.uint64(((1 << 32) + b - 1) // b)
        assert np.array_equal((x * magic) >> np.uint64(32), x // np.uint64(b)), b


@pytest.mark.parametrize("m", [1, 2, 3, 8, 64, 1000])
def test_rowwise_layout_matches_oracle(m):
    w = synth.workload("ragged_mix_m4")
    r, c, _ = w.arrays()
    chunk, q, off = rb.dbuf_rowwise_layout(r, c, m)
    oq, ooff, oc = oracle.rowwise_layout(r, c, m)
    assert chunk == oc and q == oq.tolist() and off == ooff.tolist()


def test_rowwise_layout_rejects_invalid():
    for rows, cols, m in (([0], [3], 2), ([4], [0], 2), ([4], [3], 0), ([], [], 2)):
        with pytest.raises(rb.DbufError) as e:
            rb.dbuf_rowwise_layout(rows, cols, m)
        assert e.value.status == rb.DBUF_EINVAL


@pytest.mark.parametrize("name", ["tiles_mix_m4", "tiles_mix_m8", "llama_layer_32x32_m8"])
def test_work_table_tiles_cover_once_and_number_like_oracle(name):
    """2-D blocks: STRIP entries cover every element of the tiled tensors once
    (rows x columns with the row stride); the tiles they own are the oracle's
    tiles in the oracle's numbering; other entries still cover the rest."""
    w = synth.workload(name)
    r, c, k = w.arrays()
    bc = w.block_cols()
    p = rb.dbuf_plan(r, c, k, w.m, 16, block_cols=bc)
    info = rb.dbuf_plan_info(p)
    S = info["bucket"]
    base, trows, width, stride = oracle.tiles(r, c, k, bc, info["offsets"])
    assert info["n_blocks"] == base.size
    cover = np.zeros(S, np.int32)
    seen = np.zeros(base.size, np.int32)
    for t in rb.dbuf_work_table(p):
        e0, n = t["first_elem"], t["n_elems"]
        if t["kind"] == 3:
            C, rows, W = t["block_elems"], t["n_blocks"], t["tile_cols"]
            assert n <= 4096 and n % 16 == 0 and C % 16 == 0 and e0 % 16 == 0
            for rr in range(rows):
                cover[e0 + rr * C:e0 + rr * C + n] += 1
            G = -(-n // W)
            assert G <= 256
            for g in range(G):
                j = t["first_block"] + g
                assert base[j] == e0 + g * W and trows[j] == rows and stride[j] == C
                assert width[j] == min(W, n - g * W)
                seen[j] += 1
        else:
            cover[e0:e0 + n] += 1
            if t["kind"] == 0:
                seen[t["first_block"]:t["first_block"] + t["n_blocks"]] += 1
            elif t["kind"] == 1:
                seen[t["first_block"]] += 1
    assert np.all(cover == 1)
    assert np.all(seen == 1)


@pytest.mark.parametrize("bc,cols,ok", [(32, 96, True), (16, 4096, True), (4096, 8192, True), (0, 7, True),
                                        (96, 96, True), (200, 96, True), (24, 96, False), (8, 96, False),
                                        (32, 100, False), (8192, 16384, False)])
def test_plan_block_cols_rules(bc, cols, ok):
    """Tiles need block_cols a power of two in [16, 4096] and cols % 16 == 0;
    block_cols 0 or >= cols means whole rows and is always accepted."""
    if ok:
        p = rb.dbuf_plan([64], [cols], [32], 2, 16, block_cols=[bc])
        tiles = -(-cols // bc) if 0 < bc < cols else 1
        assert rb.dbuf_plan_info(p)["n_blocks"] == 2 * tiles
    else:
        with pytest.raises(rb.DbufError) as e:
            rb.dbuf_plan([64], [cols], [32], 2, 16, block_cols=[bc])
        assert e.value.status == rb.DBUF_EINVAL


@pytest.mark.parametrize("name", ["tiny_m4", "llama_layer_m8", "moe_layer_m64", "ragged_stress_m8",
                                  "ragged_stress_m128", "ragged_stress_m1024", "ragged_mix_m4", "ragged_mix_m8",
                                  "tiles_mix_m4", "tiles_mix_m8", "llama_layer_32x32_m8"])
def test_every_work_entry_lies_in_one_slice(name):
    """RaggedShard's point: blocks never straddle a rank's slice, so each
    rank can step its own slice with no exchange.  The work table keeps
    that: every entry (padding entries too) lies inside one slice, so the
    entries of slice r are exactly rank r's work."""
    w = synth.workload(name)
    r, c, k = w.arrays()
    p = rb.dbuf_plan(r, c, k, w.m, 16, block_cols=w.block_cols())
    s = rb.dbuf_plan_info(p)["slice"]
    for t in rb.dbuf_work_table(p):
        lo = t["first_elem"]
        hi = lo + ((t["n_blocks"] - 1) * t["block_elems"] + t["n_elems"] if t["kind"] == 3 else t["n_elems"])
        assert lo // s == (hi - 1) // s, t


@pytest.mark.parametrize("name", ["tiny_m4", "llama_layer_m8", "moe_layer_m64", "ragged_stress_m128",
                                  "ragged_stress_m1024", "ragged_mix_m4", "ragged_mix_m8", "tiles_mix_m8"])
def test_plan_shards_match_oracle_and_keep_blocks_whole(name):
    """dbuf_plan_shards equals the oracle's placement; every tensor's rows
    are covered once, in rank order, and each boundary between two ranks
    is a k-row block edge (RaggedShard: a block is never split)."""
    w = synth.workload(name)
    r, c, k = w.arrays()
    p = rb.dbuf_plan(r, c, k, w.m, 16, block_cols=w.block_cols())
    info = rb.dbuf_plan_info(p)
    got = rb.dbuf_plan_shards(p, w.m)
    assert got == oracle.shards(r, c, info["offsets"], info["slice"], w.m)
    for i, per in enumerate(got):
        assert per[0][0] == 0 and per[-1][1] == r[i]
        for (b0, e0), (b1, e1) in zip(per, per[1:]):
            assert b0 <= e0 == b1 <= e1
        for b, e in per:
            if e > b:
                assert b % k[i] == 0 and (e % k[i] == 0 or e == r[i])


def test_oracle_shards_against_per_element_slices():
    """Brute force on the ragged mix: assign every bucket element its slice
    and count each tensor's elements per slice."""
    w = synth.workload("ragged_mix_m4")
    r, c, k = w.arrays()
    st, off, s = oracle.plan(r, c, k, w.m, 16)
    sh = oracle.shards(r, c, off, s, w.m)
    for i in range(len(r)):
        e = int(off[i]) + np.arange(int(r[i] * c[i]))
        counts = np.bincount(e // s, minlength=w.m)
        assert [(hi - lo) * int(c[i]) for lo, hi in sh[i]] == counts.tolist()


def test_allocation_hook_failures_are_reported_before_device_work():
    """DBuffer's allocation hook (the caller's memory pool): a hook that
    fails, or returns no memory or the wrong kind of memory, is reported as a
    DbufError before any device call, so this runs without a GPU."""
    p = rb.dbuf_plan([64, 8], [64, 16], [4, 8], 2, 16)
    need = max(rb.dbuf_required_bytes(p), 256)
    asked = []

    def none(n):
        asked.append(n)
        return None

    def raises(n):
        raise MemoryError("pool exhausted")

    for hook, status in ((none, rb.DBUF_ENOMEM), (raises, rb.DBUF_ENOMEM),
                         (lambda n: torch.empty(n, dtype=torch.float32), rb.DBUF_EINVAL),
                         (lambda n: torch.empty((n, 2), dtype=torch.uint8), rb.DBUF_EINVAL)):
        with pytest.raises(rb.DbufError) as e:
            rb.DBuffer(p, alloc=hook)
        assert e.value.status == status
    assert asked == [need]
