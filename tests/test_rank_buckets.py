"""Rank buckets from the library (dbuf_plan_rank) against the oracle (CPU).

A slice of a RaggedShard bucket is a bucket of its own (paper Sec. 3; page
section "1. RaggedShard": blocks never straddle a slice).  The oracle's
rank buckets are pinned against the whole bucket in
test_oracle_rank_buckets.py; here the library's must equal them:
  * parts, offsets, padding, block counts and first block;
  * the work table of a rank bucket is the whole bucket's work table
    restricted to that slice, rebased, in the same order (so the step
    kernel runs the same entries on the same data).
"""
import numpy as np
import pytest

import oracle
import ragged_bucket_layout_b200 as rb

from test_oracle_rank_buckets import SMALL, _case


def _plans(name):
    r, c, k, bc, m, align = _case(name)
    P = rb.dbuf_plan(r, c, k, m, align, block_cols=bc)
    st, off, s = oracle.plan(r, c, k, m, align)
    assert st == 0 and off.tolist() == rb.dbuf_plan_info(P)["offsets"]
    return r, c, k, bc, m, align, P, off, s


def _block_count(rk):
    G = [1 if b <= 0 or b >= c else -(-c // b) for c, b in zip(rk["cols"], rk["block_cols"])]
    return int(sum(g * -(-int(rr) // int(kk)) for g, rr, kk in zip(G, rk["rows"], rk["k"])))


@pytest.mark.parametrize("name", SMALL + ["llama_layer_m8", "llama_layer_32x32_m8", "ragged_stress_m8",
                                          "moe_layer_m64"])
def test_rank_plans_match_the_oracle(name):
    r, c, k, bc, m, align, P, off, s = _plans(name)
    parent = rb.dbuf_plan_info(P)
    small = name in SMALL
    covered = np.zeros(len(r), np.int64)
    blocks_before = 0
    for q in range(m):
        R = rb.dbuf_plan_rank(P, q)
        want = oracle.rank_bucket(r, c, k, off, s, m, q, bc)
        info = rb.dbuf_plan_info(R)
        assert R.parts == want["parts"]
        assert R.n == len(want["parts"])
        assert info["slice"] == info["bucket"] == s
        assert info["offsets"] == want["offsets"].tolist()
        assert R.first_block == want["first_block"] == blocks_before
        if small:
            pad = int(oracle.padding_mask(want["rows"], want["cols"], want["offsets"], s).sum())
            nb = int(oracle.tiles(want["rows"], want["cols"], want["k"], want["block_cols"], want["offsets"])[0].size)
        else:
            pad = s - int(np.sum(want["rows"] * want["cols"]))
            nb = _block_count(want)
        assert info["padding"] == pad
        assert info["n_blocks"] == nb
        assert R.shapes == [(b - a, int(c[i])) for i, a, b in R.parts]
        blocks_before += nb
        for i, a, b in R.parts:
            assert covered[i] == a, "the parts of a tensor follow one another rank by rank"
            covered[i] = b
    assert covered.tolist() == r.tolist()
    assert blocks_before == parent["n_blocks"]


@pytest.mark.parametrize("name", ["tiny_m4", "ragged_mix_m8", "tiles_mix_m8", "llama_layer_m8",
                                  "llama_layer_32x32_m8", "empty_slices_m4", "short_tail_m3", "tiles_cut_m4"])
def test_rank_work_table_is_the_parents_slice(name):
    r, c, k, bc, m, align, P, off, s = _plans(name)
    parent = rb.dbuf_work_table(P)
    total = 0
    for q in range(m):
        R = rb.dbuf_plan_rank(P, q)
        lo, hi = q * s, (q + 1) * s
        want = []
        for e in parent:
            if lo <= e["first_elem"] < hi:
                assert e["first_elem"] + e["n_elems"] <= hi
                x = dict(e, first_elem=e["first_elem"] - lo)
                if e["kind"] != 2:                       # padding entries carry no block index
                    x["first_block"] = e["first_block"] - R.first_block
                want.append(x)
        assert rb.dbuf_work_table(R) == want
        total += len(want)
    assert total == len(parent)


def test_plan_rank_errors_and_identity():
    r, c, k, bc, m, align, P, off, s = _plans("tiny_m4")
    for bad in (-1, m):
        with pytest.raises(rb.DbufError) as e:
            rb.dbuf_plan_rank(P, bad)
        assert e.value.status == rb.DBUF_EINVAL
    # A plan of one slice is its own rank bucket.
    P1 = rb.dbuf_plan(r, c, k, 1, align)
    R = rb.dbuf_plan_rank(P1, 0)
    a, b = rb.dbuf_plan_info(P1), rb.dbuf_plan_info(R)
    assert a == b and R.first_block == 0 and R.parts == [(i, 0, int(x)) for i, x in enumerate(r)]
    assert rb.dbuf_work_table(R) == rb.dbuf_work_table(P1)


@pytest.mark.parametrize("name", ["tiny_m4", "tiles_cut_m4", "empty_slices_m4", "moe_layer_m64"])
def test_rank_parts_agree_with_the_shard_table(name):
    """The binding's per-rank part list (from offsets and shapes) equals the
    rows dbuf_plan_shards gives for that rank; the library's rank plan holds
    as many tensors and puts each at its parent offset minus q*s."""
    r, c, k, bc, m, align, P, off, s = _plans(name)
    table = rb.dbuf_plan_shards(P, m)
    for q in range(m):
        R = rb.dbuf_plan_rank(P, q)
        assert R.parts == [(i, a, b) for i, per in enumerate(table) for a, b in [per[q]] if b > a]
        assert rb.dbuf_plan_dims(R) == (len(R.parts), 1)
        want = [int(off[i]) + a * int(c[i]) - q * s for i, a, b in R.parts]
        assert rb.dbuf_plan_info(R)["offsets"] == want


def test_golden_rank_buckets_of_the_tiny_layout(golden_dir):
    """The library's rank plans of the tiny layout against the hand-worked
    values in tests/golden/rank_buckets_tiny.json."""
    import json
    import os
    g = json.load(open(os.path.join(golden_dir, "rank_buckets_tiny.json")))
    P = rb.dbuf_plan(g["rows"], g["cols"], g["k"], g["m"], 16)
    assert rb.dbuf_plan_info(P)["offsets"] == g["offsets"] and rb.dbuf_plan_info(P)["slice"] == g["s"]
    for q, want in enumerate(g["ranks"]):
        R = rb.dbuf_plan_rank(P, q)
        info = rb.dbuf_plan_info(R)
        assert [list(p) for p in R.parts] == want["parts"]
        assert info["offsets"] == want["offsets"] and info["padding"] == want["padding"]
        assert info["n_blocks"] == want["n_blocks"] and R.first_block == want["first_block"]


def _random_bucket(rng):
    n = int(rng.integers(1, 8))
    rows, cols, k, bc = [], [], [], []
    for _ in range(n):
        tiled = rng.random() < 0.3
        C = int(rng.choice([16, 32, 48, 64])) if tiled else int(rng.integers(1, 70))
        R = int(rng.integers(1, 90))
        rows.append(R)
        cols.append(C)
        k.append(int(rng.integers(1, R + 1)))
        bc.append(int(rng.choice([16, 32])) if tiled and C > 16 else 0)
    return rows, cols, k, bc, int(rng.integers(1, 9))


def test_random_buckets_rank_plans_and_work_tables():
    """300 seeded random buckets (1-7 tensors, ragged rows and blocks, some
    2-D blocks, m up to 8): for every rank the library's rank plan equals
    the oracle's rank bucket and its work table is the parent's slice."""
    rng = np.random.default_rng(2024)
    for _ in range(300):
        rows, cols, k, bc, m = _random_bucket(rng)
        P = rb.dbuf_plan(rows, cols, k, m, 16, block_cols=bc)
        info = rb.dbuf_plan_info(P)
        s, off = info["slice"], info["offsets"]
        parent = rb.dbuf_work_table(P)
        for q in range(m):
            R = rb.dbuf_plan_rank(P, q)
            want = oracle.rank_bucket(rows, cols, k, off, s, m, q, bc)
            ri = rb.dbuf_plan_info(R)
            assert R.parts == want["parts"] and ri["offsets"] == want["offsets"].tolist()
            assert R.first_block == want["first_block"]
            exp = []
            for e in parent:
                if q * s <= e["first_elem"] < (q + 1) * s:
                    x = dict(e, first_elem=e["first_elem"] - q * s)
                    if e["kind"] != 2:
                        x["first_block"] = e["first_block"] - R.first_block
                    exp.append(x)
            assert rb.dbuf_work_table(R) == exp, (rows, cols, k, bc, m, q)
