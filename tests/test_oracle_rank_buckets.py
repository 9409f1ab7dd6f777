"""Pins of the oracle's rank buckets (oracle.rank_bucket), CPU only.

RaggedShard (paper Sec. 3; page section "1. RaggedShard"): every block lies
whole inside one device's slice, so a slice is a bucket of its own.  The
oracle's rank bucket is checked against the whole bucket, not against
itself:
  * every rank bucket stepped alone gives the whole bucket's step, bit for
    bit (master, bf16 copy, codes, scales);
  * its first block is the number of whole-bucket blocks that start before
    the slice (oracle.tiles numbering);
  * the parts of every tensor follow one another rank by rank and cover it;
  * they are the RaggedShard rows of oracle.shards, and their padding laid
    side by side is the whole bucket's;
  * on the tiny layout they equal the hand-worked values in
    tests/golden/rank_buckets_tiny.json.
"""
import numpy as np
import pytest

import oracle
import synth
from synth.rng import STREAM_GRAD, STREAM_PARAM
from synth.workloads import GRAD_SIGMA, PARAM_SIGMA

# Small layouts with the edge cases: ranks with no tensor at all, a part
# shorter than k rows (a tensor's short last block alone on a rank), 2-D
# blocks cut by a slice boundary.
EDGE_CASES = {
    "empty_slices_m4": ([1000, 48], [1, 16], [1000, 48], None, 4),
    "short_tail_m3": ([100, 7], [32, 16], [16, 3], None, 3),
    "tiles_cut_m4": ([96, 40, 5], [64, 32, 16], [8, 4, 5], [16, 16, 0], 4),
}
SMALL = ["tiny_m4", "ragged_mix_m8", "tiles_mix_m4", "empty_slices_m4", "short_tail_m3", "tiles_cut_m4"]


def _case(name):
    """(rows, cols, k, block_cols, m, align) of a workload or an edge case."""
    if name in EDGE_CASES:
        rows, cols, k, bc, m = EDGE_CASES[name]
        bc = bc if bc is not None else [0] * len(rows)
        a = lambda x: np.array(x, np.int64)
        return a(rows), a(cols), a(k), a(bc), m, 16
    w = synth.workload(name)
    r, c, k = w.arrays()
    return r, c, k, np.asarray(w.block_cols(), np.int64), w.m, w.align


def _layout(name):
    r, c, k, bc, m, align = _case(name)
    st, off, s = oracle.plan(r, c, k, m, align)
    assert st == oracle.OK
    return r, c, k, bc, m, off, s


def _fill_params(B, rows, cols, offsets, seed):
    kp = synth.stream_key(seed, STREAM_PARAM)
    at = 0
    for R, C, o in zip(rows, cols, offsets):
        n = int(R * C)
        B.p[int(o):int(o) + n] = synth.normal_f32(kp, at, n, PARAM_SIGMA)
        at += n


def _grads(rows, cols, offsets, size, seed, t):
    g = np.zeros(size, np.uint16)
    kg = synth.stream_key(seed, STREAM_GRAD * 1000 + t)
    at = 0
    for R, C, o in zip(rows, cols, offsets):
        n = int(R * C)
        g[int(o):int(o) + n] = synth.normal_bf16(kg, at, n, GRAD_SIGMA)
        at += n
    return g


@pytest.mark.parametrize("name", SMALL + ["tiles_mix_m8"])
def test_rank_buckets_step_like_the_whole_bucket(name):
    r, c, k, bc, m, off, s = _layout(name)
    W = oracle.Bucket(r, c, k, off, s, m, block_cols=bc)
    _fill_params(W, r, c, off, 91)
    ranks = [oracle.rank_bucket(r, c, k, off, s, m, q, bc) for q in range(m)]
    B = [oracle.Bucket(x["rows"], x["cols"], x["k"], x["offsets"], s, 1, block_cols=x["block_cols"]) for x in ranks]
    for q in range(m):
        B[q].p[:] = W.p[q * s:(q + 1) * s]
    for t in (1, 2, 3):
        hp = dict(synth.HPARAMS, step=t)
        W.g[:] = _grads(r, c, off, W.size, 91, t)
        W.step(hp, t, 1.0 / m)
        for q in range(m):
            B[q].g[:] = W.g[q * s:(q + 1) * s]
            B[q].step(hp, t, 1.0 / m)
    for q in range(m):
        sl = slice(q * s, (q + 1) * s)
        assert np.array_equal(B[q].p.view(np.uint32), W.p[sl].view(np.uint32))
        assert np.array_equal(B[q].pb, W.pb[sl])
        assert np.array_equal(B[q].mq, W.mq[sl]) and np.array_equal(B[q].vq, W.vq[sl])
        fb, nb = ranks[q]["first_block"], B[q].scale_m.size
        assert np.array_equal(B[q].scale_m.view(np.uint32), W.scale_m[fb:fb + nb].view(np.uint32))
        assert np.array_equal(B[q].scale_v.view(np.uint32), W.scale_v[fb:fb + nb].view(np.uint32))
    assert sum(b.scale_m.size for b in B) == W.scale_m.size


@pytest.mark.parametrize("name", SMALL)
def test_first_block_counts_the_blocks_before_the_slice(name):
    r, c, k, bc, m, off, s = _layout(name)
    base = oracle.tiles(r, c, k, bc, off)[0]          # whole-bucket blocks in bucket order
    for q in range(m):
        rk = oracle.rank_bucket(r, c, k, off, s, m, q, bc)
        assert rk["first_block"] == int(np.sum(base < q * s))
        inside = base[(base >= q * s) & (base < (q + 1) * s)] - q * s
        mine = oracle.tiles(rk["rows"], rk["cols"], rk["k"], rk["block_cols"], rk["offsets"])[0]
        assert np.array_equal(mine, inside)


@pytest.mark.parametrize("name", SMALL)
def test_parts_tile_every_tensor(name):
    r, c, k, bc, m, off, s = _layout(name)
    end = np.zeros(len(r), np.int64)
    for q in range(m):
        rk = oracle.rank_bucket(r, c, k, off, s, m, q, bc)
        for (i, a, b), o in zip(rk["parts"], rk["offsets"]):
            assert a == end[i] and b > a
            assert int(off[i]) + a * int(c[i]) == q * s + int(o)     # same elements, rebased
            end[i] = b
    assert end.tolist() == r.tolist()


def test_edge_cases_are_present():
    """The small layouts above really contain the edge cases they stand for."""
    r, c, k, bc, m, off, s = _layout("empty_slices_m4")
    assert [len(oracle.rank_bucket(r, c, k, off, s, m, q, bc)["parts"]) for q in range(m)].count(0) >= 2
    r, c, k, bc, m, off, s = _layout("short_tail_m3")
    parts = [x for q in range(m) for x in oracle.rank_bucket(r, c, k, off, s, m, q, bc)["parts"]]
    assert any(a > 0 and b - a < k[i] for i, a, b in parts)
    r, c, k, bc, m, off, s = _layout("tiles_cut_m4")
    parts = [x for q in range(m) for x in oracle.rank_bucket(r, c, k, off, s, m, q, bc)["parts"]]
    assert any(a > 0 and bc[i] > 0 for i, a, b in parts)


def test_a_cut_block_is_refused():
    """A layout whose slice boundary falls inside a block is not a RaggedShard
    layout: one tensor of 8 rows x 16 in blocks of 4 rows with slices of 48
    elements (3 rows) has its first block cut."""
    with pytest.raises(AssertionError):
        oracle.rank_bucket([8], [16], [4], [0], 48, 3, 1)


@pytest.mark.parametrize("name", SMALL)
def test_rank_buckets_agree_with_the_shard_rows_and_the_padding(name):
    """Two other oracle functions, written separately, say the same: the
    RaggedShard rows of each rank (oracle.shards) are the rank buckets'
    parts, and the rank buckets' padding laid side by side is the whole
    bucket's padding."""
    r, c, k, bc, m, off, s = _layout(name)
    rows_of = oracle.shards(r, c, off, s, m)
    pad = []
    for q in range(m):
        rk = oracle.rank_bucket(r, c, k, off, s, m, q, bc)
        want = [(i, a, b) for i, per in enumerate(rows_of) for a, b in [per[q]] if b > a]
        assert rk["parts"] == want
        pad.append(oracle.padding_mask(rk["rows"], rk["cols"], rk["offsets"], s))
    assert np.array_equal(np.concatenate(pad), oracle.padding_mask(r, c, off, m * s))


def test_golden_rank_buckets_of_the_tiny_layout(golden_dir):
    """The rank buckets of the tiny layout, worked by hand
    (tests/golden/rank_buckets_tiny.json)."""
    import json
    import os
    g = json.load(open(os.path.join(golden_dir, "rank_buckets_tiny.json")))
    for q, want in enumerate(g["ranks"]):
        rk = oracle.rank_bucket(g["rows"], g["cols"], g["k"], g["offsets"], g["s"], g["m"], q)
        assert [list(p) for p in rk["parts"]] == want["parts"]
        assert rk["offsets"].tolist() == want["offsets"]
        assert rk["first_block"] == want["first_block"]
        assert int(oracle.padding_mask(rk["rows"], rk["cols"], rk["offsets"], g["s"]).sum()) == want["padding"]
        assert oracle.blocks(rk["rows"], rk["cols"], rk["k"], rk["offsets"])[0].size == want["n_blocks"]


def test_random_buckets_step_like_the_whole_bucket():
    """60 seeded random buckets (ragged rows and blocks, some 2-D blocks, m up
    to 6), two steps: every rank bucket stepped alone equals its slice of
    the whole bucket."""
    rng = np.random.default_rng(77)
    for case in range(60):
        n = int(rng.integers(1, 6))
        r, c, k, bc = [], [], [], []
        for _ in range(n):
            tiled = rng.random() < 0.3
            C = int(rng.choice([16, 32, 48])) if tiled else int(rng.integers(1, 50))
            R = int(rng.integers(1, 60))
            r.append(R)
            c.append(C)
            k.append(int(rng.integers(1, R + 1)))
            bc.append(16 if tiled and C > 16 else 0)
        m = int(rng.integers(1, 7))
        st, off, s = oracle.plan(r, c, k, m, 16)
        assert st == oracle.OK
        W = oracle.Bucket(r, c, k, off, s, m, block_cols=bc)
        _fill_params(W, r, c, off, case)
        ranks = [oracle.rank_bucket(r, c, k, off, s, m, q, bc) for q in range(m)]
        B = [oracle.Bucket(x["rows"], x["cols"], x["k"], x["offsets"], s, 1, block_cols=x["block_cols"])
             for x in ranks]
        for q in range(m):
            B[q].p[:] = W.p[q * s:(q + 1) * s]
        for t in (1, 2):
            hp = dict(synth.HPARAMS, step=t)
            W.g[:] = _grads(r, c, off, W.size, case, t)
            W.step(hp, t, 1.0 / m)
            for q in range(m):
                B[q].g[:] = W.g[q * s:(q + 1) * s]
                B[q].step(hp, t, 1.0 / m)
        for q in range(m):
            sl = slice(q * s, (q + 1) * s)
            assert np.array_equal(B[q].p.view(np.uint32), W.p[sl].view(np.uint32)), (case, q)
            assert np.array_equal(B[q].pb, W.pb[sl]) and np.array_equal(B[q].mq, W.mq[sl]), (case, q)
            fb = ranks[q]["first_block"]
            assert np.array_equal(B[q].scale_v, W.scale_v[fb:fb + B[q].scale_v.size]), (case, q)
