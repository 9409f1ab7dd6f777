"""Rank buckets: one slice of a bucket as a bucket of its own (CPU).

RaggedShard (paper Sec. 3; page section "1. RaggedShard") keeps every block
whole inside one device's slice, so each device can step its slice with no
exchange.  These tests pin that:
  * the oracle's per-rank buckets, each stepped alone, give the whole
    bucket's result bit for bit (master, bf16 copy, codes, scales);
  * the library's dbuf_plan_rank gives the oracle's rank buckets (parts,
    offsets, padding, block counts, first block);
  * the library's work table of a rank bucket is the whole bucket's work
    table restricted to that slice, rebased, in the same order.
"""
import numpy as np
import pytest

import oracle
import ragged_bucket_layout_b200 as rb
import synth
from synth.rng import STREAM_GRAD, STREAM_PARAM
from synth.workloads import GRAD_SIGMA, PARAM_SIGMA

# Small layouts with the edge cases: a rank with no tensor at all (slices 1-3
# of the first), a part shorter than k rows (a tensor's short last block on
# its own), 2-D blocks cut by a slice boundary.
EDGE_CASES = {
    "empty_slices_m4": ([1000, 48], [1, 16], [1000, 48], None, 4),
    "short_tail_m3": ([100, 7], [32, 16], [16, 3], None, 3),
    "tiles_cut_m4": ([96, 40, 5], [64, 32, 16], [8, 4, 5], [16, 16, 0], 4),
}


def _edge(name):
    rows, cols, k, bc, m = EDGE_CASES[name]
    z = [0] * len(rows)
    return (np.array(rows, np.int64), np.array(cols, np.int64), np.array(k, np.int64),
            np.array(bc if bc is not None else z, np.int64), m, 16)


def _case(name):
    if name in EDGE_CASES:
        return _edge(name)
    w = synth.workload(name)
    r, c, k = w.arrays()
    return r, c, k, np.asarray(w.block_cols(), np.int64), w.m, w.align


def _plans(name):
    r, c, k, bc, m, align = _case(name)
    P = rb.dbuf_plan(r, c, k, m, align, block_cols=bc)
    st, off, s = oracle.plan(r, c, k, m, align)
    assert st == 0 and off.tolist() == rb.dbuf_plan_info(P)["offsets"]
    return r, c, k, bc, m, align, P, off, s


def _block_count(rk):
    G = [1 if b <= 0 or b >= c else -(-c // b) for c, b in zip(rk["cols"], rk["block_cols"])]
    return int(sum(g * -(-int(rr) // int(kk)) for g, rr, kk in zip(G, rk["rows"], rk["k"])))


SMALL = ["tiny_m4", "ragged_mix_m8", "tiles_mix_m4", "empty_slices_m4", "short_tail_m3", "tiles_cut_m4"]


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


def test_edge_cases_are_present():
    """The small layouts above really contain the edge cases they stand for."""
    r, c, k, bc, m, align, P, off, s = _plans("empty_slices_m4")
    assert [rb.dbuf_plan_rank(P, q).n for q in range(m)].count(0) >= 2
    r, c, k, bc, m, align, P, off, s = _plans("short_tail_m3")
    parts = [x for q in range(m) for x in rb.dbuf_plan_rank(P, q).parts]
    assert any(a > 0 and b - a < k[i] for i, a, b in parts)
    r, c, k, bc, m, align, P, off, s = _plans("tiles_cut_m4")
    assert any(a > 0 and bc[i] > 0 for q in range(m) for i, a, b in rb.dbuf_plan_rank(P, q).parts)


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
def test_oracle_rank_buckets_step_like_the_whole_bucket(name):
    r, c, k, bc, m, align, P, off, s = _plans(name)
    W = oracle.Bucket(r, c, k, off, s, m, block_cols=bc)
    _fill_params(W, r, c, off, 91)
    ranks = [oracle.rank_bucket(r, c, k, off, s, m, q, bc) for q in range(m)]
    B = [oracle.Bucket(x["rows"], x["cols"], x["k"], x["offsets"], s, 1, block_cols=x["block_cols"]) for x in ranks]
    for q in range(m):
        B[q].p[:] = W.p[q * s:(q + 1) * s]
    hp0 = dict(synth.HPARAMS)
    for t in (1, 2, 3):
        W.g[:] = _grads(r, c, off, W.size, 91, t)
        W.step(dict(hp0, step=t), t, 1.0 / m)
        for q in range(m):
            B[q].g[:] = W.g[q * s:(q + 1) * s]
            B[q].step(dict(hp0, step=t), t, 1.0 / m)
    for q in range(m):
        sl = slice(q * s, (q + 1) * s)
        assert np.array_equal(B[q].p.view(np.uint32), W.p[sl].view(np.uint32))
        assert np.array_equal(B[q].pb, W.pb[sl])
        assert np.array_equal(B[q].mq, W.mq[sl]) and np.array_equal(B[q].vq, W.vq[sl])
        fb, nb = ranks[q]["first_block"], B[q].scale_m.size
        assert np.array_equal(B[q].scale_m.view(np.uint32), W.scale_m[fb:fb + nb].view(np.uint32))
        assert np.array_equal(B[q].scale_v.view(np.uint32), W.scale_v[fb:fb + nb].view(np.uint32))
    assert sum(b.scale_m.size for b in B) == W.scale_m.size


def test_oracle_rank_bucket_catches_a_cut_block():
    """A layout whose slice boundary falls inside a block is not a RaggedShard
    layout: the oracle's rank bucket refuses it."""
    with pytest.raises(AssertionError):
        # one tensor of 8 rows x 16 in blocks of 4 rows, slices of 48 elements
        # (3 rows): the boundary cuts the first block.
        oracle.rank_bucket([8], [16], [4], [0], 48, 3, 1)


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
