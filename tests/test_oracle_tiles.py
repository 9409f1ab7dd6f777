"""Pins of the oracle's 2-D block (tile) step, the 32x32-element blocks the
8-bit Adam case study allows per parameter (CPU only).

- a first step worked by hand (tests/golden/tiles2d_first_step.json);
- tiles as wide as the tensor are exactly the row blocks, and stepping them
  equals the pinned contiguous-block step bit for bit;
- every tile equals the contiguous-block step applied to that tile cut out
  of the tensor with numpy slicing;
- every nonzero tile has an m code at +-127 and a v code at 255.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from synth.rng import STREAM_GRAD, STREAM_PARAM

HERE = os.path.dirname(os.path.abspath(__file__))
HP = dict(synth.HPARAMS)


def _plan(r, c, k, m):
    st, off, s = oracle.plan(r, c, k, m, 16)
    assert st == oracle.OK
    return off, s


def test_golden_tiles_first_step():
    G = json.load(open(os.path.join(HERE, "golden", "tiles2d_first_step.json")))
    r, c, k = [G["rows"]], [G["cols"]], [G["k"]]
    off, s = _plan(r, c, k, G["m"])
    B = oracle.Bucket(r, c, k, off, s, G["m"], block_cols=[G["block_cols"]])
    o = int(off[0])
    n = G["rows"] * G["cols"]
    B.g[o:o + n] = oracle.bf16_round(np.asarray(G["g"], np.float32).reshape(-1))
    B.step(HP, 1, 1.0)
    assert B.mq[o:o + n].reshape(G["rows"], G["cols"]).tolist() == G["mq"]
    assert B.vq[o:o + n].reshape(G["rows"], G["cols"]).tolist() == G["vq"]
    sc = oracle.step_scalars(HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], 1)
    omb1, omb2 = sc[1], sc[3]
    sq = np.sqrt(np.float32(omb2), dtype=np.float32)
    for j, e in enumerate(G["tile_max_log2"]):
        assert B.scale_m[j] == np.float32(omb1) * np.float32(2.0 ** e)
        assert B.scale_v[j] == sq * np.float32(2.0 ** e)


def _fill(B, seed):
    for i in range(len(B.rows)):
        sl = B.tensor_slice(i)
        n = sl.stop - sl.start
        B.p[sl] = synth.normal_f32(synth.stream_key(seed, STREAM_PARAM), sl.start, n, 0.02)
        B.g[sl] = synth.normal_bf16(synth.stream_key(seed, STREAM_GRAD), sl.start, n, 1e-3)


def test_full_width_tiles_are_row_blocks():
    w = synth.workload("ragged_mix_m4")
    r, c, k = w.arrays()
    off, s = _plan(r, c, k, w.m)
    base, trows, width, stride = oracle.tiles(r, c, k, c, off)      # block_cols = cols
    start, length = oracle.blocks(r, c, k, off)
    assert np.array_equal(base, start) and np.array_equal(trows * width, length)
    A = oracle.Bucket(r, c, k, off, s, w.m)
    Bt = oracle.Bucket(r, c, k, off, s, w.m)
    Bt.tiles, Bt.tiled = (base, trows, width, stride), True
    for B in (A, Bt):
        _fill(B, 5)
    for t in (1, 2, 3):
        A.step(HP, t, 0.25)
        Bt.step(HP, t, 0.25)
        for f in ("p", "pb", "mq", "vq", "scale_m", "scale_v"):
            assert np.array_equal(getattr(A, f), getattr(Bt, f)), (t, f)


def _tiled_shapes():
    rows = np.array([70, 33, 5, 64, 1], np.int64)
    cols = np.array([96, 40, 7, 1024, 300], np.int64)
    k = np.array([32, 32, 2, 32, 1], np.int64)
    bc = np.array([32, 16, 3, 32, 0], np.int64)
    return rows, cols, k, bc


@pytest.mark.parametrize("m", [1, 4])
def test_each_tile_is_a_block_of_the_cut_out_tile(m):
    r, c, k, bc = _tiled_shapes()
    off, s = _plan(r, c, k, m)
    B = oracle.Bucket(r, c, k, off, s, m, block_cols=bc)
    _fill(B, 9)
    B.step(HP, 1, 1.0)
    p0 = B.p.copy()
    B.step(HP, 2, 1.0)
    # replay step 2 tile by tile from the state after step 1, cutting tiles out with numpy
    A = oracle.Bucket(r, c, k, off, s, m, block_cols=bc)
    _fill(A, 9)
    A.step(HP, 1, 1.0)
    assert np.array_equal(A.p, p0)
    j = 0
    for i in np.argsort(off, kind="stable"):
        R, C, K = int(r[i]), int(c[i]), int(k[i])
        W = C if bc[i] <= 0 or bc[i] >= C else int(bc[i])
        idx = (int(off[i]) + np.arange(R * C, dtype=np.int64)).reshape(R, C)
        for r0 in range(0, R, K):
            for c0 in range(0, C, W):
                at = idx[r0:r0 + K, c0:c0 + W].reshape(-1)
                p, g, mq, vq, pb = (np.ascontiguousarray(x[at]) for x in (A.p, A.g, A.mq, A.vq, A.pb))
                sm, sv = A.scale_m[j:j + 1].copy(), A.scale_v[j:j + 1].copy()
                oracle.adam8_step([0], [at.size], [0], p, g, mq, vq, sm, sv, pb, HP, 2, 1.0)
                assert np.array_equal(p, B.p[at]) and np.array_equal(mq, B.mq[at]) and np.array_equal(vq, B.vq[at])
                assert sm[0] == B.scale_m[j] and sv[0] == B.scale_v[j]
                j += 1
    assert j == B.scale_m.size


def test_every_nonzero_tile_reaches_full_scale():
    r, c, k, bc = _tiled_shapes()
    off, s = _plan(r, c, k, 4)
    B = oracle.Bucket(r, c, k, off, s, 4, block_cols=bc)
    _fill(B, 3)
    B.step(HP, 1, 1.0)
    base, trows, width, stride = B.tiles
    for j in range(base.size):
        at = (base[j] + np.arange(trows[j])[:, None] * stride[j] + np.arange(width[j])[None, :]).reshape(-1)
        assert np.abs(B.mq[at].astype(np.int32)).max() == 127
        assert B.vq[at].max() == 255
