"""Pins of the oracle's row-wise (FSDP2-style) sharded layout and its
interleaved copy-in / copy-out, the baseline the RaggedShard bucket removes
(CPU only).

- a layout worked by hand (tests/golden/rowwise_tiny.json);
- every shard equals torch.chunk(tensor, m, dim=0)[r] (the primitive FSDP2
  shards with), zero-padded to ceil(rows/m) rows;
- copy-out inverts copy-in at scale 1, and copy-in scales like the copy-in
  of the bucket (bf16(float(g) * scale)).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from synth.rng import STREAM_GRAD, STREAM_SHAPES

HERE = os.path.dirname(os.path.abspath(__file__))


def _bits(vals):
    return oracle.bf16_round(np.asarray(vals, dtype=np.float32))


def _golden():
    return json.load(open(os.path.join(HERE, "golden", "rowwise_tiny.json")))


def test_golden_rowwise_layout():
    G = _golden()
    rows = [t["rows"] for t in G["tensors"]]
    cols = [t["cols"] for t in G["tensors"]]
    q, off, C = oracle.rowwise_layout(rows, cols, G["m"])
    assert list(q) == G["q"] and list(off) == G["offsets"] and C == G["chunk"]
    grads = [_bits(G["values"][t["name"]]) for t in G["tensors"]]
    buf = oracle.rowwise_copy_in(grads, rows, cols, G["m"], 1.0)
    assert np.array_equal(buf, _bits(G["gathered"]))
    half = oracle.rowwise_copy_in(grads, rows, cols, G["m"], 0.5)
    assert np.array_equal(half, _bits(np.asarray(G["gathered"], dtype=np.float32) * 0.5))
    outs = oracle.rowwise_copy_out(_bits(G["gathered"]), rows, cols, G["m"])
    for o, g in zip(outs, grads):
        assert np.array_equal(o, g)


def _random_shapes(seed, n):
    u = synth.uniform_f64(synth.stream_key(seed, STREAM_SHAPES), 0, 2 * n).reshape(n, 2)
    rows = (1 + (u[:, 0] * 40)).astype(np.int64)
    cols = np.array([(1, 3, 8, 16, 33)[int(x * 5)] for x in u[:, 1]], dtype=np.int64)
    return rows, cols


@pytest.mark.parametrize("m", [1, 2, 3, 4, 7, 8, 64])
def test_shards_are_torch_chunks_padded(m):
    rows, cols = _random_shapes(11 + m, 9)
    q, off, C = oracle.rowwise_layout(rows, cols, m)
    grads = [synth.normal_bf16(synth.stream_key(m, STREAM_GRAD), int(i) * 4096, int(r * c), 1.0)
             for i, (r, c) in enumerate(zip(rows, cols))]
    buf = oracle.rowwise_copy_in(grads, rows, cols, m, 1.0)
    assert buf.size == m * C
    for t in range(len(rows)):
        T = torch.from_numpy(grads[t].astype(np.int32)).view(int(rows[t]), int(cols[t]))
        parts = torch.chunk(T, m, dim=0)
        for r in range(m):
            want = parts[r].reshape(-1).numpy() if r < len(parts) else np.zeros(0, np.int32)
            seg = buf[r * C + off[t]: r * C + off[t] + q[t] * cols[t]]
            assert np.array_equal(seg[:want.size], want.astype(np.uint16)), (t, r)
            assert not seg[want.size:].any(), (t, r)          # padding rows are zero


@pytest.mark.parametrize("m", [2, 5, 8])
def test_copy_out_inverts_copy_in(m):
    rows, cols = _random_shapes(40 + m, 12)
    grads = [synth.normal_bf16(synth.stream_key(m, STREAM_GRAD), int(i) * 4096, int(r * c), 1e-3)
             for i, (r, c) in enumerate(zip(rows, cols))]
    outs = oracle.rowwise_copy_out(oracle.rowwise_copy_in(grads, rows, cols, m, 1.0), rows, cols, m)
    for o, g in zip(outs, grads):
        assert np.array_equal(o, g)
    # copy-in scales element by element exactly like the bucket copy-in
    buf = oracle.rowwise_copy_in(grads, rows, cols, m, 0.3)
    back = oracle.rowwise_copy_out(buf, rows, cols, m)
    for o, g in zip(back, grads):
        want = np.zeros_like(g)
        oracle.pack(g, want, 0.3)
        assert np.array_equal(o, want)
