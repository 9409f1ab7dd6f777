"""GPU parity of the row-wise (FSDP2-style) baseline's interleaved copy-in /
copy-out against the oracle, through the C-ABI: bit-exact, with tensor and
buffer pointers at every 2-byte offset within 16 bytes, padding rows
written as zeros, and the Llama-layer shapes at full size."""
import numpy as np
import pytest
import torch

import oracle
import ragged_bucket_layout_b200 as rb
import synth
from synth.rng import STREAM_GRAD

pytestmark = pytest.mark.gpu


def _dev_bits(bits, shift):
    """A device bf16 view of `bits` starting `shift` elements into a fresh buffer."""
    buf = torch.zeros(bits.size + 16, dtype=torch.int16, device="cuda")
    buf[shift:shift + bits.size].copy_(torch.from_numpy(bits.view(np.int16)))
    return buf, buf[shift:shift + bits.size]


def _np(t):
    return t.cpu().numpy().view(np.uint16)


def _grads(rows, cols, seed):
    key = synth.stream_key(seed, STREAM_GRAD)
    return [synth.normal_bf16(key, i * (1 << 24), int(r) * int(c), 1e-3) for i, (r, c) in enumerate(zip(rows, cols))]


@pytest.mark.parametrize("m", [1, 3, 8, 64])
@pytest.mark.parametrize("flat_shift", [0, 1, 5])
def test_copy_in_and_out_match_oracle(m, flat_shift):
    w = synth.workload("ragged_mix_m4")
    rows, cols, _ = w.arrays()
    R = rb.Rowwise(rows, cols, m)
    q, off, C = oracle.rowwise_layout(rows, cols, m)
    assert R.chunk == C and R.shard_rows == q.tolist() and R.offsets == off.tolist()
    grads = _grads(rows, cols, 100 + m)
    keep = [_dev_bits(g, (i + flat_shift) % 8) for i, g in enumerate(grads)]
    # copy-in into a buffer full of garbage: every element must be written
    flat_buf = torch.full((m * C + 16,), 0x3F80, dtype=torch.int16, device="cuda")
    flat = flat_buf[flat_shift:flat_shift + m * C]
    R.copy_in([v for _, v in keep], 0.3, flat)
    torch.cuda.synchronize()
    want = oracle.rowwise_copy_in(grads, rows, cols, m, 0.3)
    assert np.array_equal(_np(flat), want)
    # copy-out of an arbitrary gathered buffer into tensors at odd offsets
    gathered = synth.normal_bf16(synth.stream_key(7, STREAM_GRAD), 0, m * C, 1.0)
    gkeep, gdev = _dev_bits(gathered, flat_shift)
    outs = [_dev_bits(np.zeros(g.size, np.uint16), (3 * i + flat_shift) % 8) for i, g in enumerate(grads)]
    R.copy_out(gdev, [v for _, v in outs])
    torch.cuda.synchronize()
    want = oracle.rowwise_copy_out(gathered, rows, cols, m)
    for i, (o, x) in enumerate(zip(outs, want)):
        assert np.array_equal(_np(o[1]), x), i
    assert R.status() == 0


def test_full_size_llama_round_trip():
    """Llama-layer shapes (218M parameters), m = 8: copy-in then copy-out at
    scale 1 returns every gradient bit for bit; copy-out equals the oracle's."""
    w = synth.workload("llama_layer_m8")
    rows, cols, _ = w.arrays()
    m = 8
    R = rb.Rowwise(rows, cols, m)
    grads = _grads(rows, cols, 9)
    dg = [torch.from_numpy(g.view(np.int16)).cuda() for g in grads]
    flat = torch.empty(m * R.chunk, dtype=torch.int16, device="cuda")
    R.copy_in(dg, 1.0, flat)
    outs = [torch.empty_like(g) for g in dg]
    R.copy_out(flat, outs)
    torch.cuda.synchronize()
    for o, g in zip(outs, dg):
        assert torch.equal(o, g)
    flat_np = _np(flat)
    want = oracle.rowwise_copy_in(grads, rows, cols, m, 1.0)
    assert np.array_equal(flat_np, want)
    assert R.status() == 0


def test_invalid_pointers_rejected():
    R = rb.Rowwise([4, 3], [2, 5], 2)
    flat = torch.zeros(2 * R.chunk + 2, dtype=torch.int16, device="cuda")
    a = torch.zeros(8, dtype=torch.int16, device="cuda")
    b = torch.zeros(15, dtype=torch.int16, device="cuda")
    with pytest.raises(rb.DbufError) as e:
        R.copy_out(flat, [a.data_ptr() + 1, b])
    assert e.value.status == rb.DBUF_EINVAL
    with pytest.raises(rb.DbufError):
        R.copy_in([a, 0], 1.0, flat)
    assert R.status() == 0
