"""GPU parity of the fused bucket step and the copy-in against the oracle,
element by element over whole buckets (sizes the oracle finishes in
seconds, spanning many tiles, blocks of 1 to 286,720 elements, partial last
blocks and ragged tails).  Calls go through the C-ABI (libdbuf).
"""
import numpy as np
import pytest
import torch

import oracle
import ragged_bucket_layout_b200 as rb
import synth
from bucket_pair import GRAD, MASTER, PARAM, Pair, compare, hp_at, to_torch_bf16

pytestmark = pytest.mark.gpu


def run_steps(name, steps, restart=True, exact=False):
    P = Pair(synth.workload(name))
    P.load_params()
    counts = []
    for t in range(1, steps + 1):
        P.load_grads(t)
        P.D.step(hp_at(t), 1.0 / P.w.m)
        P.O.step(hp_at(t), t, 1.0 / P.w.m)
        g = P.gpu_state()
        c = compare(g, P.oracle_state(), P.O.pad)
        counts.append(c)
        if exact:
            assert all(v == 0 for v in c.values()), c
        if restart:
            P.adopt_gpu_state(g)
    assert P.D.device_status() == 0
    return counts


def test_tiny_bucket_ten_steps_bit_exact():
    """W[512,256] k=16, bias, LayerNorm; m=4; 10 steps.  Same op order on both
    sides, so every array is bit-identical (stronger than the tolerance)."""
    run_steps("tiny_m4", 10, restart=False, exact=True)


@pytest.mark.parametrize("name", ["ragged_mix_m4", "ragged_mix_m8"])
def test_ragged_mix(name):
    counts = run_steps(name, 4)
    print(name, counts)


def test_first_step_zero_grad_gives_zero_codes():
    P = Pair(synth.workload("ragged_mix_m4"))
    P.load_params()
    P.D.step(hp_at(1), 0.25)
    P.O.step(hp_at(1), 1, 0.25)
    g = P.gpu_state()
    compare(g, P.oracle_state(), P.O.pad)
    assert not g["mq"].any() and not g["vq"].any() and not g["sc"].any()


@pytest.mark.parametrize("name", ["ragged_mix_m4", "tiny_m4"])
def test_copy_in_equals_zero_copy(name):
    """Copy-in (separate per-tensor gradients packed with 1/m, step with
    grad_scale 1) and zero-copy (gradients resident in the bucket, step with
    grad_scale 1/m) give bit-identical buckets for power-of-two m."""
    w = synth.workload(name)
    A, B = Pair(w), Pair(w, with_oracle=False)
    A.load_params()
    B.load_params()
    for t in (1, 2, 3):
        grads = []
        for i in range(len(A.n)):
            grads.append(to_torch_bf16(A.grads_of(i, t)).cuda().view(int(A.r[i]), int(A.c[i])))
        A.D.pack(grads, 1.0 / w.m)
        A.D.step(hp_at(t), 1.0)
        B.load_grads(t)
        B.D.step(hp_at(t), 1.0 / w.m)
        # oracle of the copy-in path
        for i in range(len(A.n)):
            sl = A.O.tensor_slice(i)
            src = A.grads_of(i, t)
            A.O.g[sl] = 0
            oracle.pack(src, A.O.g[sl], 1.0 / w.m)
        A.O.step(hp_at(t), t, 1.0)
        ga, gb = A.gpu_state(), B.gpu_state()
        for key in ("p", "pb", "mq", "vq", "sc"):   # the grad buckets hold g/m and g
            assert np.array_equal(ga[key].view(np.uint8), gb[key].view(np.uint8)), key
        gb_scaled = np.zeros_like(gb["g"])
        oracle.pack(gb["g"], gb_scaled, 1.0 / w.m)
        assert np.array_equal(ga["g"], gb_scaled)
        compare(ga, A.oracle_state(), A.O.pad)
    assert A.D.device_status() == 0


def test_pack_matches_oracle_unaligned_sources():
    """Copy-in from sources at every 2-byte offset modulo 16 bytes (bulk-copy
    path and element-wise path)."""
    w = synth.workload("ragged_mix_m4")
    P = Pair(w)
    grads, srcs = [], []
    for i in range(len(P.n)):
        bits = P.grads_of(i, 1)
        shift = i % 8
        buf = torch.zeros(int(P.n[i]) + 8, dtype=torch.bfloat16, device="cuda")
        buf[shift:shift + int(P.n[i])].copy_(to_torch_bf16(bits))
        grads.append(buf[shift:shift + int(P.n[i])])
        srcs.append(bits)
    for scale in (1.0 / 4, 0.3):
        P.D.pack(grads, scale)
        torch.cuda.synchronize()
        got = P.gpu_state()["g"]
        want = np.zeros_like(P.O.g)
        for i in range(len(P.n)):
            sl = P.O.tensor_slice(i)
            oracle.pack(srcs[i], want[sl], scale)
        assert np.array_equal(got, want)
    assert P.D.device_status() == 0


def test_views_are_zero_copy_slices():
    P = Pair(synth.workload("tiny_m4"))
    base = P.D.array(MASTER)
    for i, v in enumerate(P.D.views(MASTER)):
        assert v.data_ptr() == base.data_ptr() + 4 * int(P.off[i])
        assert tuple(v.shape) == (int(P.r[i]), int(P.c[i]))
    pb = P.D.array(PARAM)
    for i, v in enumerate(P.D.views(PARAM)):
        assert v.data_ptr() == pb.data_ptr() + 2 * int(P.off[i])
