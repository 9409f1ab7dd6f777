"""GPU parity of the DBuffer group operations beyond scale/zero: gradient
accumulation (group add), the global gradient norm and the clipped step,
each against the oracle through the C-ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bucket_pair import GRAD, Pair, bf16_to_np, compare, hp_at, to_torch_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["ragged_mix_m4", "tiny_m4"])
@pytest.mark.parametrize("scale", [0.25, 0.3])
def test_accumulate_matches_oracle(name, scale):
    P = Pair(synth.workload(name))
    P.load_grads(1)
    srcs, bits_list = [], []
    for i in range(len(P.n)):
        bits = P.grads_of(i, 2)
        shift = i % 8                                   # every 2-byte offset mod 16 bytes
        buf = torch.zeros(int(P.n[i]) + 8, dtype=torch.bfloat16, device="cuda")
        buf[shift:shift + int(P.n[i])].copy_(to_torch_bf16(bits))
        srcs.append(buf[shift:shift + int(P.n[i])])
        bits_list.append(bits)
    for rep in range(2):                                # two micro-batches
        P.D.accumulate(srcs, scale)
        for i in range(len(P.n)):
            oracle.accumulate(bits_list[i], P.O.g[P.O.tensor_slice(i)], scale)
        torch.cuda.synchronize()
        assert np.array_equal(bf16_to_np(P.D.array(GRAD)), P.O.g), rep
    assert P.D.device_status() == 0


def _norm_bound(n):
    # fp64 sums of n non-negative terms in two different orders differ by at
    # most about 2 n 2^-53 of the sum; the norm by half that, relatively.
    return max(1e-15, n * 2.0 ** -53)


@pytest.mark.parametrize("name", ["ragged_mix_m4", "llama_layer_m8"])
@pytest.mark.parametrize("gs", [1.0, 0.125])
def test_grad_norm_matches_oracle_and_is_deterministic(name, gs):
    P = Pair(synth.workload(name), with_oracle=False)
    P.load_grads(1)
    out = torch.zeros(2, dtype=torch.float64, device="cuda")
    P.D.grad_norm(gs, out[0:1])
    P.D.grad_norm(gs, out[1:2])
    torch.cuda.synchronize()
    a, b = out.cpu().numpy()
    assert a == b                                       # same bits run to run
    g = bf16_to_np(P.D.array(GRAD))
    want = oracle.grad_norm(g, gs)
    assert abs(a - want) <= _norm_bound(g.size) * want + 1e-300
    assert P.D.device_status() == 0


@pytest.mark.parametrize("max_norm", [1e-4, 0.05, 1e3])
def test_clipped_step_matches_oracle(max_norm):
    """The clipped step equals the oracle's step at the scale the oracle's
    own clipping rule gives for the device's norm; the device norm equals
    the oracle's within the fp64 summation bound."""
    w = synth.workload("ragged_mix_m4")
    P = Pair(w)
    P.load_params()
    gs = 1.0 / w.m
    norm = torch.zeros(1, dtype=torch.float64, device="cuda")
    for t in (1, 2, 3):
        P.load_grads(t)
        P.D.step_clipped(hp_at(t), gs, max_norm, norm)
        torch.cuda.synchronize()
        n_gpu = float(norm.item())
        n_orc = oracle.grad_norm(P.O.g, gs)
        assert abs(n_gpu - n_orc) <= _norm_bound(P.O.g.size) * n_orc
        gs_eff = oracle.clipped_scale(n_gpu, gs, max_norm)
        if max_norm < 1e-3:
            assert gs_eff < gs                          # clipping is active
        if max_norm > 1.0:
            assert gs_eff == np.float32(gs)
        P.O.step(hp_at(t), t, gs_eff)
        g = P.gpu_state()
        c = compare(g, P.oracle_state(), P.O.pad)
        assert all(v == 0 for v in c.values()), c
        P.adopt_gpu_state(g)
    assert P.D.device_status() == 0


def test_empty_bucket_norm_is_zero():
    import ragged_bucket_layout_b200 as rb
    D = rb.DBuffer(rb.dbuf_plan([], [], [], 4, 16))
    out = torch.full((1,), 7.0, dtype=torch.float64, device="cuda")
    D.grad_norm(1.0, out)
    D.step_clipped(hp_at(1), 1.0, 1.0, out)
    torch.cuda.synchronize()
    assert out.item() == 0.0 and D.device_status() == 0
