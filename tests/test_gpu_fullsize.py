"""Parity at the full workload sizes the bench times, in the same launch
configuration, on sampled blocks the oracle computes one by one, plus
properties checked over the whole bucket:

* sampled blocks: the first and last block of every tensor, the blocks on
  either side of every slice boundary, and random blocks;
* everywhere: the bf16 copy is the round-to-nearest-even of the master, the
  bf16 padding is zero, the device status word stays 0.

The 200-tensor copy-in bucket (4.8e9 parameters, bucket offsets past 2^32)
also checks copy-in against zero-copy bit for bit over the whole bucket.
"""
import gc

import numpy as np
import pytest
import torch

import oracle
import synth
from bucket_pair import (GRAD, MASTER, MQ, PARAM, VQ, Pair, bf16_to_np, compare, grad_key, hp_at,
                         to_torch_bf16)
from synth.workloads import GRAD_SIGMA

pytestmark = pytest.mark.gpu


def block_table(P):
    """(tensor, first element, length, block index) of every block, bucket order."""
    rows = []
    blk = 0
    for i in np.argsort(P.off, kind="stable"):
        n, b = int(P.n[i]), int(P.b[i])
        nb = -(-n // b)
        rows.append((i, int(P.off[i]), n, b, nb, blk))
        blk += nb
    return rows


def sample(P, rng, n_random=150):
    picks = set()
    tab = block_table(P)
    s = P.s
    for (i, o, n, b, nb, blk) in tab:
        picks.add((i, 0))
        picks.add((i, nb - 1))
        # blocks touching a slice boundary inside or at the tensor
        for R in range(((o // s) + 1) * s, o + n, s):
            j = (R - o) // b
            picks.add((i, min(j, nb - 1)))
            picks.add((i, max(j - 1, 0)))
    for _ in range(n_random):
        (i, o, n, b, nb, blk) = tab[rng.integers(len(tab))]
        picks.add((i, int(rng.integers(nb))))
    info = {t[0]: t for t in tab}
    out = []
    for (i, j) in sorted(picks):
        (_, o, n, b, nb, blk) = info[i]
        out.append((i, j, o + j * b, min(b, n - j * b), blk + j))
    return out


def pull(P, blocks):
    M, Q, V = P.D.array(MASTER), P.D.array(MQ), P.D.array(VQ)
    pb = P.D.array(PARAM)
    sc = P.D.scales()
    res = []
    for (_, _, e, ln, bi) in blocks:
        res.append(dict(p=M[e:e + ln].cpu().numpy(), mq=Q[e:e + ln].cpu().numpy(), vq=V[e:e + ln].cpu().numpy(),
                        pb=bf16_to_np(pb[e:e + ln]), sc=sc[bi].cpu().numpy()))
    return res


def oracle_on_blocks(P, blocks, pre, t, grad_scale):
    lens = np.array([b[3] for b in blocks], np.int64)
    start = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    p = np.concatenate([x["p"] for x in pre]).astype(np.float32)
    mq = np.concatenate([x["mq"] for x in pre]).astype(np.int8)
    vq = np.concatenate([x["vq"] for x in pre]).astype(np.uint8)
    sm = np.array([x["sc"][0] for x in pre], np.float32)
    sv = np.array([x["sc"][1] for x in pre], np.float32)
    g = np.concatenate([synth.normal_bf16(grad_key(P.w.seed, t), int(P.cum[i]) + j * int(P.b[i]), ln, GRAD_SIGMA)
                        for (i, j, _, ln, _) in blocks])
    pb = np.zeros(p.size, np.uint16)
    oracle.adam8_step(start, lens, np.arange(lens.size), p, g, mq, vq, sm, sv, pb, hp_at(t), t, grad_scale)
    return dict(p=p, pb=pb, mq=mq, vq=vq, sc=np.stack([sm, sv], 1))


def stack(blocks_state):
    return dict(p=np.concatenate([x["p"] for x in blocks_state]), pb=np.concatenate([x["pb"] for x in blocks_state]),
                mq=np.concatenate([x["mq"] for x in blocks_state]), vq=np.concatenate([x["vq"] for x in blocks_state]),
                sc=np.stack([x["sc"] for x in blocks_state]))


def whole_bucket_properties(P):
    M, pb = P.D.array(MASTER), P.D.array(PARAM)
    torch.cuda.synchronize()
    want = M.to(torch.bfloat16)
    pad = torch.ones(P.info["bucket"], dtype=torch.bool, device="cuda")
    for i in range(len(P.n)):
        pad[int(P.off[i]):int(P.off[i] + P.n[i])] = False
    want[pad] = 0
    assert torch.equal(pb.view(torch.int16), want.view(torch.int16))
    del want, pad


def run_full(name, steps=2, seed=0):
    P = Pair(synth.workload(name), with_oracle=False)
    P.load_params()
    rng = np.random.default_rng(seed)
    blocks = sample(P, rng)
    for t in range(1, steps + 1):
        P.load_grads(t)
        torch.cuda.synchronize()
        pre = pull(P, blocks)
        P.D.step(hp_at(t), 1.0 / P.w.m)
        torch.cuda.synchronize()
        post = stack(pull(P, blocks))
        want = oracle_on_blocks(P, blocks, pre, t, 1.0 / P.w.m)
        c = compare(post, want)
        print(name, "step", t, "sampled blocks", len(blocks), "mismatches", c)
    whole_bucket_properties(P)
    assert P.D.device_status() == 0
    return P


@pytest.mark.parametrize("name", ["llama_layer_m8", "moe_layer_m64", "ragged_stress_m8",
                                  "ragged_stress_m128", "ragged_stress_m1024"])
def test_full_size_sampled(name):
    P = run_full(name)
    P.D.close()
    del P
    gc.collect()
    torch.cuda.empty_cache()


def test_copy_in_200_tensors_full_size():
    """4.8e9 parameters in 200 separate gradient allocations: packed with 1/m
    then stepped, against gradients resident in a second bucket stepped with
    grad_scale 1/m.  Whole buckets compared bit for bit on the device;
    sampled blocks against the oracle."""
    w = synth.workload("copyin_200_m64")
    A = Pair(w, with_oracle=False)
    A.load_params()
    B = Pair(w, with_oracle=False)
    B.D.array(MASTER).copy_(A.D.array(MASTER))
    grads = []
    for i in range(len(A.n)):
        grads.append(to_torch_bf16(A.grads_of(i, 1)).cuda().view(int(A.r[i]), int(A.c[i])))
    bviews = B.D.views(GRAD)
    for i, g in enumerate(grads):
        bviews[i].copy_(g)
    blocks = sample(A, np.random.default_rng(1), n_random=60)
    torch.cuda.synchronize()
    pre = pull(A, blocks)
    A.D.pack(grads, 1.0 / w.m)
    A.D.step(hp_at(1), 1.0)
    B.D.step(hp_at(1), 1.0 / w.m)
    torch.cuda.synchronize()
    for which in (MASTER, PARAM, MQ, VQ):
        assert torch.equal(A.D.array(which).view(torch.uint8) if which in (MQ, VQ) else
                           A.D.array(which).view(torch.int16 if which == PARAM else torch.int32),
                           B.D.array(which).view(torch.uint8) if which in (MQ, VQ) else
                           B.D.array(which).view(torch.int16 if which == PARAM else torch.int32))
    assert torch.equal(A.D.scales().view(torch.int32), B.D.scales().view(torch.int32))
    post = stack(pull(A, blocks))
    want = oracle_on_blocks(A, blocks, pre, 1, 1.0 / w.m)
    compare(post, want)
    assert A.D.device_status() == 0 and B.D.device_status() == 0
    A.D.close()
    B.D.close()
