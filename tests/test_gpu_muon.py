"""GPU parity of the Muon path against the oracle, through the C-ABI.

- momentum (fp32, same operation order) and the bf16 param copy of the
  master weights are bit-exact;
- the orthogonalised update (bf16 Newton-Schulz with fp32 accumulation)
  is within MUON_TOL relative Frobenius error of the oracle's float64
  iteration.  Reading of the bar: bf16 keeps 8 significant bits (unit
  roundoff 2^-9 = 0.002); each of the five iterations rounds its three
  products to bf16, and the iteration maps errors in singular values near
  the fixed band with a slope of at most about 1.5, so about
  15 * 0.002 = 0.03 bounds the relative error; measured values are near
  0.01.
"""
import numpy as np
import pytest
import torch

import oracle
import ragged_bucket_layout_b200 as rb
import synth
from bucket_pair import MASTER, PARAM, Pair, bf16_to_np
from synth.rng import STREAM_GRAD

pytestmark = pytest.mark.gpu

MUON_TOL = 0.03
HP = dict(lr=0.02, momentum=0.95, weight_decay=0.01, eps=1e-7, ns_steps=5, nesterov=1)


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _bf16_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("shape", [(256, 1024), (1024, 256), (512, 512), (300, 700), (4096, 4096)])
def test_orthogonalize_matches_oracle(shape):
    R, C = shape
    r = np.array([R], np.int64)
    c = np.array([C], np.int64)
    plan = rb.dbuf_plan(r, c, r, 1, 16)
    D = rb.DBuffer(plan)
    M = rb.Muon(D, [0])
    u = synth.normal_f32(synth.stream_key(R + C, STREAM_GRAD), 0, R * C, 1.0).reshape(R, C)
    x = M.orthogonalize(torch.from_numpy(u).cuda(), steps=5, eps=1e-7)
    torch.cuda.synchronize()
    want = oracle.newton_schulz(u.astype(np.float64), 5, 1e-7)
    err = _rel(_bf16_to_f64(x), want)
    print(shape, "relative error", err)
    assert err <= MUON_TOL


def _tensor_ids(w):
    return [i for i, t in enumerate(w.tensors) if t.rows >= 2 and t.cols >= 2]


@pytest.mark.parametrize("name", ["tiny_m4", "ragged_mix_m4"])
def test_muon_step_matches_oracle(name):
    w = synth.workload(name)
    P = Pair(w, with_oracle=False)
    P.load_params()
    ids = _tensor_ids(w)
    M = rb.Muon(P.D, ids)
    gs = 1.0 / w.m
    masters = [P.D.views(MASTER)[i].detach().cpu().numpy().reshape(-1).copy() for i in ids]
    moms = [np.zeros(int(P.n[i]), np.float32) for i in ids]
    for t in (1, 2, 3):
        P.load_grads(t)
        M.step(HP, gs)
        torch.cuda.synchronize()
        views_m = P.D.views(MASTER)
        views_p = P.D.views(PARAM)
        for j, i in enumerate(ids):
            R, C = int(P.r[i]), int(P.c[i])
            U = oracle.muon_momentum(moms[j], P.grads_of(i, t), HP["momentum"], gs, nesterov=True)
            gm = M.momentum(j).cpu().numpy()
            assert np.array_equal(gm, moms[j]), (t, i)               # fp32, same op order
            X = oracle.newton_schulz(U.reshape(R, C).astype(np.float64), HP["ns_steps"], HP["eps"])
            lrs = HP["lr"] * oracle.muon_update_scale(R, C)
            decay = np.float32(1.0 - HP["lr"] * HP["weight_decay"])
            p_new = views_m[i].detach().cpu().numpy().reshape(-1)
            implied = (masters[j].astype(np.float64) * np.float64(decay) - p_new.astype(np.float64)) / lrs
            assert _rel(implied.reshape(R, C), X) <= MUON_TOL, (t, i)
            pb = bf16_to_np(views_p[i].reshape(-1))
            assert np.array_equal(pb, oracle.bf16_round(p_new)), (t, i)
            masters[j] = p_new.copy()


def test_muon_rejects_bad_ids():
    w = synth.workload("tiny_m4")
    P = Pair(w, with_oracle=False)
    for ids in ([1], [0, 0], [7], [-1]):      # tensor 1 is a vector (cols 1)
        with pytest.raises(rb.DbufError) as e:
            rb.Muon(P.D, ids)
        assert e.value.status == rb.DBUF_EINVAL
