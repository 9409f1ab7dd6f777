"""A workload set up twice with the same bytes: on the GPU through the C-ABI
(libdbuf via the Python binding) and on the host in the oracle.

Inputs come from the counter-based generator in ``synth`` only.  Element e
of tensor i has generator index cum[i] + e (cum = running element count in
the caller's tensor order), so any block can be regenerated on its own.
"""
import numpy as np
import torch

import oracle
import ragged_bucket_layout_b200 as rb
import synth
from synth.rng import STREAM_GRAD, STREAM_PARAM
from synth.workloads import GRAD_SIGMA, PARAM_SIGMA

MASTER, PARAM, GRAD, MQ, VQ = (rb.DBUF_MASTER_F32, rb.DBUF_PARAM_BF16, rb.DBUF_GRAD_BF16,
                               rb.DBUF_M_I8, rb.DBUF_V_U8)


def hp_at(t):
    return dict(synth.HPARAMS, step=t)


def grad_key(seed, t):
    return synth.stream_key(seed, STREAM_GRAD * 1000 + t)


def to_torch_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def bf16_to_np(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class Pair:
    def __init__(self, w, with_oracle=True):
        self.w = w
        self.r, self.c, self.k = w.arrays()
        self.bc = w.block_cols()
        self.n = self.r * self.c
        self.b = self.k * self.c
        self.plan = rb.dbuf_plan(self.r, self.c, self.k, w.m, w.align, block_cols=self.bc)
        self.info = rb.dbuf_plan_info(self.plan)
        st, off, s = oracle.plan(self.r, self.c, self.k, w.m, w.align)
        assert st == oracle.OK
        assert off.tolist() == self.info["offsets"] and s == self.info["slice"], "layouts differ"
        self.off = off
        self.s = s
        self.cum = np.concatenate([[0], np.cumsum(self.n)]).astype(np.int64)
        self.D = rb.DBuffer(self.plan)
        self.O = oracle.Bucket(self.r, self.c, self.k, off, s, w.m, block_cols=self.bc) if with_oracle else None

    # ------------------------------------------------------------ inputs
    def load_params(self):
        key = synth.stream_key(self.w.seed, STREAM_PARAM)
        views = self.D.views(MASTER)
        for i in range(len(self.n)):
            vals = synth.normal_f32(key, int(self.cum[i]), int(self.n[i]), PARAM_SIGMA)
            if self.O is not None:
                self.O.p[self.O.tensor_slice(i)] = vals
            views[i].copy_(torch.from_numpy(vals).view(views[i].shape))

    def grads_of(self, i, t):
        return synth.normal_bf16(grad_key(self.w.seed, t), int(self.cum[i]), int(self.n[i]), GRAD_SIGMA)

    def load_grads(self, t):
        views = self.D.views(GRAD)
        for i in range(len(self.n)):
            bits = self.grads_of(i, t)
            if self.O is not None:
                self.O.g[self.O.tensor_slice(i)] = bits
            views[i].copy_(to_torch_bf16(bits).view(views[i].shape))

    # ------------------------------------------------------------ state
    def gpu_state(self):
        torch.cuda.synchronize()
        return dict(p=self.D.array(MASTER).cpu().numpy(), pb=bf16_to_np(self.D.array(PARAM)),
                    g=bf16_to_np(self.D.array(GRAD)),
                    mq=self.D.array(MQ).cpu().numpy(), vq=self.D.array(VQ).cpu().numpy(),
                    sc=self.D.scales().cpu().numpy())

    def oracle_state(self):
        O = self.O
        return dict(p=O.p, pb=O.pb, g=O.g, mq=O.mq, vq=O.vq, sc=np.stack([O.scale_m, O.scale_v], 1))

    def adopt_gpu_state(self, st):
        """Restart the oracle from the GPU's state (so a code that differs at a
        rounding tie does not carry into later steps)."""
        O = self.O
        O.p[:] = st["p"]
        O.mq[:] = st["mq"]
        O.vq[:] = st["vq"]
        O.scale_m[:] = st["sc"][:, 0]
        O.scale_v[:] = st["sc"][:, 1]


def compare(gpu, orc, pad_mask=None):
    """Check the parity bar; return mismatch counts.

    Bar: int8/uint8 codes equal apart from at most 1e-4 of codes off by +-1;
    fp32 master within 1e-6*|p| + 1e-7; bf16 copy within 1 ulp; scales within
    the master tolerance.  Returns exact-mismatch counts for the record.
    """
    out = {}
    p_g, p_o = gpu["p"], orc["p"]
    assert p_g.shape == p_o.shape
    assert np.all(np.abs(p_g.astype(np.float64) - p_o) <= 1e-6 * np.abs(p_o.astype(np.float64)) + 1e-7), \
        "master weights outside 1e-6|p|+1e-7"
    out["p"] = int(np.count_nonzero(p_g.view(np.uint32) != p_o.view(np.uint32)))
    d = np.abs(gpu["pb"].astype(np.int32) - orc["pb"].astype(np.int32))
    assert np.all(d <= 1), "bf16 copy off by more than 1 ulp"
    out["pb"] = int(np.count_nonzero(d))
    for key in ("mq", "vq"):
        dd = np.abs(gpu[key].astype(np.int32) - orc[key].astype(np.int32))
        assert np.all(dd <= 1), f"{key} codes off by more than 1"
        nbad = int(np.count_nonzero(dd))
        assert nbad <= 1e-4 * dd.size + 1, f"{key}: {nbad} codes off by 1"
        out[key] = nbad
    sc_g, sc_o = gpu["sc"], orc["sc"]
    assert sc_g.shape == sc_o.shape
    assert np.all(np.abs(sc_g.astype(np.float64) - sc_o) <= 1e-6 * np.abs(sc_o.astype(np.float64)) + 1e-12)
    out["sc"] = int(np.count_nonzero(sc_g.view(np.uint32) != sc_o.view(np.uint32)))
    if pad_mask is not None:
        assert not gpu["pb"][pad_mask].any(), "bf16 padding not zero"
    return out
