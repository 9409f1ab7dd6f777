"""Rank buckets on the device: every slice stepped as a bucket of its own.

A device of a data-parallel job holds only its slice (dbuf_plan_rank: fp32
master, codes and scales of s elements).  Stepped alone with that slice of
the gradients, each rank bucket must hold exactly that slice of the whole
bucket stepped at once (RaggedShard, paper Sec. 3: blocks never straddle a
slice, so the step exchanges nothing).  Both sides run the library's step
kernel; the whole bucket is itself checked against the oracle elsewhere.
"""
import pytest
import torch

import ragged_bucket_layout_b200 as rb
import synth

from test_oracle_rank_buckets import EDGE_CASES, _case

pytestmark = pytest.mark.gpu

KINDS = (rb.DBUF_MASTER_F32, rb.DBUF_PARAM_BF16, rb.DBUF_GRAD_BF16, rb.DBUF_M_I8, rb.DBUF_V_U8)
_INT_VIEW = {torch.float32: torch.int32, torch.bfloat16: torch.int16, torch.int8: torch.int8, torch.uint8: torch.uint8}


def _bits(t):
    return t.view(_INT_VIEW[t.dtype])


@pytest.mark.parametrize("name", ["tiny_m4", "ragged_mix_m8", "tiles_mix_m8", "llama_layer_m8",
                                  "llama_layer_32x32_m8"] + sorted(EDGE_CASES))
def test_rank_buckets_step_like_the_whole_bucket(name):
    torch.cuda.set_device(0)
    r, c, k, bc, m, align = _case(name)
    plan = rb.dbuf_plan(r, c, k, m, align, block_cols=bc)
    s = rb.dbuf_plan_info(plan)["slice"]
    W = rb.DBuffer(plan)
    rank_plans = [rb.dbuf_plan_rank(plan, q) for q in range(m)]
    R = [rb.DBuffer(p) for p in rank_plans]
    gen = torch.Generator(device="cuda").manual_seed(5)
    for v in W.views(rb.DBUF_MASTER_F32):
        v.copy_(torch.randn(v.shape, generator=gen, device="cuda") * 0.02)
    for q in range(m):
        R[q].array(rb.DBUF_MASTER_F32).copy_(W.array(rb.DBUF_MASTER_F32)[q * s:(q + 1) * s])
    for t in (1, 2, 3):
        for v in W.views(rb.DBUF_GRAD_BF16):
            v.copy_((torch.randn(v.shape, generator=gen, device="cuda") * 1e-3).to(torch.bfloat16))
        hp = dict(synth.HPARAMS, step=t)
        W.step(hp, 1.0 / m)
        for q in range(m):
            R[q].array(rb.DBUF_GRAD_BF16).copy_(W.array(rb.DBUF_GRAD_BF16)[q * s:(q + 1) * s])
            R[q].step(hp, 1.0 / m)
    torch.cuda.synchronize()
    assert W.device_status() == 0
    whole_scales = W.scales()
    for q in range(m):
        assert R[q].device_status() == 0, f"rank {q}"
        for which in KINDS:
            got, want = R[q].array(which), W.array(which)[q * s:(q + 1) * s]
            assert torch.equal(_bits(got), _bits(want)), f"rank {q}, array {which}"
        fb = rank_plans[q].first_block
        sc = R[q].scales()
        assert torch.equal(_bits(sc), _bits(whole_scales[fb:fb + sc.shape[0]])), f"rank {q}, scales"
    for d in R:
        d.close()
    W.close()
