"""The library's own device allocation failing (CUDA, B200).

Run after the parity tests: it drives the device allocator to a refusal on
purpose (no fault: cudaMalloc returns an error), then checks that the
device still works.
"""
import pytest
import torch

import ragged_bucket_layout_b200 as rb
import synth
from bucket_pair import Pair, compare, hp_at

pytestmark = pytest.mark.gpu


def test_allocation_failure_is_reported_and_the_device_keeps_working():
    """A bucket larger than the device: one tensor of 2^35 elements in one
    block, about 343 GB of state on a 183 GB B200.  The library's own
    cudaMalloc fails, dbuf_create returns DBUF_ENOMEM naming the size, and
    the device keeps working: a tiny bucket created afterwards steps
    bit-identically to the oracle."""
    p = rb.dbuf_plan([1 << 18], [1 << 17], [1 << 18], 1, 16)
    need = rb.dbuf_required_bytes(p)
    assert need > torch.cuda.mem_get_info()[1]
    with pytest.raises(rb.DbufError) as e:
        rb.dbuf_create(p)
    assert e.value.status == rb.DBUF_ENOMEM and str(need) in str(e.value)
    P = Pair(synth.workload("tiny_m4"))
    P.load_params()
    P.load_grads(1)
    P.D.step(hp_at(1), 0.25)
    P.O.step(hp_at(1), 1, 0.25)
    compare(P.gpu_state(), P.oracle_state(), P.O.pad)
    assert P.D.device_status() == 0
