"""The allocation-free gradient norm, checked against the bucket's own norm.

dbuf_grad_norm_noalloc is for callers that cannot allocate device memory
(code inside an allocator or memory-pool callback, a runtime that owns all
device memory, a loop that must not touch the allocator): its scratch is a
static device array of the library, so it takes only the input array and
the output location.  This file is collected last on purpose: if it fails,
a run that stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import ragged_bucket_layout_b200 as rb
import synth
from bucket_pair import GRAD, Pair, bf16_to_np

pytestmark = pytest.mark.gpu


def _bound(n):
    return max(1e-15, n * 2.0 ** -53)   # fp64 sums in two orders, relative


@pytest.mark.parametrize("gs", [1.0, 0.125])
def test_noalloc_norm_matches_bucket_norm_on_two_calls(gs):
    P = Pair(synth.workload("ragged_mix_m4"), with_oracle=False)
    P.load_grads(1)
    grad = P.D.array(GRAD)
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    P.D.grad_norm(gs, out[0:1])                      # the existing entry point
    stream = torch.cuda.current_stream()
    for call in (1, 2):                               # two calls in a row share the static scratch
        rb.dbuf_grad_norm_noalloc(grad.data_ptr(), grad.numel(), gs, out[call:call + 1].data_ptr(), stream)
    torch.cuda.synchronize()
    ref, a, b = out.cpu().numpy()
    assert ref > 0
    assert abs(a - ref) <= _bound(grad.numel()) * ref
    assert abs(b - ref) <= _bound(grad.numel()) * ref
    assert a == b


def test_noalloc_norm_odd_length_and_limits():
    rng = np.random.default_rng(0)
    n = 3 * (1 << 20) + 5                             # several CTAs and a tail shorter than a vector
    bits = torch.from_numpy(rng.normal(0, 1e-3, n).astype(np.float32)).to(torch.bfloat16)
    g = bits.cuda()
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    rb.dbuf_grad_norm_noalloc(g.data_ptr(), n, 0.5, out.data_ptr(), torch.cuda.current_stream())
    torch.cuda.synchronize()
    want = oracle.grad_norm(bits.view(torch.int16).numpy().view(np.uint16), 0.5)
    assert abs(out.item() - want) <= _bound(n) * want
    with pytest.raises(rb.DbufError) as e:
        rb.dbuf_grad_norm_noalloc(g.data_ptr(), (1 << 31) + 1, 1.0, out.data_ptr(), None)
    assert e.value.status == rb.DBUF_EINVAL
