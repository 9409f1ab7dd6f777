"""The host-buffer step (dbuf_adam8_step_host) runs a chunked pipeline on
large buckets: gradients arrive chunk by chunk on one stream, each chunk is
stepped once its gradients have landed, and its bf16 params leave on
another stream.  It must give exactly what the resident step gives: same
master weights, codes and scales, and a host copy equal to the bf16
bucket.  Full-size buckets with one-pass entries, LARGE blocks and 2-D
strips."""
import numpy as np
import pytest
import torch

import ragged_bucket_layout_b200 as rb
import synth
from bucket_pair import GRAD, MASTER, MQ, PARAM, VQ, Pair, bf16_to_np, hp_at

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["llama_layer_m8", "llama_layer_32x32_m8", "moe_layer_m64"])
def test_host_pipeline_equals_resident_step(name):
    w = synth.workload(name)
    A = Pair(w, with_oracle=False)      # host-buffer path
    B = Pair(w, with_oracle=False)      # resident path
    A.load_params()
    B.load_params()
    S = A.info["bucket"]
    out = torch.empty(S, dtype=torch.int16).pin_memory()
    for t in (1, 2):
        B.load_grads(t)
        g_host = B.D.array(GRAD).view(torch.int16).cpu().pin_memory()
        A.D.step_host(hp_at(t), 1.0 / w.m, g_host.data_ptr(), out.data_ptr())
        B.D.step(hp_at(t), 1.0 / w.m)
        torch.cuda.synchronize()
        assert np.array_equal(out.numpy().view(np.uint16), bf16_to_np(B.D.array(PARAM))), t
        for kind in (MASTER, MQ, VQ):
            assert torch.equal(A.D.array(kind), B.D.array(kind)), (t, kind)
        assert torch.equal(A.D.scales(), B.D.scales()), t
        assert torch.equal(A.D.array(GRAD), B.D.array(GRAD)), t
    assert A.D.device_status() == 0 and B.D.device_status() == 0
