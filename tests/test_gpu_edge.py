"""Edge cases of the bucket step on the GPU, each against the oracle."""
import numpy as np
import pytest
import torch

import ragged_bucket_layout_b200 as rb
import synth
from bucket_pair import Pair, compare, hp_at
from synth.workloads import TensorSpec, Workload

pytestmark = pytest.mark.gpu


class _Raw:
    """A device pointer exposed to torch through __cuda_array_interface__."""

    def __init__(self, ptr, n, typestr):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": typestr, "data": (ptr, False),
                                         "version": 3}


def check(tensors, m, steps=2, seed=11):
    w = Workload("edge", tensors, m=m, seed=seed)
    P = Pair(w)
    P.load_params()
    for t in range(1, steps + 1):
        P.load_grads(t)
        P.D.step(hp_at(t), 1.0 / m)
        P.O.step(hp_at(t), t, 1.0 / m)
        g = P.gpu_state()
        c = compare(g, P.oracle_state(), P.O.pad)
        assert all(v == 0 for v in c.values()), c
        P.adopt_gpu_state(g)
    assert P.D.device_status() == 0
    return P


def test_empty_bucket():
    p = rb.dbuf_plan([], [], [], 4, 16)
    D = rb.DBuffer(p)
    D.step(hp_at(1), 0.25)
    torch.cuda.synchronize()
    assert D.device_status() == 0


@pytest.mark.parametrize("tensors,m", [
    ([TensorSpec("one", 1, 1, 1)], 1),                          # a single element
    ([TensorSpec("vec", 4097, 1, 1)], 4),                       # every element its own block
    ([TensorSpec("b3", 999, 1, 3)], 2),                         # 3-element blocks, unaligned
    ([TensorSpec("b4080", 3, 4080, 1), TensorSpec("b4096", 3, 4096, 1),
      TensorSpec("b4095", 3, 4095, 1), TensorSpec("b4097", 3, 4097, 1)], 2),  # around one tile
    ([TensorSpec("giant", 1, 300001, 1)], 1),                   # one odd block of 300,001
    ([TensorSpec("rows", 33, 7168, 16)], 8),                    # partial last block (1 row)
    ([TensorSpec("m1", 64, 64, 4)], 1),                         # one device
    ([TensorSpec(f"t{i}", 1 + i, 3 + 2 * i, 1 + i // 2) for i in range(40)], 16),  # many tiny tensors
])
def test_edge_layouts(tensors, m):
    check(tensors, m)


def test_zero_gradient_keeps_zero_state():
    w = Workload("zeros", [TensorSpec("a", 100, 48, 3), TensorSpec("b", 7, 1, 7)], m=2, seed=1)
    P = Pair(w)
    P.load_params()
    P.D.step(hp_at(1), 0.5)
    P.O.step(hp_at(1), 1, 0.5)
    g = P.gpu_state()
    compare(g, P.oracle_state(), P.O.pad)
    assert not g["sc"].any() and not g["mq"].any() and not g["vq"].any()


def test_invalid_hparams_and_wrong_arguments():
    P = Pair(synth.workload("tiny_m4"), with_oracle=False)
    with pytest.raises(rb.DbufError) as e:
        P.D.step(dict(hp_at(1), step=0), 1.0)
    assert e.value.status == rb.DBUF_EINVAL
    with pytest.raises(rb.DbufError) as e:
        P.D.step(dict(hp_at(1), beta1=1.0), 1.0)
    assert e.value.status == rb.DBUF_EINVAL
    with pytest.raises(rb.DbufError) as e:
        rb.dbuf_pack_grads(P.D.handle, [0, 0, 0], 1.0, P.D.stream)
    assert e.value.status == rb.DBUF_EINVAL
    # a plan whose alignment is not a multiple of 16 cannot back a device bucket
    p = rb.dbuf_plan([4], [4], [1], 2, 8)
    with pytest.raises(rb.DbufError) as e:
        rb.DBuffer(p)
    assert e.value.status == rb.DBUF_EINVAL
    # caller memory too small
    p = rb.dbuf_plan([64], [64], [1], 2, 16)
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(rb.DbufError) as e:
        rb.dbuf_create(p, small.data_ptr(), small.numel(), None)
    assert e.value.status == rb.DBUF_EINVAL


def test_library_allocated_bucket_and_host_step():
    """dbuf_create with NULL base (library cudaMalloc) and the host-buffer
    step: same results as the oracle."""
    w = synth.workload("ragged_mix_m4")
    P = Pair(w)
    own = rb.dbuf_create(P.plan, None, 0, None)
    try:
        S = P.info["bucket"]
        stream = torch.cuda.current_stream()
        # parameters into the library-owned master via its bucket pointer
        ptr, n = rb.dbuf_bucket(own, rb.DBUF_MASTER_F32)
        assert n == S
        P.load_params()
        torch.cuda.synchronize()
        master = torch.as_tensor(_Raw(ptr, S, "<f4"), device="cuda")
        master.copy_(torch.from_numpy(P.O.p.copy()))
        P.load_grads(1)
        gh = torch.from_numpy(P.O.g.view(np.int16).copy()).pin_memory()
        out = torch.empty(S, dtype=torch.int16).pin_memory()
        rb.dbuf_adam8_step_host(own, hp_at(1), 0.25, gh.data_ptr(), out.data_ptr(), stream)
        torch.cuda.synchronize()
        P.O.step(hp_at(1), 1, 0.25)
        assert np.array_equal(out.numpy().view(np.uint16), P.O.pb)
        assert rb.dbuf_get_device_status(own, stream) == 0
    finally:
        rb.dbuf_destroy(own)

