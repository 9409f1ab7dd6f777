"""GPU parity of the fused step on 2-D quantisation blocks (tiles of k rows x
block_cols columns, the 32x32 blocks of the 8-bit Adam case study) against
the oracle, through the C-ABI: the tile mix over every STRIP path (several
rows per chunk, one row piece per chunk, a narrow last strip, 256 tiles in a
strip, a tile as wide as a strip, short last row blocks) and the Llama layer
with 32x32 blocks at full size."""
import os

import numpy as np
import pytest

import synth
from bucket_pair import Pair, compare, hp_at, to_torch_bf16

pytestmark = pytest.mark.gpu


def _run(name, steps, threads=1):
    P = Pair(synth.workload(name))
    P.load_params()
    for t in range(1, steps + 1):
        P.load_grads(t)
        P.D.step(hp_at(t), 1.0 / P.w.m)
        P.O.step(hp_at(t), t, 1.0 / P.w.m, threads=threads)
        c = compare(P.gpu_state(), P.oracle_state(), P.O.pad)
        assert all(v == 0 for v in c.values()), (t, c)
    assert P.D.device_status() == 0


@pytest.mark.parametrize("name", ["tiles_mix_m4", "tiles_mix_m8"])
def test_tiles_mix_bit_exact(name):
    _run(name, 4)


def test_tiles_first_step_zero_grad_gives_zero_codes():
    P = Pair(synth.workload("tiles_mix_m4"))
    P.load_params()
    P.D.step(hp_at(1), 0.25)
    P.O.step(hp_at(1), 1, 0.25)
    g = P.gpu_state()
    c = compare(g, P.oracle_state(), P.O.pad)
    assert all(v == 0 for v in c.values()), c
    assert not g["mq"].any() and not g["vq"].any() and not g["sc"].any()


def test_tiles_copy_in_equals_zero_copy():
    w = synth.workload("tiles_mix_m4")
    A, B = Pair(w, with_oracle=False), Pair(w, with_oracle=False)
    A.load_params()
    B.load_params()
    for t in (1, 2):
        grads = [to_torch_bf16(A.grads_of(i, t)).cuda().view(int(A.r[i]), int(A.c[i])) for i in range(len(A.n))]
        A.D.pack(grads, 1.0 / w.m)
        A.D.step(hp_at(t), 1.0)
        B.load_grads(t)
        B.D.step(hp_at(t), 1.0 / w.m)
        a, b = A.gpu_state(), B.gpu_state()
        for key in ("p", "pb", "mq", "vq", "sc"):
            assert np.array_equal(a[key], b[key]), (t, key)


def test_full_size_llama_32x32_bit_exact():
    """218M parameters, 212,994 tiles of 32x32 elements, m = 8; two steps
    against the whole-bucket oracle (OpenMP over tiles)."""
    _run("llama_layer_32x32_m8", 2, threads=os.cpu_count() or 1)
