"""The seeded input generator (synth/gen.c) against its published definitions.

It feeds both the library and the oracle, so parity does not depend on it;
these checks make sure it is the generator it says it is.
"""
import numpy as np
import torch

import synth
from synth.rng import load_lib


def test_counter_mode_is_splitmix64():
    """With key 0, element i is output i of SplitMix64 (Steele, Lea and
    Flood, OOPSLA 2014; the mixer of Vigna's reference splitmix64.c)
    started from state 0: its first outputs are 0xE220A8397B1DCDAF,
    0x6E789E6AA1B965F4, 0x06C45D188009454F."""
    lib = load_lib()
    assert [lib.synth_u64(0, i) for i in range(3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                                       0x06C45D188009454F]


def test_box_muller_normals_have_the_stated_moments():
    """2^20 draws of sigma * N(0, 1): mean, standard deviation, skew and
    excess kurtosis within a few standard errors of 0, sigma, 0, 0."""
    n, sigma = 1 << 20, 0.02
    x = synth.normal_f32(synth.stream_key(11, 1), 0, n, sigma).astype(np.float64)
    z = x / sigma
    se = 1.0 / np.sqrt(n)
    assert abs(z.mean()) < 5 * se
    assert abs(z.std() - 1.0) < 5 * se
    assert abs(np.mean(z ** 3)) < 5 * np.sqrt(6.0) * se
    assert abs(np.mean(z ** 4) - 3.0) < 5 * np.sqrt(24.0) * se


def test_bf16_stream_is_the_rounded_f32_stream():
    """normal_bf16 is round-to-nearest-even of the same fp32 values (torch's
    float32 -> bfloat16 conversion), element for element."""
    key = synth.stream_key(5, 3)
    f = synth.normal_f32(key, 1000, 4096, 1e-3)
    b = synth.normal_bf16(key, 1000, 4096, 1e-3)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b, want)


def test_elements_regenerate_on_their_own():
    """Element e does not depend on where a request starts (counter mode)."""
    key = synth.stream_key(2, 7)
    whole = synth.normal_f32(key, 0, 5000, 1.0)
    assert np.array_equal(synth.normal_f32(key, 1234, 100, 1.0), whole[1234:1334])
