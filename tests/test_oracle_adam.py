"""Pins of the oracle's block-wise 8-bit Adam step and copy-in pack (CPU only).

The pages (8-bit Adam case study, paper Sec. 6.3) state only that states are
quantised per block, locally, with blocks aligned to shards; the quantiser and
update formulas are this project's reading (linear absmax codes, int8 m,
uint8 sqrt(v), Adam with bias correction and decoupled weight decay).  What
pins the oracle, other than itself:

* a first step worked by hand (tests/golden/first_step_codes.json);
* the closed form of the first step from a zero state,
  p1 = p0 (1 - lr wd) - lr g / (|g| + eps), on random blocks including
  gradients near eps;
* brute force over all 255 / 256 codes: each stored code is the nearest
  level to the closed-form state;
* a special case that reduces to a library routine: when every element of a
  block keeps the same |g| (fixed signs), the codes are exact and the 8-bit
  step is plain AdamW (torch.optim.AdamW in float64) for many steps;
* quantiser invariants: an extreme code in every non-zero block, codes in
  range, dequantise/requantise is idempotent;
* bf16 rounding and the copy-in pack against torch's own conversion.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def f32(x):
    return float(np.float32(x))


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16).copy()


def bits_to_f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def one_bucket(block_lens):
    """Bucket holding consecutive blocks of the given lengths (no padding)."""
    lens = np.asarray(block_lens, np.int64)
    start = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    S = int(lens.sum())
    st = dict(p=np.zeros(S, np.float32), g=np.zeros(S, np.uint16), mq=np.zeros(S, np.int8),
              vq=np.zeros(S, np.uint8), pb=np.zeros(S, np.uint16),
              sm=np.zeros(lens.size, np.float32), sv=np.zeros(lens.size, np.float32))
    return start, lens, st


def run(start, lens, st, t, hp=HP, grad_scale=1.0, threads=1):
    oracle.adam8_step(start, lens, np.arange(lens.size), st["p"], st["g"], st["mq"], st["vq"],
                      st["sm"], st["sv"], st["pb"], hp, t, grad_scale, threads)


def test_golden_first_step(golden_dir):
    G = json.load(open(os.path.join(golden_dir, "first_step_codes.json")))
    g = np.array([a * 2.0 ** e for a, e in G["g_exponent_form"]], np.float32)
    start, lens, st = one_bucket([g.size])
    st["g"][:] = bf16_bits(g)
    assert np.array_equal(bits_to_f32(st["g"]), g)
    st["p"][:] = np.array(G["p0"], np.float32)
    hp = G["hparams"]
    run(start, lens, st, 1, hp)
    assert st["mq"].tolist() == G["qm"]
    assert st["vq"].tolist() == G["qv"]
    omb1 = 1.0 - f32(hp["beta1"])
    omb2 = 1.0 - f32(hp["beta2"])
    assert st["sm"][0] == pytest.approx(omb1 * 2.0 ** -10, rel=1e-6)
    assert st["sv"][0] == pytest.approx(np.sqrt(omb2) * 2.0 ** -10, rel=1e-6)
    lr, wd, eps = f32(hp["lr"]), f32(hp["weight_decay"]), f32(hp["eps"])
    p0 = np.array(G["p0"], np.float64)
    gd = g.astype(np.float64)
    want = p0 * (1 - lr * wd) - lr * gd / (np.abs(gd) + eps)
    assert np.all(np.abs(st["p"] - want) <= 1e-6 * np.abs(want) + 1e-7)


def _first_step_case(seed, lens):
    rng = np.random.default_rng(seed)
    start, lens, st = one_bucket(lens)
    S = st["p"].size
    g = rng.normal(0, 1e-3, S).astype(np.float32)
    # gradients near eps and exact zeros exercise the eps term and empty blocks
    tiny = rng.random(S) < 0.05
    g[tiny] = rng.normal(0, 3e-8, tiny.sum())
    g[rng.random(S) < 0.02] = 0.0
    g[int(start[-1]):] = 0.0  # last block all zero
    st["g"][:] = bf16_bits(g)
    st["p"][:] = rng.normal(0, 0.02, S).astype(np.float32)
    return start, lens, st


@pytest.mark.parametrize("grad_scale", [1.0, 0.125])
def test_first_step_closed_form(grad_scale):
    start, lens, st = _first_step_case(0, [1, 7, 16, 100, 4096, 333, 9])
    p0 = st["p"].astype(np.float64).copy()
    g = bits_to_f32(st["g"]).astype(np.float64) * grad_scale
    run(start, lens, st, 1, grad_scale=grad_scale)
    lr, wd, eps = f32(HP["lr"]), f32(HP["weight_decay"]), f32(HP["eps"])
    want = p0 * (1 - lr * wd) - lr * g / (np.abs(g) + eps)
    err = np.abs(st["p"] - want)
    assert np.all(err <= 1e-6 * np.abs(want) + 1e-7), err.max()
    # bf16 copy is the rounded master
    assert np.array_equal(st["pb"], bf16_bits(st["p"]))


def test_first_step_codes_are_nearest_levels():
    """Brute force: every code is the nearest of all 255 (m) / 256 (v) levels
    to the closed-form state m = (1-b1) g, sqrt(v) = sqrt(1-b2) |g|."""
    start, lens, st = _first_step_case(1, [1, 8, 16, 257, 4096, 999])
    g = bits_to_f32(st["g"]).astype(np.float64)
    run(start, lens, st, 1)
    omb1 = 1.0 - f32(HP["beta1"])
    omb2 = 1.0 - f32(HP["beta2"])
    levels_m = np.arange(-127, 128)
    levels_v = np.arange(0, 256)
    ties = 0
    for j, (a, n) in enumerate(zip(start, lens)):
        sl = slice(int(a), int(a + n))
        m = omb1 * g[sl]
        r = np.sqrt(omb2) * np.abs(g[sl])
        am, ar = np.abs(m).max(), r.max()
        assert st["sm"][j] == pytest.approx(am, rel=1e-6, abs=0)
        assert st["sv"][j] == pytest.approx(ar, rel=1e-6, abs=0)
        if am == 0:
            assert not st["mq"][sl].any() and not st["vq"][sl].any()
            continue
        xm = m * 127 / am
        xv = r * 255 / ar
        best_m = levels_m[np.argmin(np.abs(xm[:, None] - levels_m[None, :]), axis=1)]
        best_v = levels_v[np.argmin(np.abs(xv[:, None] - levels_v[None, :]), axis=1)]
        near_m = np.abs(np.abs(xm - np.floor(xm)) - 0.5) < 1e-4
        near_v = np.abs(np.abs(xv - np.floor(xv)) - 0.5) < 1e-4
        ok_m = (st["mq"][sl] == best_m) | (near_m & (np.abs(st["mq"][sl] - best_m) <= 1))
        ok_v = (st["vq"][sl] == best_v) | (near_v & (np.abs(st["vq"][sl].astype(int) - best_v) <= 1))
        assert ok_m.all() and ok_v.all()
        ties += int((st["mq"][sl] != best_m).sum() + (st["vq"][sl] != best_v).sum())
    # bf16 gradients have 8 significant bits, so exact half-way ratios are
    # common; a code may sit on either side only there.
    print(f"codes off the fp64 nearest level (all at half-way points): {ties}")


def test_uniform_magnitude_blocks_reduce_to_adamw():
    """Fixed per-element signs and one |g| per block per step: |m| and v are
    uniform inside each block, so the codes hold them exactly (up to fp32
    rounding) and the 8-bit step must follow torch.optim.AdamW."""
    rng = np.random.default_rng(4)
    lens = [1, 5, 16, 64, 300]
    start, lens_a, st = one_bucket(lens)
    S = st["p"].size
    sign = np.where(rng.random(S) < 0.5, -1.0, 1.0)
    st["p"][:] = rng.normal(0, 0.02, S).astype(np.float32)
    ref = torch.tensor(st["p"].astype(np.float64), requires_grad=True)
    opt = torch.optim.AdamW([ref], lr=f32(HP["lr"]), betas=(f32(HP["beta1"]), f32(HP["beta2"])),
                            eps=f32(HP["eps"]), weight_decay=f32(HP["weight_decay"]))
    blk = np.repeat(np.arange(len(lens)), lens)
    for t in range(1, 31):
        mag = np.exp(rng.uniform(np.log(1e-5), np.log(1e-2), len(lens)))
        mag = bits_to_f32(bf16_bits(mag.astype(np.float32))).astype(np.float64)
        g = sign * mag[blk]
        st["g"][:] = bf16_bits(g.astype(np.float32))
        run(start, lens_a, st, t)
        ref.grad = torch.tensor(bits_to_f32(st["g"]).astype(np.float64))
        opt.step()
        want = ref.detach().numpy()
        err = np.abs(st["p"] - want)
        assert np.all(err <= 1e-6 * np.abs(want) + 1e-7), (t, err.max())
        assert np.all(np.abs(st["mq"]) == 127)
        assert np.all(st["vq"] == 255)


def test_quantiser_invariants_many_steps():
    rng = np.random.default_rng(9)
    lens = [1, 2, 8, 16, 48, 512, 4096, 5000]
    start, lens_a, st = one_bucket(lens)
    S = st["p"].size
    st["p"][:] = rng.normal(0, 0.02, S).astype(np.float32)
    for t in range(1, 8):
        st["g"][:] = bf16_bits(rng.normal(0, 1e-3, S).astype(np.float32))
        run(start, lens_a, st, t)
        assert np.all(st["mq"] >= -127)
        for j, (a, n) in enumerate(zip(start, lens_a)):
            sl = slice(int(a), int(a + n))
            if st["sm"][j] > 0:
                assert np.abs(st["mq"][sl].astype(int)).max() == 127
            if st["sv"][j] > 0:
                assert st["vq"][sl].max() == 255


def test_requantise_is_idempotent():
    """With b1 = b2 = 1 and a zero gradient the step rebuilds m and sqrt(v)
    from the codes and requantises them: codes and scales come back."""
    rng = np.random.default_rng(2)
    lens = [1, 9, 16, 700]
    start, lens_a, st = one_bucket(lens)
    S = st["p"].size
    st["mq"][:] = rng.integers(-127, 128, S).astype(np.int8)
    st["vq"][:] = rng.integers(0, 256, S).astype(np.uint8)
    for j, (a, n) in enumerate(zip(start, lens_a)):  # each block holds its extremes
        st["mq"][a] = 127 if j % 2 else -127
        st["vq"][a + n - 1] = 255
    st["sm"][:] = rng.uniform(1e-4, 1e-2, len(lens)).astype(np.float32)
    st["sv"][:] = rng.uniform(1e-4, 1e-2, len(lens)).astype(np.float32)
    mq0, vq0, sm0, sv0 = st["mq"].copy(), st["vq"].copy(), st["sm"].copy(), st["sv"].copy()
    hp = dict(lr=1e-3, beta1=1.0, beta2=1.0, eps=1e-8, weight_decay=0.0)
    with np.errstate(all="ignore"):
        run(start, lens_a, st, 1, hp)
    assert np.array_equal(st["mq"], mq0)
    assert np.array_equal(st["vq"], vq0)
    assert np.allclose(st["sm"], sm0, rtol=2e-7, atol=0)
    assert np.allclose(st["sv"], sv0, rtol=2e-7, atol=0)


def test_threads_do_not_change_results():
    start, lens, st1 = _first_step_case(3, [3, 17, 4096, 1, 64] * 20)
    st2 = {k: v.copy() for k, v in st1.items()}
    for t in (1, 2):
        run(start, lens, st1, t, threads=1)
        run(start, lens, st2, t, threads=4)
        for k in st1:
            assert np.array_equal(st1[k], st2[k]), k


def test_step_scalars_closed_forms():
    c = oracle.step_scalars(1e-3, 0.9, 0.999, 1e-8, 0.01, 3)
    b1, omb1, b2, omb2, sq2, eps_hat, step_hat, decay = [float(x) for x in c]
    B1, B2, lr, wd, eps = f32(0.9), f32(0.999), f32(1e-3), f32(0.01), f32(1e-8)
    assert b1 == f32(B1) and omb1 == f32(1 - B1) and b2 == f32(B2) and omb2 == f32(1 - B2)
    assert sq2 == f32(np.sqrt(1 - B2 ** 3))
    assert eps_hat == f32(eps * np.sqrt(1 - B2 ** 3))
    assert step_hat == f32(lr * np.sqrt(1 - B2 ** 3) / (1 - B1 ** 3))
    assert decay == f32(1 - lr * wd)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, 1, 100000).astype(np.float32),
                        rng.normal(0, 1e-30, 1000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 65504.0, 3e38, -3e38, np.inf, -np.inf], np.float32)])
    # exact ties: low 16 bits = 0x8000
    u = rng.integers(0, 2 ** 31, 2000, dtype=np.uint64).astype(np.uint32)
    ties = ((u & 0x7F7F0000) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties])
    assert np.array_equal(oracle.bf16_round(x), bf16_bits(x))


@pytest.mark.parametrize("scale", [1.0, 1 / 64, 1 / 8, 0.3])
def test_pack_matches_torch(scale):
    rng = np.random.default_rng(1)
    src = bf16_bits(rng.normal(0, 1e-3, 5000).astype(np.float32))
    dst = np.zeros(6000, np.uint16)
    oracle.pack(src, dst, scale)
    want = (torch.from_numpy(bits_to_f32(src)) * np.float32(scale)).to(torch.bfloat16)
    assert np.array_equal(dst[:5000], want.view(torch.int16).numpy().view(np.uint16))
    assert not dst[5000:].any()
