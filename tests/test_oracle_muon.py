"""Pins of the oracle's Muon pieces (CPU only).

- Newton-Schulz is a spectral map: for U = P diag(s) Q^T the result is
  P diag(phi(s / (||U||_F + eps))) Q^T with phi the quintic
  p(x) = a x + b x^3 + c x^5 applied `steps` times, checked against numpy's
  SVD for wide, tall and square matrices;
- after five steps every singular value that starts in [0.02, 1] lies in
  the band the published coefficients are chosen for (about 0.7 to 1.2);
- momentum of a constant gradient follows g (1 - beta^t) / (1 - beta), and
  the Nesterov direction is g + beta * mom;
- the shape factor is sqrt(max(1, rows / cols)).
"""
import numpy as np
import pytest

import oracle
import synth
from synth.rng import STREAM_GRAD


def _phi(x, steps):
    a, b, c = oracle.NS_COEFFS
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


@pytest.mark.parametrize("shape", [(48, 96), (96, 48), (64, 64), (5, 300)])
@pytest.mark.parametrize("steps", [1, 5])
def test_newton_schulz_is_the_spectral_map(shape, steps):
    R, C = shape
    U = synth.normal_f32(synth.stream_key(R * 1000 + C, STREAM_GRAD), 0, R * C, 1.0).reshape(R, C).astype(np.float64)
    eps = 1e-7
    X = oracle.newton_schulz(U, steps, eps)
    P, s, QT = np.linalg.svd(U, full_matrices=False)
    want = (P * _phi(s / (np.linalg.norm(U) + eps), steps)) @ QT
    assert X.shape == U.shape
    assert np.max(np.abs(X - want)) <= 1e-10 * max(1.0, np.max(np.abs(want)))


def test_five_steps_land_in_the_band():
    x = np.linspace(0.02, 1.0, 2000)
    y = _phi(x, 5)
    assert y.min() > 0.6 and y.max() < 1.25
    # the oracle's iteration does the same to a matrix with those singular values
    n = 64
    rng_q = synth.normal_f32(synth.stream_key(7, STREAM_GRAD), 0, 2 * n * n, 1.0).astype(np.float64)
    P, _ = np.linalg.qr(rng_q[:n * n].reshape(n, n))
    Q, _ = np.linalg.qr(rng_q[n * n:].reshape(n, n))
    s = np.linspace(0.02, 1.0, n)
    U = (P * s) @ Q.T
    X = oracle.newton_schulz(U * (np.linalg.norm(U) + 1e-7), 5, 1e-7)   # normalisation restores s
    sv = np.linalg.svd(X, compute_uv=False)
    assert sv.min() > 0.6 and sv.max() < 1.25


def test_momentum_of_a_constant_gradient():
    g = oracle.bf16_round(np.array([1e-3, -2.5e-4, 0.0, 7.0], np.float32))
    gf = (g.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    beta, gs = 0.95, 0.5
    mom = np.zeros(4, np.float32)
    for t in range(1, 31):
        U = oracle.muon_momentum(mom, g, beta, gs, nesterov=True)
        want = gf * gs * (1 - beta ** t) / (1 - beta)
        assert np.allclose(mom, want, rtol=t * 2e-7, atol=0)
        assert np.allclose(U, gf * gs + beta * want, rtol=t * 2e-7, atol=0)
    plain = np.zeros(4, np.float32)
    V = oracle.muon_momentum(plain, g, beta, gs, nesterov=False)
    assert np.array_equal(V, plain)


def test_shape_factor():
    assert oracle.muon_update_scale(4096, 14336) == 1.0
    assert oracle.muon_update_scale(14336, 4096) == pytest.approx(np.sqrt(14336 / 4096))
