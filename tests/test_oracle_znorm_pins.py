"""Pins for the oracle's normalised variant, y = phi(q)^T S / (phi(q) . z) ("六十四：MiniMax-01",
section 3), with no GPU.

(a) V = 1 gives y = 1 exactly: the numerator is (phi(q) . z) times a row of ones.
(b) The masked-matrix form: y = (A V + phi(Q) S0) / (A 1 + phi(Q) z0), A = phi(Q) phi(K)^T (.) M.
(c) One token from a zero state: y = v.
(d) Continuation: a sequence split in two, the second half started from the first half's
    (S, z), equals the whole sequence; S equals the plain form's state; z = z0 + sum phi(k).
(e) The norm and gate are the plain output transform applied to the raw normalised y.
Inputs are shifted to positive values so the denominators stay away from zero.
"""
import numpy as np
import pytest

import oracle
import synth


def _inputs(seed, T, H, D, shift=1.0):
    q, k, v, g = synth.prefill_inputs(seed, T, H, D, "f32", 0.5, True)
    return (q + shift).astype(np.float32), (k + shift).astype(np.float32), v, g


def _f(x, phi):
    return x / (1.0 + np.exp(-x)) if phi == oracle.PHI_SILU else x


@pytest.mark.parametrize("phi", [oracle.PHI_SILU, oracle.PHI_IDENTITY])
def test_ones_value_gives_ones(phi):
    q, k, _, _ = _inputs(2201, 50, 2, 16)
    v = np.ones_like(q)
    out, _, _ = oracle.forward_znorm_packed(q, k, v, None, [0, 20, 50], 2, 16, phi=phi, mode=oracle.MODE_RAW)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("phi", [oracle.PHI_SILU, oracle.PHI_IDENTITY])
def test_masked_matrix_form_with_initial_state(phi):
    T, H, D = 41, 3, 16
    q, k, v, _ = _inputs(2211, T, H, D)
    s0 = np.abs(synth.normal(2211, 12, (1, H, D, D), 0.3, "f32"))
    z0 = np.abs(synth.normal(2211, 13, (1, H, D), 1.0, "f32"))
    out, _, _ = oracle.forward_znorm_packed(q, k, v, None, [0, T], H, D, state_in=s0, z_in=z0, phi=phi,
                                            mode=oracle.MODE_RAW)
    M = np.tril(np.ones((T, T)))
    for h in range(H):
        Q, K, V = (_f(a[:, h].astype(np.float64), p) for a, p in ((q, phi), (k, phi), (v, oracle.PHI_IDENTITY)))
        A = (Q @ K.T) * M
        num = A @ V + Q @ s0[0, h].astype(np.float64)
        den = A.sum(axis=1) + Q @ z0[0, h].astype(np.float64)
        np.testing.assert_allclose(out[:, h * D:(h + 1) * D], num / den[:, None], rtol=1e-10, atol=1e-12)


def test_one_token_from_zero_state_returns_v():
    q, k, v, _ = _inputs(2221, 1, 4, 32)
    out, _, _ = oracle.forward_znorm_packed(q, k, v, None, [0, 1], 4, 32, mode=oracle.MODE_RAW)
    np.testing.assert_allclose(out.reshape(1, 4, 32), v.astype(np.float64), rtol=1e-12, atol=0)


def test_continuation_state_and_z():
    T, H, D, cut = 60, 2, 16, 23
    q, k, v, g = _inputs(2231, T, H, D)
    whole, S, z = oracle.forward_znorm_packed(q, k, v, g, [0, T], H, D)
    a, Sa, za = oracle.forward_znorm_packed(q[:cut], k[:cut], v[:cut], g[:cut], [0, cut], H, D)
    b, Sb, zb = oracle.forward_znorm_packed(q[cut:], k[cut:], v[cut:], g[cut:], [0, T - cut], H, D,
                                            state_in=Sa.astype(np.float32), z_in=za.astype(np.float32))
    np.testing.assert_allclose(np.concatenate([a, b]), whole, rtol=1e-6, atol=1e-6 * np.abs(whole).max())
    _, S_plain, _ = oracle.forward_packed(q, k, v, g, [0, T], H, D)
    np.testing.assert_allclose(S, S_plain, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z[0], _f(k.astype(np.float64), oracle.PHI_SILU).sum(axis=0), rtol=1e-12)


def test_output_transform_is_the_plain_one():
    T, H, D = 30, 2, 16
    q, k, v, g = _inputs(2241, T, H, D)
    raw, _, _ = oracle.forward_znorm_packed(q, k, v, None, [0, T], H, D, mode=oracle.MODE_RAW)
    gated, _, _ = oracle.forward_znorm_packed(q, k, v, g, [0, T], H, D, mode=oracle.MODE_RMSNORM_GATE)
    np.testing.assert_allclose(gated, oracle.transform(raw.reshape(T, H, D), oracle.MODE_RMSNORM_GATE, g=g),
                               rtol=1e-12, atol=1e-14)
