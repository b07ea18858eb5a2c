"""Pins for the oracle's backward of the normalised variant (no GPU needed).

The pages print no gradients; the backward is pinned to the forward it differentiates:
central finite differences of ``oracle.forward_znorm_packed`` along a random direction, one
input at a time (q, k, v, gate, initial S, initial z, norm weight), for the loss
sum(out * dout) + sum(S_T * dS_T) + sum(z_T * dz_T), in the raw and gated modes and both
feature maps, over packed sequences with an empty and a one-token one.  A dropped term of
the denominator's gradient, an exclusive z, a wrong sign or the numerator's gradient not
divided by the denominator each fails its own check.  Inputs are shifted so that the
denominators stay away from zero.  Closed forms: an empty sequence passes dS_T and dz_T
through to its initial state; from zero initial states with V = 1 the raw output is
identically 1, so no gradient reaches q or k.
"""
import numpy as np
import pytest

import oracle
import synth

CU = np.array([0, 9, 9, 10, 24], dtype=np.int32)   # lengths 9, 0, 1, 14
H, D = 2, 8


def _inputs(seed, mode, phi):
    n = int(CU[-1])
    shift = 1.0 if phi == oracle.PHI_SILU else 2.0
    q, k, v, g = synth.prefill_inputs(seed, n, H, D, "f32", 0.5, True)
    q, k = (q + shift).astype(np.float32), (k + shift).astype(np.float32)
    N = len(CU) - 1
    s0 = np.abs(synth.normal(seed, 12, (N, H, D, D), 0.3, "f32"))
    z0 = np.abs(synth.normal(seed, 15, (N, H, D), 1.0, "f32"))
    w = (1.0 + 0.25 * synth.normal(seed, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    dout = synth.normal(seed, 11, (n, H * D), 1.0, "f32")
    dsT = synth.normal(seed, 16, (N, H, D, D), 0.3, "f32")
    dzT = synth.normal(seed, 17, (N, H, D), 0.3, "f32")
    if mode != oracle.MODE_RMSNORM_GATE:
        g = None
    return dict(q=q, k=k, v=v, g=g, state_in=s0, z_in=z0, w=w), dout, dsT, dzT


def _loss(x, dout, dsT, dzT, phi, mode):
    out, st, z = oracle.forward_znorm_packed(x["q"], x["k"], x["v"], x["g"], CU, H, D, state_in=x["state_in"],
                                             z_in=x["z_in"], phi=phi, mode=mode, norm_weight=x["w"])
    return float(np.sum(out * dout.astype(np.float64)) + np.sum(st * dsT.astype(np.float64)) +
                 np.sum(z * dzT.astype(np.float64)))


@pytest.mark.parametrize("phi", [oracle.PHI_SILU, oracle.PHI_IDENTITY])
@pytest.mark.parametrize("mode", [oracle.MODE_RAW, oracle.MODE_RMSNORM_GATE])
def test_znorm_backward_matches_finite_differences(phi, mode):
    x, dout, dsT, dzT = _inputs(2301 + 10 * phi + mode, mode, phi)
    dq, dk, dv, dg, dst, dz, dw = oracle.backward_znorm_packed(
        x["q"], x["k"], x["v"], x["g"], dout, CU, H, D, state_in=x["state_in"], z_in=x["z_in"], phi=phi, mode=mode,
        norm_weight=x["w"], dstate_out=dsT, dz_out=dzT)
    grads = dict(q=dq, k=dk, v=dv, g=dg, state_in=dst, z_in=dz, w=dw if mode != oracle.MODE_RAW else None)
    rng = np.random.default_rng(2301)
    for name, grad in grads.items():
        if x[name] is None or grad is None:
            continue
        delta = rng.standard_normal(x[name].shape)
        e = 1e-3
        xp, xm = dict(x), dict(x)
        xp[name] = (x[name] + e * delta).astype(np.float32)
        xm[name] = (x[name] - e * delta).astype(np.float32)
        step = xp[name].astype(np.float64) - xm[name].astype(np.float64)   # the fp32-rounded step
        fd = _loss(xp, dout, dsT, dzT, phi, mode) - _loss(xm, dout, dsT, dzT, phi, mode)
        pred = float(np.sum(grad * step))
        scale = float(np.sum(np.abs(grad * step)))
        assert abs(fd - pred) <= 2e-5 * scale, (name, fd, pred, scale)


def test_empty_sequence_passes_final_gradients_through_and_ones_value_gives_q_k_no_gradient():
    x, dout, dsT, dzT = _inputs(2311, oracle.MODE_RAW, oracle.PHI_SILU)
    v1 = np.ones_like(x["v"])
    dq, dk, dv, _, dst, dz, _ = oracle.backward_znorm_packed(
        x["q"], x["k"], v1, None, dout, CU, H, D, mode=oracle.MODE_RAW)
    # from S0 = 0 and z0 = 0 with V = 1 the numerator equals the denominator in every column,
    # so y = 1 whatever q and k are: no gradient reaches them, while v's does
    np.testing.assert_allclose(dq, 0.0, atol=1e-10)
    np.testing.assert_allclose(dk, 0.0, atol=1e-10)
    assert np.abs(dv).max() > 1e-3
    # the empty sequence (index 1): its initial-state gradients are the final ones
    _, _, _, _, dst, dz, _ = oracle.backward_znorm_packed(
        x["q"], x["k"], x["v"], None, dout, CU, H, D, state_in=x["state_in"], z_in=x["z_in"], mode=oracle.MODE_RAW,
        dstate_out=dsT, dz_out=dzT)
    np.testing.assert_array_equal(dst[1], dsT[1].astype(np.float64))
    np.testing.assert_array_equal(dz[1], dzT[1].astype(np.float64))
