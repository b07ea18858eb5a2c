"""Pins for the oracle's backward pass (no GPU needed).

The pages print no gradient formulas, so the backward is pinned to the forward it
differentiates: (a) central finite differences of ``oracle.forward_packed`` along a
random direction, one input at a time (q, k, v, gate, initial state), in every output
mode and both feature maps, over packed sequences that include an empty and a one-token
sequence; a wrong term, sign, index or a gradient routed to the wrong input fails its own
check.  (b) The masked-matrix form of the same gradients on a tiny case (dA = dY V^T (.) M,
dphi(Q) = dA phi(K) + dY S0^T, dphi(K) = dA^T phi(Q), dV = A^T dY, dS0 = phi(Q)^T dY),
which pins inclusive versus exclusive sums independently of the recurrences.
"""
import numpy as np
import pytest

import oracle
import synth

CU = np.array([0, 11, 11, 12, 29], dtype=np.int32)   # lengths 11, 0, 1, 17
H, D = 2, 8


def _inputs(seed, mode):
    n = int(CU[-1])
    q, k, v, g = synth.prefill_inputs(seed, n, H, D, "f32", 0.7, True)
    dout = synth.normal(seed, 11, (n, H * D), 1.0, "f32")
    s0 = synth.normal(seed, 12, (len(CU) - 1, H, D, D), 0.3, "f32")
    w = (1.0 + 0.25 * synth.normal(seed, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    if mode != oracle.MODE_RMSNORM_GATE:
        g = None
    return dict(q=q, k=k, v=v, g=g, state_in=s0), dout, w


def _loss(x, dout, phi, mode, w):
    out, _, _ = oracle.forward_packed(x["q"], x["k"], x["v"], x["g"], CU, H, D, state_in=x["state_in"], phi=phi,
                                      mode=mode, norm_weight=w)
    return float(np.sum(out * dout.astype(np.float64)))


@pytest.mark.parametrize("phi", [oracle.PHI_SILU, oracle.PHI_IDENTITY])
@pytest.mark.parametrize("mode", [oracle.MODE_RAW, oracle.MODE_RMSNORM, oracle.MODE_RMSNORM_GATE])
def test_backward_matches_finite_differences(phi, mode):
    x, dout, w = _inputs(2101 + 7 * mode + phi, mode)
    dq, dk, dv, dg, dst, dw = oracle.backward_packed(x["q"], x["k"], x["v"], x["g"], dout, CU, H, D,
                                                     state_in=x["state_in"], phi=phi, mode=mode, norm_weight=w)
    grads = {"q": dq, "k": dk, "v": dv, "state_in": dst}
    if mode == oracle.MODE_RMSNORM_GATE:
        grads["g"] = dg
    else:
        assert dg is None
    rng = np.random.default_rng(2101 + mode)
    eps = 1e-3
    for name, grad in grads.items():
        base = x[name]
        delta = rng.standard_normal(base.shape)
        plus, minus = dict(x), dict(x)
        plus[name] = (base + eps * delta).astype(np.float32)
        minus[name] = (base - eps * delta).astype(np.float32)
        step = plus[name].astype(np.float64) - minus[name].astype(np.float64)   # the step actually taken
        fd = _loss(plus, dout, phi, mode, w) - _loss(minus, dout, phi, mode, w)
        pred = float(np.sum(grad.reshape(step.shape) * step))
        scale = float(np.sum(np.abs(grad.reshape(step.shape) * step)))
        assert abs(fd - pred) <= 1e-5 * scale, f"{name}: finite difference {fd:.9e} vs gradient {pred:.9e}"


def test_empty_sequence_gradient_of_state_is_zero_and_one_token_closed_form():
    """An empty sequence gets dS0 = 0; a one-token raw sequence has dv = (phi(q).phi(k)) dy,
    dphi(q) = S_1 dy, dphi(k) = (dy.v) phi(q), dS0 = phi(q) dy^T (hand-derived)."""
    x, dout, w = _inputs(2151, oracle.MODE_RAW)
    phi = oracle.PHI_IDENTITY
    dq, dk, dv, _, dst, _ = oracle.backward_packed(x["q"], x["k"], x["v"], None, dout, CU, H, D,
                                                state_in=x["state_in"], phi=phi, mode=oracle.MODE_RAW)
    assert np.all(dst[1] == 0.0)
    t = int(CU[2])                      # the one-token sequence is sequence 2
    for h in range(H):
        a = x["q"][t, h].astype(np.float64)
        b = x["k"][t, h].astype(np.float64)
        vv = x["v"][t, h].astype(np.float64)
        dy = dout[t, h * D:(h + 1) * D].astype(np.float64)
        S1 = x["state_in"][2, h].astype(np.float64) + np.outer(b, vv)
        np.testing.assert_allclose(dv[t, h], (a @ b) * dy, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dq[t, h], S1 @ dy, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dk[t, h], (dy @ vv) * a, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dst[2, h], np.outer(a, dy), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("phi", [oracle.PHI_SILU, oracle.PHI_IDENTITY])
def test_backward_matches_masked_matrix_form(phi):
    T, Hh, Dd = 37, 3, 16
    q, k, v, _ = synth.prefill_inputs(2161, T, Hh, Dd, "f32", 0.7, False)
    dout = synth.normal(2161, 11, (T, Hh * Dd), 1.0, "f32")
    s0 = synth.normal(2161, 12, (1, Hh, Dd, Dd), 0.3, "f32")
    dq, dk, dv, _, dst, _ = oracle.backward_packed(q, k, v, None, dout, [0, T], Hh, Dd, state_in=s0, phi=phi,
                                                mode=oracle.MODE_RAW)
    f = (lambda z: z / (1.0 + np.exp(-z))) if phi == oracle.PHI_SILU else (lambda z: z)
    df = (lambda z: (1 / (1 + np.exp(-z))) * (1 + z * (1 - 1 / (1 + np.exp(-z))))) if phi == oracle.PHI_SILU \
        else (lambda z: np.ones_like(z))
    M = np.tril(np.ones((T, T)))
    for h in range(Hh):
        Q, K, V = (a[:, h].astype(np.float64) for a in (q, k, v))
        dY = dout[:, h * Dd:(h + 1) * Dd].astype(np.float64)
        S0 = s0[0, h].astype(np.float64)
        A = (f(Q) @ f(K).T) * M
        dA = (dY @ V.T) * M
        np.testing.assert_allclose(dq[:, h], (dA @ f(K) + dY @ S0.T) * df(Q), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dk[:, h], (dA.T @ f(Q)) * df(K), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dv[:, h], A.T @ dY, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dst[0, h], f(Q).T @ dY, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("mode", [oracle.MODE_RAW, oracle.MODE_RMSNORM_GATE])
def test_final_state_gradient_matches_finite_differences(mode):
    """With a gradient dS_T reaching each sequence's final state, the loss is
    sum(dout * o) + sum(dS_T * S_T); its finite differences pin the reverse sum's start."""
    x, dout, w = _inputs(2171 + mode, mode)
    dST = synth.normal(2171, 14, (len(CU) - 1, H, D, D), 0.5, "f32")
    phi = oracle.PHI_SILU

    def loss(xx):
        out, st, _ = oracle.forward_packed(xx["q"], xx["k"], xx["v"], xx["g"], CU, H, D, state_in=xx["state_in"],
                                           phi=phi, mode=mode, norm_weight=w)
        return float(np.sum(out * dout.astype(np.float64)) + np.sum(st * dST.astype(np.float64)))

    dq, dk, dv, dg, dst, _ = oracle.backward_packed(x["q"], x["k"], x["v"], x["g"], dout, CU, H, D,
                                                    state_in=x["state_in"], phi=phi, mode=mode, norm_weight=w,
                                                    dstate_out=dST)
    grads = {"q": dq, "k": dk, "v": dv, "state_in": dst}
    rng = np.random.default_rng(2171)
    eps = 1e-3
    for name, grad in grads.items():
        base = x[name]
        delta = rng.standard_normal(base.shape)
        plus, minus = dict(x), dict(x)
        plus[name] = (base + eps * delta).astype(np.float32)
        minus[name] = (base - eps * delta).astype(np.float32)
        step = plus[name].astype(np.float64) - minus[name].astype(np.float64)
        fd = loss(plus) - loss(minus)
        pred = float(np.sum(grad.reshape(step.shape) * step))
        scale = float(np.sum(np.abs(grad.reshape(step.shape) * step)))
        assert abs(fd - pred) <= 1e-5 * scale, f"{name}: finite difference {fd:.9e} vs gradient {pred:.9e}"


@pytest.mark.parametrize("mode", [oracle.MODE_RMSNORM, oracle.MODE_RMSNORM_GATE])
def test_norm_weight_gradient_matches_finite_differences(mode):
    """dw (the RMSNorm weight's gradient, summed over tokens) against central differences
    of the forward in w; zero in raw mode."""
    x, dout, w = _inputs(2181 + mode, mode)
    *_, dw = oracle.backward_packed(x["q"], x["k"], x["v"], x["g"], dout, CU, H, D, state_in=x["state_in"],
                                    mode=mode, norm_weight=w)
    rng = np.random.default_rng(2181)
    delta = rng.standard_normal(w.shape)
    eps = 1e-3
    wp, wm = (w + eps * delta).astype(np.float32), (w - eps * delta).astype(np.float32)
    step = wp.astype(np.float64) - wm.astype(np.float64)
    fd = _loss(x, dout, oracle.PHI_SILU, mode, wp) - _loss(x, dout, oracle.PHI_SILU, mode, wm)
    pred = float(np.sum(dw * step))
    assert abs(fd - pred) <= 1e-5 * float(np.sum(np.abs(dw * step))), (fd, pred)
    *_, dw_raw = oracle.backward_packed(x["q"], x["k"], x["v"], None, dout, CU, H, D, mode=oracle.MODE_RAW)
    assert np.all(dw_raw == 0.0)


@pytest.mark.parametrize("mode", [oracle.MODE_RAW, oracle.MODE_RMSNORM, oracle.MODE_RMSNORM_GATE])
def test_transform_backward_matches_finite_differences(mode):
    """oracle.transform_backward (the output transform's backward alone) against central
    differences of oracle.transform in y, in the gate and in the norm weight, each along a
    random direction; in raw mode dy = dout and dw = 0."""
    tokens = 7
    rng = np.random.default_rng(2191 + mode)
    y = rng.standard_normal((tokens, H, D))
    g = synth.normal(2191, 3, (tokens, H * D), 1.0, "f32") if mode == oracle.MODE_RMSNORM_GATE else None
    w = (1.0 + 0.25 * synth.normal(2191, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    dout = synth.normal(2191, 11, (tokens, H * D), 1.0, "f32")
    dy, dg, dw = oracle.transform_backward(y, dout, mode, norm_weight=w, g=g)
    loss = lambda yy, gg, ww: float(np.sum(oracle.transform(yy, mode, norm_weight=ww, g=gg) * dout.astype(np.float64)))
    e = 1e-4
    d = rng.standard_normal(y.shape)
    fd = (loss(y + e * d, g, w) - loss(y - e * d, g, w)) / (2 * e)
    pred = float(np.sum(dy * d.reshape(tokens, H * D)))
    assert abs(fd - pred) <= 1e-7 * float(np.sum(np.abs(dy * d.reshape(tokens, H * D)))), ("y", fd, pred)
    if mode == oracle.MODE_RAW:
        np.testing.assert_array_equal(dy, dout.astype(np.float64))
        assert np.all(dw == 0.0) and dg is None
        return
    dlt = rng.standard_normal(w.shape)
    wp, wm = (w + 1e-3 * dlt).astype(np.float32), (w - 1e-3 * dlt).astype(np.float32)
    step = wp.astype(np.float64) - wm.astype(np.float64)
    fd = loss(y, g, wp) - loss(y, g, wm)
    pred = float(np.sum(dw * step))
    assert abs(fd - pred) <= 1e-5 * float(np.sum(np.abs(dw * step))), ("w", fd, pred)
    if mode == oracle.MODE_RMSNORM_GATE:
        dlt = rng.standard_normal(g.shape)
        gp, gm = (g + 1e-3 * dlt).astype(np.float32), (g - 1e-3 * dlt).astype(np.float32)
        step = gp.astype(np.float64) - gm.astype(np.float64)
        fd = loss(y, gp, w) - loss(y, gm, w)
        pred = float(np.sum(dg * step))
        assert abs(fd - pred) <= 1e-5 * float(np.sum(np.abs(dg * step))), ("g", fd, pred)
