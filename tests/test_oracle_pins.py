"""Pins for the fp64 CPU oracle (no GPU needed).

The pages print no worked numeric example for the attention, so the oracle is pinned
by (a) a hand-derived closed-form fixture (tests/golden/hand_example_t2.json), (b)
brute force on tiny inputs (the quadratic masked form, and exact integer arithmetic
in numpy), (c) textbook special cases (final state = phi(K)^T V as one GEMM; V = 1
gives the running sum of phi(k) of the normalised form; T = 1; gate = 0), and (d)
invariants (block size, packing, decode-after-prefill, causality, norm axis).

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
transposed state, read-before-update, a per-head instead of a head-concat norm, the
gate applied before the norm, a missing mask) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _silu_np(x):
    return x / (1.0 + np.exp(-x))


def _rand_inputs(seed, T, H, D, dtype="f32", scale=1.0, gate=True):
    q, k, v, g = synth.prefill_inputs(seed, T, H, D, dtype, scale, gate)
    return q, k, v, g


def _as_f64(a):
    if a.dtype == np.uint16:
        return synth.bf16_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


# --------------------------------------------------------------------------------------
# (a) hand-derived closed form
# --------------------------------------------------------------------------------------
def test_hand_example_closed_form():
    fx = json.load(open(os.path.join(GOLDEN, "hand_example_t2.json")))
    a32 = np.float32(math.log(3.0))
    a = float(a32)
    q = (np.array(fx["q_coef"], np.float32) * a32).reshape(1, 2, 1, 2)
    k = (np.array(fx["k_coef"], np.float32) * a32).reshape(1, 2, 1, 2)
    v = np.array(fx["v"], np.float32).reshape(1, 2, 1, 2)
    g = (np.array(fx["g_coef"], np.float32) * a32).reshape(1, 2, 2)
    y, st, _ = oracle.prefill(q, k, v, None, mode=oracle.MODE_RAW)
    exp_y = np.array(fx["y_raw_coef_a2"]) * a * a
    np.testing.assert_allclose(y[0], exp_y, rtol=1e-6)
    np.testing.assert_allclose(st[0, 0], np.array(fx["state_coef_a"]) * a, rtol=1e-6, atol=1e-7)
    o, _, _ = oracle.prefill(q, k, v, g, mode=oracle.MODE_RMSNORM_GATE, eps=fx["eps"])
    r = 1.0 / np.sqrt((exp_y ** 2).mean(axis=1, keepdims=True) + fx["eps"])
    exp_o = exp_y * r * np.array(fx["gate_sigmoid"])
    np.testing.assert_allclose(o[0], exp_o, rtol=1e-6)


def test_silu_closed_form_values():
    # T = 1: y = (phi(q) . phi(k)) v.  With q = k = [x] (D = 1): y = SiLU(x)^2 v.
    for x, s in [(math.log(3.0), 0.75), (-math.log(3.0), 0.25), (math.log(7.0), 0.875), (0.0, 0.5)]:
        x32 = float(np.float32(x))
        q = np.array([[[[x32]]]], np.float32)
        y, _, _ = oracle.prefill(q, q, np.ones_like(q), None, mode=oracle.MODE_RAW)
        assert y[0, 0, 0] == pytest.approx((x * s) ** 2, rel=2e-6, abs=1e-30)
    # identity feature map leaves values untouched
    q = np.array([[[[3.0]]]], np.float32)
    y, _, _ = oracle.prefill(q, q, q, None, phi=oracle.PHI_IDENTITY, mode=oracle.MODE_RAW)
    assert y[0, 0, 0] == 27.0


# --------------------------------------------------------------------------------------
# (b) brute force
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_recurrence_equals_quadratic_tiny_config(dtype):
    # The tiny workload itself: B1 H2 T512 D64, fp32, N(0,1).
    w = synth.WORKLOADS["tiny_f32"]
    q, k, v, _ = _rand_inputs(w.seed, w.T, w.H, w.D, dtype, w.qkv_scale, gate=False)
    y_rec, _, _ = oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RAW)
    y_quad = oracle.quadratic(q, k, v)
    ref = y_quad.reshape(w.T, -1)
    err = np.abs(y_rec[0] - ref).max() / np.abs(ref).max()
    assert err < 1e-12


def test_integer_brute_force_numpy():
    # phi = identity on sparse ternary inputs: every quantity is an exact integer, so the
    # oracle must equal integer numpy: Y = (Q K^T (.) tril) V, S_T = K^T V.
    T, H, D = 200, 3, 16
    q = synth.ternary(11, 0, (T, H, D), 0.3, "f32")
    k = synth.ternary(11, 1, (T, H, D), 0.3, "f32")
    v = synth.ternary(11, 2, (T, H, D), 0.3, "f32")
    y, st, _ = oracle.prefill(q[None], k[None], v[None], None, phi=oracle.PHI_IDENTITY, mode=oracle.MODE_RAW)
    qi, ki, vi = (a.astype(np.int64) for a in (q, k, v))
    tril = np.tril(np.ones((T, T), np.int64))
    for h in range(H):
        P = (qi[:, h] @ ki[:, h].T) * tril
        Y = P @ vi[:, h]
        np.testing.assert_array_equal(y[0].reshape(T, H, D)[:, h], Y)
        np.testing.assert_array_equal(st[0, h], ki[:, h].T @ vi[:, h])


# --------------------------------------------------------------------------------------
# (c) special cases
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_final_state_is_one_gemm(dtype):
    T, H, D = 777, 4, 32
    q, k, v, _ = _rand_inputs(21, T, H, D, dtype, 0.5, gate=False)
    _, st, _ = oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RAW)
    kf, vf = _as_f64(k), _as_f64(v)
    for h in range(H):
        S = _silu_np(kf[:, h]).T @ vf[:, h]
        np.testing.assert_allclose(st[0, h], S, rtol=1e-11, atol=1e-11)


def test_state_in_adds_phiq_times_s0():
    # With an initial state S0 the output gains exactly phi(q_t)^T S0 for every t.
    T, H, D = 50, 2, 8
    q, k, v, _ = _rand_inputs(31, T, H, D, "f32", 1.0, gate=False)
    s0 = synth.normal(31, 9, (1, H, D, D), 1.0, "f32")
    y0, st0, _ = oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RAW)
    y1, st1, _ = oracle.prefill(q[None], k[None], v[None], None, state_in=s0, mode=oracle.MODE_RAW)
    fq = _silu_np(q.astype(np.float64))
    for h in range(H):
        extra = fq[:, h] @ s0[0, h].astype(np.float64)
        np.testing.assert_allclose(y1[0].reshape(T, H, D)[:, h] - y0[0].reshape(T, H, D)[:, h], extra,
                                   rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(st1 - st0, s0.astype(np.float64), rtol=1e-12, atol=1e-12)


def test_v_ones_gives_running_sum_of_phik():
    # V = 1: y_t[j] = phi(q_t) . sum_{i<=t} phi(k_i) for every j -- the numerator of the
    # normalised form with the running sum z_t ("六十四：MiniMax-01", section 3).
    T, H, D = 64, 2, 16
    q, k, _, _ = _rand_inputs(41, T, H, D, "f32", 1.0, gate=False)
    v = np.ones_like(q)
    y, _, _ = oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RAW)
    fq, fk = _silu_np(q.astype(np.float64)), _silu_np(k.astype(np.float64))
    z = np.cumsum(fk, axis=0)
    expect = np.einsum("thd,thd->th", fq, z)
    got = y[0].reshape(T, H, D)
    for j in range(D):
        np.testing.assert_allclose(got[:, :, j], expect, rtol=1e-12)


def test_t1_closed_form():
    H, D = 3, 8
    q, k, v, _ = _rand_inputs(51, 1, H, D, "f32", 1.0, gate=False)
    y, _, _ = oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RAW)
    fq, fk = _silu_np(q[0].astype(np.float64)), _silu_np(k[0].astype(np.float64))
    expect = (fq * fk).sum(axis=1, keepdims=True) * v[0].astype(np.float64)
    np.testing.assert_allclose(y[0, 0].reshape(H, D), expect, rtol=1e-12)


def test_gate_zero_is_half_of_rmsnorm():
    T, H, D = 20, 4, 8
    q, k, v, _ = _rand_inputs(61, T, H, D, "f32", 1.0, gate=False)
    g = np.zeros((T, H * D), np.float32)
    o_gate, _, _ = oracle.prefill(q[None], k[None], v[None], g[None], mode=oracle.MODE_RMSNORM_GATE)
    o_norm, _, _ = oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RMSNORM)
    np.testing.assert_array_equal(o_gate, 0.5 * o_norm)


def test_rmsnorm_constant_vector_and_weight():
    y = np.full((3, 2, 4), 2.0)
    o = oracle.transform(y, oracle.MODE_RMSNORM, eps=1e-6)
    np.testing.assert_allclose(o, 2.0 / math.sqrt(4.0 + 1e-6), rtol=1e-15)
    w = np.linspace(0.5, 2.0, 8).astype(np.float32)
    ow = oracle.transform(y, oracle.MODE_RMSNORM, eps=1e-6, norm_weight=w)
    np.testing.assert_allclose(ow, o * w.astype(np.float64), rtol=1e-15)
    # eps sits inside the square root: y = 0 gives 0, not NaN
    assert np.all(oracle.transform(np.zeros((1, 1, 4)), oracle.MODE_RMSNORM) == 0)


# --------------------------------------------------------------------------------------
# (d) invariants
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("C", [1, 7, 32, 64, 256, 600])
def test_chunked_equals_recurrence_any_block(C):
    T, H, D = 513, 2, 16
    q, k, v, _ = _rand_inputs(71, T, H, D, "bf16", 0.5, gate=False)
    s0 = synth.normal(71, 9, (H, D, D), 0.2, "f32").astype(np.float64)
    y_rec, st_rec, _ = oracle.prefill(q[None], k[None], v[None], None, state_in=s0[None].astype(np.float32),
                                      mode=oracle.MODE_RAW)
    y_chk, st_chk = oracle.chunked(q, k, v, C, s0=s0.astype(np.float32).astype(np.float64))
    scale = np.abs(y_rec).max()
    assert np.abs(y_chk.reshape(T, -1) - y_rec[0]).max() <= 1e-12 * scale
    np.testing.assert_allclose(st_chk, st_rec[0], rtol=1e-12, atol=1e-12 * np.abs(st_rec).max())


def test_chunked_block_ge_T_is_quadratic():
    T, H, D = 96, 2, 16
    q, k, v, _ = _rand_inputs(72, T, H, D, "f32", 1.0, gate=False)
    y_chk, _ = oracle.chunked(q, k, v, 4096)
    y_quad = oracle.quadratic(q, k, v)
    np.testing.assert_allclose(y_chk, y_quad, rtol=1e-12, atol=1e-12 * np.abs(y_quad).max())


def test_decode_after_prefill_equals_prefill_t_plus_1():
    T, H, D = 300, 4, 16
    q, k, v, g = _rand_inputs(81, T + 1, H, D, "bf16", 0.5, gate=True)
    o_full, st_full, _ = oracle.prefill(q[None], k[None], v[None], g[None])
    _, st_T, _ = oracle.prefill(q[None, :T], k[None, :T], v[None, :T], g[None, :T])
    o_dec, st_dec, _ = oracle.decode(q[T:], k[T:], v[T:], g[T:], st_T.astype(np.float32))
    # the prefill state is rounded to fp32 before the decode step reads it
    np.testing.assert_allclose(o_dec[0], o_full[0, T], rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(st_dec, st_full, rtol=1e-6, atol=1e-6)


def test_varlen_equals_separate_calls_and_state_reset():
    H, D = 2, 16
    lens = [5, 0, 130, 1, 64]
    cu = synth.cu_seqlens_of(lens)
    tot = int(cu[-1])
    q, k, v, g = _rand_inputs(91, tot, H, D, "bf16", 0.5, gate=True)
    o_pk, st_pk, _ = oracle.forward_packed(q, k, v, g, cu, H, D)
    for s, L in enumerate(lens):
        a, b = cu[s], cu[s + 1]
        o_s, st_s, _ = oracle.prefill(q[None, a:b], k[None, a:b], v[None, a:b], g[None, a:b])
        np.testing.assert_array_equal(o_pk[a:b], o_s[0])
        np.testing.assert_array_equal(st_pk[s], st_s[0])
    assert np.all(st_pk[1] == 0)  # empty sequence: state stays the initial (zero) state


def test_zero_padding_rows_change_nothing():
    # A K/V row of zeros (a padded tail row) adds nothing to the state; its own output row
    # is whatever phi(q) reads from the state, and no other row sees it.
    T, H, D = 40, 2, 8
    q, k, v, _ = _rand_inputs(95, T, H, D, "f32", 1.0, gate=False)
    kp = np.concatenate([k, np.zeros((24, H, D), np.float32)])
    vp = np.concatenate([v, np.zeros((24, H, D), np.float32)])
    qp = np.concatenate([q, synth.normal(95, 7, (24, H, D), 1.0, "f32")])
    y, st, _ = oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RAW)
    yp, stp, _ = oracle.prefill(qp[None], kp[None], vp[None], None, mode=oracle.MODE_RAW)
    np.testing.assert_array_equal(yp[0, :T], y[0])
    np.testing.assert_array_equal(stp, st)


def test_causality():
    T, H, D = 64, 2, 8
    q, k, v, g = _rand_inputs(97, T, H, D, "f32", 1.0, gate=True)
    o, _, _ = oracle.prefill(q[None], k[None], v[None], g[None])
    k2, v2 = k.copy(), v.copy()
    k2[40:] += 1.0
    v2[40:] -= 2.0
    o2, _, _ = oracle.prefill(q[None], k2[None], v2[None], g[None])
    np.testing.assert_array_equal(o[0, :40], o2[0, :40])
    assert np.abs(o[0, 40:] - o2[0, 40:]).max() > 1e-3


def test_norm_axis_is_head_concat():
    T, H, D = 16, 4, 8
    q, k, v, g = _rand_inputs(99, T, H, D, "f32", 1.0, gate=True)
    o, _, _ = oracle.prefill(q[None], k[None], v[None], g[None])
    v1 = v.copy()
    v1[:, 0] *= 3.0  # scale head 0 only
    o1, _, _ = oracle.prefill(q[None], k[None], v1[None], g[None])
    o, o1 = o[0].reshape(T, H, D), o1[0].reshape(T, H, D)
    # a head-concat norm rescales the other heads too (a per-head norm would not)
    assert np.abs(o1[:, 1:] - o[:, 1:]).max() > 1e-3
    ratio = o1[:, 1:] / o[:, 1:]
    np.testing.assert_allclose(ratio, np.broadcast_to(ratio[:, :1, :1], ratio.shape), rtol=1e-9)
    # scaling every head's V by c > 0 leaves the normalised output unchanged (up to eps)
    o2, _, _ = oracle.prefill(q[None], k[None], (v * 5.0)[None], g[None])
    np.testing.assert_allclose(o2[0].reshape(T, H, D), o, rtol=1e-5)


def test_streaming_compare_matches_stored_result():
    T, H, D = 300, 4, 16
    q, k, v, g = _rand_inputs(101, T, H, D, "bf16", 0.5, gate=True)
    o, st, _ = oracle.prefill(q[None], k[None], v[None], g[None])
    cand = synth.f32_to_bf16(o.astype(np.float32))
    cand_st = st.astype(np.float32)
    cand[0, 17, 5] ^= 0x0040  # perturb one element
    _, _, stats = oracle.prefill(q[None], k[None], v[None], g[None], store=False, cand_out=cand,
                                 cand_state=cand_st)
    assert stats["out_argmax"] == 17 * H * D + 5
    assert stats["out_max_ref"] == pytest.approx(np.abs(o).max(), rel=1e-15)
    assert stats["state_max_err"] <= np.abs(st).max() * 2 ** -24
    assert stats["out_nonfinite"] == 0
