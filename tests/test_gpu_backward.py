"""GPU parity of the backward pass against the oracle's fp64 gradients.

Every gradient (dq, dk, dv, the gate's dg, the initial state's dS0 and the norm weight's dw)
is compared element by element with the oracle (which finite differences of the forward pin) at the forward's
tolerance: bf16 2e-2 * max|ref|, fp32 1e-4 * max|ref|.  Cases span several blocks with a
ragged tail, both tensor-core block sizes, the three output modes, a norm weight, initial
states, packed sequences with an empty and a one-token sequence, and the fp32 path.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import assert_close, mode_code, to_dev, to_host

pytestmark = pytest.mark.gpu


def _la():
    from long_context_attn_b200 import lightning_attn as la
    return la


def _run_fixed(B, T, H, D, C, dtype, mode, with_state, seed, expect=None, want_dw=True):
    """with_state: an initial state S0 and a final-state gradient dS_T as well; want_dw: ask
    for the norm weight's gradient (the norm/gate backward then runs its token-blocked
    kernel, else the one-CTA-per-token kernel)."""
    import torch
    la = _la()
    m = mode_code(mode)
    q, k, v, g = synth.prefill_inputs(seed, B * T, H, D, dtype, 0.5, True)
    dout = synth.normal(seed, 21, (B * T, H * D), 1.0, dtype)
    s0 = synth.normal(seed, 22, (B, H, D, D), 0.05, "f32") if with_state else None
    dsT = synth.normal(seed, 24, (B, H, D, D), 0.05, "f32") if with_state else None
    w = (1.0 + 0.2 * synth.normal(seed, 23, (H * D,), 1.0, "f32")).astype(np.float32) if m else None
    shp, gshp = (B, T, H, D), (B, T, H * D)
    dq_, dk_, dv_, dg_ = (to_dev(a).reshape(shp if i < 3 else gshp) for i, a in enumerate((q, k, v, g)))
    ddo = to_dev(dout).reshape(gshp)
    gq, gk, gv = (torch.full_like(dq_, float("nan")) for _ in range(3))
    gg = torch.full_like(dg_, float("nan")) if m == la.LA_OUT_RMSNORM_GATE else None
    gs = torch.full((B, H, D, D), float("nan"), dtype=torch.float32, device="cuda")
    gw = torch.full((H * D,), float("nan"), dtype=torch.float32, device="cuda") if want_dw else None
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, B, T, 0, H, D, C, la._dtype(dq_), m))
    la.lightning_attn_backward(dq_, dk_, dv_, dg_ if m == la.LA_OUT_RMSNORM_GATE else None, ddo, gq, gk, gv, dg=gg,
                               state_in=None if s0 is None else to_dev(s0), dstate_in=gs, block_size=C, mode=m,
                               norm_weight=None if w is None else to_dev(w), workspace=ws,
                               dstate_out=None if dsT is None else to_dev(dsT), dnorm_weight=gw)
    if expect:
        assert la.lightning_attn_last_path() == expect
    la.lightning_attn_check(ws)
    r = lambda a, s: a.reshape(s)
    ref = oracle.backward(r(q, shp), r(k, shp), r(v, shp), r(g, gshp) if m == la.LA_OUT_RMSNORM_GATE else None,
                          r(dout, gshp), state_in=s0, mode=m, norm_weight=w, dstate_out=dsT)
    assert_close(to_host(gq), ref[0], dtype, "dq")
    assert_close(to_host(gk), ref[1], dtype, "dk")
    assert_close(to_host(gv), ref[2], dtype, "dv")
    if gg is not None:
        assert_close(to_host(gg), ref[3], dtype, "dg")
    assert_close(to_host(gs), ref[4], dtype, "dstate")
    if gw is None:
        return
    if m == la.LA_OUT_RAW:
        assert torch.all(gw == 0), "dw must be zero in raw mode"
    else:
        assert_close(to_host(gw), ref[5], dtype, "dw")


@pytest.mark.parametrize("C", [128, 256])
@pytest.mark.parametrize("mode", ["raw", "rmsnorm", "rmsnorm_gate"])
def test_backward_tc_fixed(C, mode, cuda_device):
    _run_fixed(2, 700, 8, 128, C, "bf16", mode, True, 3001 + C, expect="tcgen05")


@pytest.mark.parametrize("T", [1, 33, 256, 1000])
def test_backward_tc_lengths(T, cuda_device):
    _run_fixed(1, T, 8, 128, 256, "bf16", "rmsnorm_gate", False, 3101 + T, expect="tcgen05", want_dw=T >= 256)


@pytest.mark.parametrize("H", [32, 64])
def test_backward_wide_rows_gated(H, cuda_device):
    """H * D = 4096 and 8192 without the norm weight's gradient: the norm/gate backward keeps
    each token's row in registers (one read of y, dout and g)."""
    _run_fixed(1, 300, H, 128, 256, "bf16", "rmsnorm_gate", True, 3601 + H, expect="tcgen05", want_dw=False)


def test_backward_fp32_path(cuda_device):
    _run_fixed(2, 150, 4, 64, 64, "f32", "rmsnorm_gate", True, 3201, expect="simt")


@pytest.mark.parametrize("C", [128, 256])
def test_backward_varlen(C, cuda_device):
    import torch
    la = _la()
    H, D = 8, 128
    lens = [300, 0, 257, 1, 31, 129]
    tot = sum(lens)
    cu = synth.cu_seqlens_of(lens)
    n = len(lens)
    q, k, v, g = synth.prefill_inputs(3301, tot, H, D, "bf16", 0.5, True)
    dout = synth.normal(3301, 21, (tot, H * D), 1.0, "bf16")
    s0 = synth.normal(3301, 22, (n, H, D, D), 0.05, "f32")
    dsT = synth.normal(3301, 24, (n, H, D, D), 0.05, "f32")
    dq_, dk_, dv_, dg_, ddo = (to_dev(a) for a in (q, k, v, g, dout))
    gq, gk, gv = (torch.full_like(dq_, float("nan")) for _ in range(3))
    gg = torch.full_like(dg_, float("nan"))
    gs = torch.full((n, H, D, D), float("nan"), dtype=torch.float32, device="cuda")
    gw = torch.full((H * D,), float("nan"), dtype=torch.float32, device="cuda")
    w = (1.0 + 0.2 * synth.normal(3301, 23, (H * D,), 1.0, "f32")).astype(np.float32)
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD_VARLEN, n, max(lens), tot, H, D, C,
                                                           la.LA_BF16, la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_backward_varlen(dq_, dk_, dv_, dg_, ddo, gq, gk, gv, torch.from_numpy(cu).cuda(), max(lens),
                                      dg=gg, state_in=to_dev(s0), dstate_in=gs, block_size=C, workspace=ws,
                                      dstate_out=to_dev(dsT), norm_weight=to_dev(w), dnorm_weight=gw)
    assert la.lightning_attn_last_path() == "tcgen05"
    la.lightning_attn_check(ws)
    ref = oracle.backward_packed(q, k, v, g, dout, cu, H, D, state_in=s0, dstate_out=dsT, norm_weight=w)
    for got, want, name in zip((gq, gk, gv, gg, gs, gw), ref, ("dq", "dk", "dv", "dg", "dstate", "dw")):
        assert_close(to_host(got), want, "bf16", name)


def test_backward_rejects_bad_arguments(cuda_device):
    import torch
    la = _la()
    B, T, H, D = 1, 64, 8, 128
    x = torch.zeros((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    gx = torch.zeros((B, T, H * D), dtype=torch.bfloat16, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, B, T, 0, H, D, 256, la.LA_BF16,
                                                           la.LA_OUT_RMSNORM_GATE))
    d = [torch.empty_like(x) for _ in range(3)]
    with pytest.raises(la.LightningAttnError):       # gate mode without dg
        la.lightning_attn_backward(x, x, x, gx, gx, *d, dg=None, workspace=ws)
    with pytest.raises(la.LightningAttnError):       # workspace too small
        la.lightning_attn_backward(x, x, x, gx, gx, *d, dg=torch.empty_like(gx), workspace=ws[:1024])


@pytest.mark.parametrize("C", [128, 256])
@pytest.mark.parametrize("T", [256, 700])
def test_backward_exact_integers(C, T, cuda_device):
    """Raw output, identity features, sparse ternary q, k, v, dout and an integer S0: every
    score, state entry and gradient is an integer of magnitude <= 256 (checked on the
    host), exact in bf16 and fp32, so the GPU gradients must equal the oracle's bit for bit
    (a wrong row of the reversal, a transposed state or a shifted mask shows as a mismatch)."""
    import torch
    la = _la()
    H, D = 4, 128
    q, k, v, dout = (synth.ternary(3501 + T, s, (T, H, D), 0.06, "bf16") for s in range(4))
    s0 = np.round(synth.normal(3501, 9, (1, H, D, D), 1.0, "f32")).astype(np.float32)
    dsT = np.round(synth.normal(3501, 10, (1, H, D, D), 1.0, "f32")).astype(np.float32)
    f = lambda a: synth.bf16_to_f32(a).astype(np.float64)
    Q, K, V, dY = f(q), f(k), f(v), f(dout)
    # every intermediate the three passes hold: running sums of v k^T (forward) and of
    # dy q^T, q dy^T (from the end), plus the forward state itself
    for a, b, rev in ((V, K, False), (dY, Q, True), (Q, dY, True), (K, V, False)):
        outer = np.einsum("thi,thj->thij", a, b)
        run = np.cumsum(outer[::-1] if rev else outer, axis=0)
        assert np.abs(run).max() + np.abs(s0).max() + np.abs(dsT).max() <= 256
    shp = (1, T, H, D)
    dq_, dk_, dv_ = (to_dev(a).reshape(shp) for a in (q, k, v))
    ddo = to_dev(dout).reshape(1, T, H * D)
    gq, gk, gv = (torch.full_like(dq_, float("nan")) for _ in range(3))
    gs = torch.full((1, H, D, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, 1, T, 0, H, D, C, la.LA_BF16,
                                                           la.LA_OUT_RAW))
    la.lightning_attn_backward(dq_, dk_, dv_, None, ddo, gq, gk, gv, state_in=to_dev(s0), dstate_in=gs,
                               block_size=C, phi=la.LA_PHI_IDENTITY, mode=la.LA_OUT_RAW, workspace=ws,
                               dstate_out=to_dev(dsT))
    assert la.lightning_attn_last_path() == "tcgen05"
    la.lightning_attn_check(ws)
    ref = oracle.backward(q.reshape(shp), k.reshape(shp), v.reshape(shp), None, dout.reshape(1, T, H * D),
                          state_in=s0, phi=oracle.PHI_IDENTITY, mode=oracle.MODE_RAW, dstate_out=dsT)
    for got, want, name in zip((gq, gk, gv, gs), (ref[0], ref[1], ref[2], ref[4]), ("dq", "dk", "dv", "dstate")):
        assert np.abs(want).max() <= 256, name
        g64 = synth.bf16_to_f32(to_host(got)).astype(np.float64) if got.dtype == torch.bfloat16 \
            else to_host(got).astype(np.float64)
        bad = np.argwhere(g64.reshape(want.shape) != want)
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first at {bad[:3].tolist()}"


@pytest.mark.slow
def test_backward_128k_full_size_samples(cuda_device):
    """The backward at the bench's full size (T 131072, H 64, D 128, block 256) in raw mode,
    where dy = dout needs no forward: dq of the first 4096 tokens depends only on them, and
    dk, dv of the last 4096 tokens only on those (sums over t >= i), so both samples are
    compared element by element with the oracle run on that prefix / suffix alone."""
    import torch
    la = _la()
    w = synth.WORKLOADS["backward_128k"]
    T, H, D, n = w.T, w.H, w.D, 4096
    q, k, v, _ = synth.prefill_inputs(w.seed, T, H, D, "bf16", w.qkv_scale, False)
    dout = synth.normal(w.seed, synth.STREAM_DOUT, (T, H * D), 1.0, "bf16")
    shp = (1, T, H, D)
    dq_, dk_, dv_ = (to_dev(a).reshape(shp) for a in (q, k, v))
    ddo = to_dev(dout).reshape(1, T, H * D)
    gq, gk, gv = (torch.empty_like(dq_) for _ in range(3))
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, 1, T, 0, H, D, w.block_size,
                                                           la.LA_BF16, la.LA_OUT_RAW))
    la.lightning_attn_backward(dq_, dk_, dv_, None, ddo, gq, gk, gv, block_size=w.block_size, mode=la.LA_OUT_RAW,
                               workspace=ws)
    # every pass (forward and reverse time) runs the 64 heads' sequence as two parallel chunks
    assert la.lightning_attn_last_path() == "tcgen05+chunks"
    la.lightning_attn_check(ws)
    got_q = to_host(gq[0, :n])
    got_k, got_v = to_host(gk[0, T - n:]), to_host(gv[0, T - n:])
    del gq, gk, gv, dq_, dk_, dv_, ddo, ws
    head = oracle.backward(q[None, :n], k[None, :n], v[None, :n], None, dout[None, :n], mode=oracle.MODE_RAW)
    assert_close(got_q[None], head[0], "bf16", "dq (first 4096 tokens)")
    tail = oracle.backward(q[None, T - n:], k[None, T - n:], v[None, T - n:], None, dout[None, T - n:],
                           mode=oracle.MODE_RAW)
    assert_close(got_k[None], tail[1], "bf16", "dk (last 4096 tokens)")
    assert_close(got_v[None], tail[2], "bf16", "dv (last 4096 tokens)")


@pytest.mark.parametrize("mode", ["rmsnorm", "rmsnorm_gate"])
def test_backward_with_saved_y_equals_recompute(mode, cuda_device):
    """Passing the forward's raw output y (prefill in raw mode) gives the same gradients as
    letting the backward recompute it (the same kernel computes y either way)."""
    import torch
    la = _la()
    m = mode_code(mode)
    B, T, H, D, C = 1, 600, 8, 128, 256
    q, k, v, g = synth.prefill_inputs(3901, T, H, D, "bf16", 0.5, True)
    dout = synth.normal(3901, 21, (T, H * D), 1.0, "bf16")
    shp, gshp = (B, T, H, D), (B, T, H * D)
    dq_, dk_, dv_ = (to_dev(a).reshape(shp) for a in (q, k, v))
    dg_, ddo = to_dev(g).reshape(gshp), to_dev(dout).reshape(gshp)
    gate = dg_ if m == la.LA_OUT_RMSNORM_GATE else None
    y = torch.empty(gshp, dtype=torch.bfloat16, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, B, T, 0, H, D, C, la.LA_BF16, m))
    la.lightning_attn_prefill(dq_, dk_, dv_, None, y, None, None, block_size=C, mode=la.LA_OUT_RAW, workspace=ws)
    res = []
    for yy in (None, y):
        gq, gk, gv = (torch.empty_like(dq_) for _ in range(3))
        gg = torch.empty_like(dg_) if gate is not None else None
        gw = torch.empty((H * D,), dtype=torch.float32, device="cuda")
        la.lightning_attn_backward(dq_, dk_, dv_, gate, ddo, gq, gk, gv, dg=gg, block_size=C, mode=m, workspace=ws,
                                   y=yy, dnorm_weight=gw)
        la.lightning_attn_check(ws)
        res.append([to_host(t) for t in (gq, gk, gv, gw) + ((gg,) if gg is not None else ())])
    for a, b in zip(*res):
        np.testing.assert_array_equal(a, b)
    # and the output transform of the kept y is the fused forward's output (tolerance: y is
    # rounded to bf16 before the norm here, the fused kernel normalises fp32 y)
    out = torch.empty(gshp, dtype=torch.bfloat16, device="cuda")
    la.lightning_attn_output_transform(y.view(B, T, H, D), gate, out, mode=m)
    ref, _, _ = oracle.prefill(q.reshape(shp), k.reshape(shp), v.reshape(shp),
                               g.reshape(gshp) if gate is not None else None, mode=m)
    assert_close(to_host(out), ref, "bf16")


def test_backward_wide_rows_norm_weight(cuda_device):
    """H*D = 10240 (more than 4 vectors of 8 per thread in the norm-weight reduction) over
    300 tokens (a full block of 256 tokens and a ragged one)."""
    _run_fixed(1, 300, 80, 128, 256, "bf16", "rmsnorm_gate", False, 3951)


def test_backward_long_sequence_few_heads_splits_every_pass(cuda_device):
    """T = 4096 with 8 heads: every pass (forward and reverse time) is cut into chunks run
    as parallel groups; gradients (with S0 and dS_T) against the oracle."""
    _run_fixed(1, 4096, 8, 128, 256, "bf16", "rmsnorm_gate", True, 3961)


@pytest.mark.parametrize("C", [128, 256])
def test_backward_exact_integers_split(C, cuda_device):
    """The split passes on integer inputs (identity features, ternary values, integer S0
    and dS_T): bit-exact against the oracle, as for the unsplit passes."""
    import torch
    la = _la()
    T, H, D = 4096, 4, 128
    q, k, v, dout = (synth.ternary(3971, s, (T, H, D), 0.03, "bf16") for s in range(4))
    s0 = np.round(synth.normal(3971, 9, (1, H, D, D), 1.0, "f32")).astype(np.float32)
    dsT = np.round(synth.normal(3971, 10, (1, H, D, D), 1.0, "f32")).astype(np.float32)
    f = lambda a: synth.bf16_to_f32(a).astype(np.float64)
    Q, K, V, dY = f(q), f(k), f(v), f(dout)
    for a, b, rev in ((V, K, False), (dY, Q, True), (Q, dY, True), (K, V, False)):
        outer = np.einsum("thi,thj->thij", a, b)
        run = np.cumsum(outer[::-1] if rev else outer, axis=0)
        assert np.abs(run).max() + np.abs(s0).max() + np.abs(dsT).max() <= 256
    shp = (1, T, H, D)
    dq_, dk_, dv_ = (to_dev(a).reshape(shp) for a in (q, k, v))
    ddo = to_dev(dout).reshape(1, T, H * D)
    gq, gk, gv = (torch.full_like(dq_, float("nan")) for _ in range(3))
    gs = torch.full((1, H, D, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, 1, T, 0, H, D, C, la.LA_BF16,
                                                           la.LA_OUT_RAW))
    la.lightning_attn_backward(dq_, dk_, dv_, None, ddo, gq, gk, gv, state_in=to_dev(s0), dstate_in=gs,
                               block_size=C, phi=la.LA_PHI_IDENTITY, mode=la.LA_OUT_RAW, workspace=ws,
                               dstate_out=to_dev(dsT))
    assert la.lightning_attn_last_path() == "tcgen05+chunks"
    la.lightning_attn_check(ws)
    ref = oracle.backward(q.reshape(shp), k.reshape(shp), v.reshape(shp), None, dout.reshape(1, T, H * D),
                          state_in=s0, phi=oracle.PHI_IDENTITY, mode=oracle.MODE_RAW, dstate_out=dsT)
    for got, want, name in zip((gq, gk, gv, gs), (ref[0], ref[1], ref[2], ref[4]), ("dq", "dk", "dv", "dstate")):
        assert np.abs(want).max() <= 256, name
        g64 = synth.bf16_to_f32(to_host(got)).astype(np.float64) if got.dtype == torch.bfloat16 \
            else to_host(got).astype(np.float64)
        bad = np.argwhere(g64.reshape(want.shape) != want)
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first at {bad[:3].tolist()}"
