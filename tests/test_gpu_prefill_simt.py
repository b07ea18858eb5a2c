"""GPU parity of the CUDA-core prefill (fp32 arithmetic) against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import TOL, assert_close, mode_code, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu


def _la():
    from long_context_attn_b200 import lightning_attn as la
    return la


def run_prefill(q, k, v, g, C, mode, phi=0, state_in=None, want_state=False, w=None, expect_path=None):
    import torch
    la = _la()
    B, T, H, D = q.shape
    dq, dk, dv = (to_dev(a) for a in (q, k, v))
    dg = to_dev(g) if g is not None else None
    out = torch.full((B, T, H * D), float("nan"), dtype=dq.dtype, device="cuda")
    si = to_dev(state_in) if state_in is not None else None
    so = torch.full((B, H, D, D), float("nan"), dtype=torch.float32, device="cuda") if want_state else None
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, B, T, 0, H, D, C, la._dtype(dq), mode))
    dw = None if w is None else to_dev(w)
    la.lightning_attn_prefill(dq, dk, dv, dg, out, si, so, block_size=C, phi=phi, mode=mode, norm_weight=dw,
                              workspace=ws)
    path = la.lightning_attn_last_path()
    la.lightning_attn_check(ws)
    if expect_path:
        assert path == expect_path
    return to_host(out), (to_host(so) if want_state else None), path


def run_varlen(q, k, v, g, lens, C, mode, phi=0, state_in=None, want_state=False, expect_path=None):
    import torch
    la = _la()
    total, H, D = q.shape
    cu = synth.cu_seqlens_of(lens)
    n = len(lens)
    dq, dk, dv = (to_dev(a) for a in (q, k, v))
    dg = to_dev(g) if g is not None else None
    out = torch.full((total, H * D), float("nan"), dtype=dq.dtype, device="cuda")
    si = to_dev(state_in) if state_in is not None else None
    so = torch.full((n, H, D, D), float("nan"), dtype=torch.float32, device="cuda") if want_state else None
    mx = int(max(lens)) if n else 0
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_VARLEN, n, mx, total, H, D, C,
                                                           la._dtype(dq), mode))
    la.lightning_attn_prefill_varlen(dq, dk, dv, dg, out, to_dev(cu), mx, si, so, block_size=C, phi=phi, mode=mode,
                                     workspace=ws)
    path = la.lightning_attn_last_path()
    la.lightning_attn_check(ws)
    if expect_path:
        assert path == expect_path
    return to_host(out), (to_host(so) if want_state else None), path


def test_tiny_config_fp32_vs_recurrence_and_quadratic(cuda_device):
    """B1 H2 T512 D64 fp32, N(0,1), SiLU on q/k, block 64, raw output: tolerance 1e-4."""
    w = synth.WORKLOADS["tiny_f32"]
    q, k, v, _ = synth.prefill_inputs(w.seed, w.T, w.H, w.D, "f32", w.qkv_scale, False)
    o, st, path = run_prefill(q[None], k[None], v[None], None, w.block_size, oracle.MODE_RAW, want_state=True,
                              expect_path="simt")
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RAW)
    assert_close(o, ref, "f32")
    assert_close(st, ref_st, "f32", "state")
    quad = oracle.quadratic(q, k, v).reshape(1, w.T, -1)
    assert rel_err(o, quad) <= TOL["f32"]


@pytest.mark.parametrize("T", [1, 31, 33, 100, 257])
@pytest.mark.parametrize("C", [16, 64, 100])
def test_fp32_shapes_blocks_tails(T, C, cuda_device):
    H, D = 3, 64
    q, k, v, g = synth.prefill_inputs(200 + T, T, H, D, "f32", 1.0, True)
    s0 = synth.normal(200 + T, 9, (1, H, D, D), 0.1, "f32")
    o, st, _ = run_prefill(q[None], k[None], v[None], g[None], C, oracle.MODE_RMSNORM_GATE, state_in=s0,
                           want_state=True, expect_path="simt")
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], g[None], state_in=s0)
    assert_close(o, ref, "f32")
    assert_close(st, ref_st, "f32", "state")


@pytest.mark.parametrize("mode", ["raw", "rmsnorm", "rmsnorm_gate"])
def test_fp32_batch_d128_modes(mode, cuda_device):
    B, T, H, D = 2, 150, 4, 128
    q, k, v, g = synth.prefill_inputs(301, B * T, H, D, "f32", 0.5, True)
    q, k, v = (a.reshape(B, T, H, D) for a in (q, k, v))
    g = g.reshape(B, T, H * D)
    wn = (synth.normal(301, 8, (H * D,), 0.3, "f32") + 1.0) if mode == "rmsnorm" else None
    o, st, _ = run_prefill(q, k, v, g, 64, mode_code(mode), want_state=True, w=wn)
    ref, ref_st, _ = oracle.prefill(q, k, v, g, mode=mode_code(mode), norm_weight=wn)
    assert_close(o, ref, "f32")
    assert_close(st, ref_st, "f32", "state")


def test_bf16_d64_goes_simt(cuda_device):
    T, H, D = 300, 4, 64
    q, k, v, g = synth.prefill_inputs(401, T, H, D, "bf16", 0.5, True)
    o, st, _ = run_prefill(q[None], k[None], v[None], g[None], 256, oracle.MODE_RMSNORM_GATE, want_state=True,
                           expect_path="simt")
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], g[None])
    assert_close(o, ref, "bf16")
    assert_close(st, ref_st, "bf16", "state")


def test_fp32_varlen_with_empty_sequences(cuda_device):
    H, D = 2, 64
    lens = [0, 70, 1, 0, 129]
    tot = sum(lens)
    q, k, v, g = synth.prefill_inputs(501, tot, H, D, "f32", 1.0, True)
    s0 = synth.normal(501, 9, (len(lens), H, D, D), 0.1, "f32")
    o, st, _ = run_varlen(q, k, v, g, lens, 32, oracle.MODE_RMSNORM_GATE, state_in=s0, want_state=True,
                          expect_path="simt")
    ref, ref_st, _ = oracle.forward_packed(q, k, v, g, synth.cu_seqlens_of(lens), H, D, state_in=s0)
    assert_close(o, ref, "f32")
    assert_close(st, ref_st, "f32", "state")
    np.testing.assert_array_equal(st[0], s0[0])  # empty sequence: state passes through


def test_fp32_identity_integer_exact(cuda_device):
    T, H, D = 200, 2, 64
    q = synth.ternary(601, 0, (T, H, D), 0.3, "f32")
    k = synth.ternary(601, 1, (T, H, D), 0.3, "f32")
    v = synth.ternary(601, 2, (T, H, D), 0.3, "f32")
    o, st, _ = run_prefill(q[None], k[None], v[None], None, 64, oracle.MODE_RAW, phi=1, want_state=True)
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], None, phi=oracle.PHI_IDENTITY, mode=oracle.MODE_RAW)
    np.testing.assert_array_equal(o.astype(np.float64), ref)
    np.testing.assert_array_equal(st.astype(np.float64), ref_st)
