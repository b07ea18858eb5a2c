"""GPU parity of lightning_attn_decode_step against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import as_f64, assert_close, mode_code, record_margin, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu


def _la():
    from long_context_attn_b200 import lightning_attn as la
    return la


def _run_decode(q, k, v, g, S, mode, phi=0, eps=1e-6, w=None, ws=None):
    import torch
    la = _la()
    B, H, D = q.shape
    dq, dk, dv, dg = (to_dev(a) for a in (q, k, v, g))
    dS = to_dev(S)
    out = torch.empty((B, H * D), dtype=dq.dtype, device="cuda")
    if ws is None:
        ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_DECODE, B, 0, 0, H, D, 0,
                                                               la._dtype(dq), mode))
    dw = None if w is None else to_dev(w)
    la.lightning_attn_decode_step(dq, dk, dv, dg, out, dS, phi=phi, mode=mode, eps=eps, norm_weight=dw, workspace=ws)
    la.lightning_attn_check(ws)
    assert la.lightning_attn_last_path() == "decode"
    return to_host(out), to_host(dS), ws


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mode", ["raw", "rmsnorm", "rmsnorm_gate"])
def test_decode_small(dtype, D, mode, cuda_device):
    B, H = 5, 6
    q, k, v, g = synth.decode_tokens(77, 0, B, H, D, dtype, 0.5)
    S = synth.decode_state(77, B, H, D)
    w = synth.normal(77, 8, (H * D,), 0.3, "f32") + 1.0 if mode == "rmsnorm" else None
    o, S_new, _ = _run_decode(q, k, v, g, S, mode_code(mode), w=w)
    ref_o, ref_S, _ = oracle.decode(q, k, v, g, S, mode=mode_code(mode), norm_weight=w)
    assert_close(o, ref_o, dtype)
    # the state is fp32 in place: tighter than the output tolerance
    assert rel_err(S_new, ref_S) <= 1e-5


def test_decode_identity_exact(cuda_device):
    # phi = identity, integer-valued inputs: update and read are exact in fp32.
    B, H, D = 3, 4, 128
    q = synth.ternary(5, 0, (B, H, D), 0.5, "bf16")
    k = synth.ternary(5, 1, (B, H, D), 0.5, "bf16")
    v = synth.ternary(5, 2, (B, H, D), 0.5, "bf16")
    g = synth.normal(5, 3, (B, H * D), 1.0, "bf16")
    S = np.round(synth.normal(5, 4, (B, H, D, D), 3.0, "f32"))
    o, S_new, _ = _run_decode(q, k, v, g, S, oracle.MODE_RAW, phi=1)
    ref_o, ref_S, _ = oracle.decode(q, k, v, g, S, phi=oracle.PHI_IDENTITY, mode=oracle.MODE_RAW)
    np.testing.assert_array_equal(S_new.astype(np.float64), ref_S)
    np.testing.assert_array_equal(as_f64(o), ref_o)  # |y| small integers: exact in bf16


def test_decode_workspace_left_zeroed_and_reusable(cuda_device):
    import torch
    B, H, D = 7, 8, 128
    q, k, v, g = synth.decode_tokens(9, 0, B, H, D, "bf16", 0.5)
    S = synth.decode_state(9, B, H, D)
    o1, _, ws = _run_decode(q, k, v, g, S, oracle.MODE_RMSNORM_GATE)
    assert int(ws[256:256 + 4 * B].view(torch.int32).abs().sum()) == 0
    o2, _, _ = _run_decode(q, k, v, g, S, oracle.MODE_RMSNORM_GATE, ws=ws)
    np.testing.assert_array_equal(o1, o2)  # deterministic: fixed-order reductions


@pytest.mark.slow
def test_decode_full_config_16_steps(cuda_device):
    """256 sequences x 64 heads x 128, S ~ N(0,1)/sqrt(128); checked after steps 1 and 16."""
    import torch
    la = _la()
    w = synth.WORKLOADS["decode_256"]
    B, H, D = w.B, w.H, w.D
    S0 = synth.decode_state(w.seed, B, H, D)
    dS = to_dev(S0)
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_DECODE, B, 0, 0, H, D, 0, la.LA_BF16,
                                                           la.LA_OUT_RMSNORM_GATE))
    out = torch.empty((B, H * D), dtype=torch.bfloat16, device="cuda")
    ref_S = S0
    for step in range(16):
        q, k, v, g = synth.decode_tokens(w.seed, step, B, H, D, "bf16", w.qkv_scale)
        la.lightning_attn_decode_step(to_dev(q), to_dev(k), to_dev(v), to_dev(g), out, dS, workspace=ws)
        ref_o, ref_S64, _ = oracle.decode(q, k, v, g, ref_S)
        ref_S = ref_S64.astype(np.float32)
        if step in (0, 15):
            la.lightning_attn_check(ws)
            e_o = assert_close(to_host(out), ref_o, "bf16", f"decode output after step {step + 1}")
            e_s = rel_err(to_host(dS), ref_S64)
            assert e_s <= 1e-5
            record_margin(f"test_decode_full_config_16_steps step {step + 1}", out=e_o, state=e_s)
