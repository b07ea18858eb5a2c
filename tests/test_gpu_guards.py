"""Guard (canary) tests: every kernel writes only the rows and states it owns.

Outputs and states are views into larger device buffers whose leading and trailing rows
hold a sentinel bit pattern; after each call the sentinels must be untouched and the
owned part must still match the oracle.  Varlen packing is checked the same way: the
rows of the packed output that belong to no sequence keep their sentinel.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu

GUARD = 64          # sentinel rows before and after each output
SENT_BF16 = 0x7FC1  # a NaN payload no kernel produces
SENT_F32 = 0x7FC00123


def _la():
    from long_context_attn_b200 import lightning_attn as la
    return la


def _guarded(rows, cols, dtype):
    """(whole buffer, view of the middle `rows` rows) filled with the sentinel."""
    import torch
    if dtype == "bf16":
        whole = torch.full((rows + 2 * GUARD, cols), SENT_BF16, dtype=torch.int16, device="cuda")
        return whole, whole[GUARD:GUARD + rows].view(torch.bfloat16)
    whole = torch.full((rows + 2 * GUARD, cols), SENT_F32, dtype=torch.int32, device="cuda")
    return whole, whole[GUARD:GUARD + rows].view(torch.float32)


def _check_guards(whole, dtype, what):
    sent = SENT_BF16 if dtype == "bf16" else SENT_F32
    host = whole.cpu().numpy()
    assert np.all(host[:GUARD] == np.array(sent, dtype=host.dtype)), f"{what}: leading guard overwritten"
    assert np.all(host[-GUARD:] == np.array(sent, dtype=host.dtype)), f"{what}: trailing guard overwritten"


@pytest.mark.parametrize("dtype,D,C,expect", [("bf16", 128, 256, "tcgen05"), ("bf16", 128, 128, "tcgen05"),
                                              ("f32", 64, 64, "simt")])
@pytest.mark.parametrize("T", [33, 300])
def test_prefill_writes_only_its_rows(dtype, D, C, expect, T, cuda_device):
    la = _la()
    H = 8
    q, k, v, g = synth.prefill_inputs(1201, T, H, D, dtype, 0.5, True)
    whole_o, out = _guarded(T, H * D, dtype)
    whole_s, st = _guarded(H * D, D, "f32")          # the state [1, H, D, D] as H*D rows of D
    dq, dk, dv, dg = (to_dev(a)[None] for a in (q, k, v, g))
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, 1, T, 0, H, D, C, la._dtype(dq),
                                                           la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_prefill(dq, dk, dv, dg, out.view(1, T, H * D), None, st.view(1, H, D, D), block_size=C,
                              workspace=ws)
    assert la.lightning_attn_last_path() == expect
    la.lightning_attn_check(ws)
    _check_guards(whole_o, dtype, "output")
    _check_guards(whole_s, "f32", "state")
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], g[None])
    assert_close(to_host(out)[None], ref, dtype)
    assert_close(to_host(st).reshape(1, H, D, D), ref_st, dtype, "state")


def test_varlen_leaves_unowned_rows_alone(cuda_device):
    """Packed rows [0, total) are owned; the buffer continues past `total` (sentinels)."""
    import torch
    la = _la()
    H, D = 8, 128
    lens = [100, 0, 257, 31]
    tot = sum(lens)
    q, k, v, g = synth.prefill_inputs(1202, tot, H, D, "bf16", 0.5, True)
    whole_o, out = _guarded(tot, H * D, "bf16")
    n = len(lens)
    whole_s, st = _guarded(n * H * D, D, "f32")
    dq, dk, dv, dg = (to_dev(a) for a in (q, k, v, g))
    cu = torch.from_numpy(synth.cu_seqlens_of(lens)).cuda()
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_VARLEN, n, max(lens), tot, H, D, 256,
                                                           la.LA_BF16, la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_prefill_varlen(dq, dk, dv, dg, out, cu, max(lens), None, st.view(n, H, D, D), block_size=256,
                                     workspace=ws)
    assert la.lightning_attn_last_path() == "tcgen05"
    la.lightning_attn_check(ws)
    _check_guards(whole_o, "bf16", "output")
    _check_guards(whole_s, "f32", "state")
    ref, ref_st, _ = oracle.forward_packed(q, k, v, g, synth.cu_seqlens_of(lens), H, D)
    assert_close(to_host(out), ref, "bf16")
    assert_close(to_host(st).reshape(n, H, D, D), ref_st, "bf16", "state")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_writes_only_its_rows(dtype, cuda_device):
    la = _la()
    B, H, D = 5, 8, 128
    S = synth.normal(1203, 4, (B, H, D, D), 0.1, "f32")
    q, k, v, g = synth.decode_tokens(1203, 0, B, H, D, dtype, 0.5)
    whole_o, out = _guarded(B, H * D, dtype)
    whole_s, st = _guarded(B * H * D, D, "f32")
    st.copy_(to_dev(S).view(B * H * D, D))
    dq, dk, dv, dg = (to_dev(a) for a in (q, k, v, g))
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_DECODE, B, 0, 0, H, D, 0, la._dtype(dq),
                                                           la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_decode_step(dq, dk, dv, dg, out, st.view(B, H, D, D), workspace=ws)
    la.lightning_attn_check(ws)
    _check_guards(whole_o, dtype, "output")
    _check_guards(whole_s, "f32", "state")
    ref_o, ref_S, _ = oracle.decode(q, k, v, g, S)
    assert_close(to_host(out), ref_o, dtype)
    assert_close(to_host(st).reshape(B, H, D, D), ref_S, dtype, "state")
