"""The workspace-free decode step (lightning_attn_decode_step_noalloc).

Some callers of this library cannot allocate device memory (their HBM is owned by another
allocator, or cudaMalloc is not allowed in their decode loop), so this entry point keeps
its scratch in a fixed array inside the library.  Two calls in a row are compared with the
workspace entry point on the same inputs and the same starting state: it runs the same
kernel, so output and state must agree bit for bit, and the second call also shows that
leftovers of the first call in the shared array do not leak into it.  Each call is also
checked against the oracle within the bf16 tolerance.  This file is collected last so a
failure here never hides the other tests.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import TOL, assert_close, mode_code, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,D,mode", [(256, 64, 128, "rmsnorm_gate"), (96, 12, 64, "rmsnorm")])
def test_noalloc_decode_two_calls_match_workspace_decode(B, H, D, mode, cuda_device):
    import torch
    from long_context_attn_b200 import lightning_attn as la

    w = synth.WORKLOADS["decode_256"]
    m = mode_code(mode)
    la_mode = {"rmsnorm_gate": la.LA_OUT_RMSNORM_GATE, "rmsnorm": la.LA_OUT_RMSNORM}[mode]
    S0 = synth.decode_state(w.seed + D, B, H, D)
    S_ref, S_new = to_dev(S0), to_dev(S0)
    S_oracle = S0
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_DECODE, B, 0, 0, H, D, 0, la.LA_BF16, la_mode))
    out_ref = torch.empty((B, H * D), dtype=torch.bfloat16, device="cuda")
    out_new = torch.empty_like(out_ref)
    for step in range(2):
        q, k, v, g = synth.decode_tokens(w.seed + D, step, B, H, D, "bf16", w.qkv_scale)
        gh = g if m == oracle.MODE_RMSNORM_GATE else None
        dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
        dg = to_dev(g) if gh is not None else None
        la.lightning_attn_decode_step(dq, dk, dv, dg, out_ref, S_ref, mode=la_mode, workspace=ws)
        la.lightning_attn_decode_step_noalloc(dq, dk, dv, dg, out_new, S_new, mode=la_mode)
        assert la.lightning_attn_last_path() == "decode"
        torch.cuda.synchronize()
        assert torch.equal(out_new, out_ref), f"call {step + 1}: output differs from the workspace decode"
        assert torch.equal(S_new, S_ref), f"call {step + 1}: state differs from the workspace decode"
        ref_o, ref_S64, _ = oracle.decode(q, k, v, gh, S_oracle, mode=m)
        S_oracle = ref_S64.astype(np.float32)
        assert_close(to_host(out_new), ref_o, "bf16", f"call {step + 1}: output vs oracle")
        assert rel_err(to_host(S_new), ref_S64) <= TOL["f32"], f"call {step + 1}: state vs oracle"
    la.lightning_attn_check(ws)


def test_noalloc_decode_rejects_batches_beyond_the_fixed_scratch(cuda_device):
    import torch
    from long_context_attn_b200 import lightning_attn as la

    B, H, D = 1024, 64, 128  # raw outputs alone need 32 MiB > the fixed scratch
    z = torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, H * D), dtype=torch.bfloat16, device="cuda")
    S = torch.zeros((4,), dtype=torch.float32, device="cuda")  # rejected before it is read
    with pytest.raises(la.LightningAttnError) as ei:
        la.lightning_attn_decode_step_noalloc(z, z, z, out, out, S)
    assert ei.value.status == la.LA_ERR_UNSUPPORTED
