"""The workspace-free decode step (lightning_attn_decode_step_noalloc).

Some callers of this library cannot allocate device memory (their HBM is owned by another
allocator, or cudaMalloc is not allowed in their decode loop), so this entry point keeps
its scratch in a fixed array inside the library.  Two calls in a row are compared with the
workspace entry point on the same inputs and the same starting state; the second call
also checks that leftovers of the first call in the shared array do not leak into it.
This file is collected last so a failure here never hides the other tests.
"""
import numpy as np
import pytest

import synth
from tests._helpers import TOL, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu


def test_noalloc_decode_two_calls_match_workspace_decode(cuda_device):
    import torch
    from long_context_attn_b200 import lightning_attn as la

    w = synth.WORKLOADS["decode_256"]
    B, H, D = w.B, w.H, w.D
    S0 = synth.decode_state(w.seed, B, H, D)
    S_ref, S_new = to_dev(S0), to_dev(S0)
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_DECODE, B, 0, 0, H, D, 0, la.LA_BF16,
                                                           la.LA_OUT_RMSNORM_GATE))
    out_ref = torch.empty((B, H * D), dtype=torch.bfloat16, device="cuda")
    out_new = torch.empty_like(out_ref)
    for step in range(2):
        q, k, v, g = (to_dev(a) for a in synth.decode_tokens(w.seed, step, B, H, D, "bf16", w.qkv_scale))
        la.lightning_attn_decode_step(q, k, v, g, out_ref, S_ref, workspace=ws)
        la.lightning_attn_decode_step_noalloc(q, k, v, g, out_new, S_new)
        torch.cuda.synchronize()
        ref = synth.bf16_to_f32(to_host(out_ref)).astype(np.float64)
        assert rel_err(to_host(out_new), ref) <= TOL["bf16"], f"call {step + 1}: output differs"
        assert rel_err(to_host(S_new), to_host(S_ref).astype(np.float64)) <= 1e-6, f"call {step + 1}: state differs"
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
