"""Failure detection on the GPU without faulting it.

The host injects the failure: the workspace's fault selector tells CTA 0 of the tensor-core
prefill never to publish its norm partials, so every CTA's bounded wait for that tile runs
out (a flag that nothing sets).  With a 50 ms limit written into the workspace, the call
must report LA_ERR_TIMEOUT through lightning_attn_check, the kernel must end on its own,
and the context must stay usable: a normal call right after gives the oracle's result.
"""
import pytest

import oracle
import synth
from tests._helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu

# Sites of the tensor-core kernel's bounded waits (producer, MMA, transform, conversion,
# epilogue, norm wait).  Every wait has the same limit, so the role that started waiting
# first (often the producer, stalled behind the blocked pipeline) records the timeout.
TC_SITES = {1, 2, 3, 4, 5, 6}


def test_norm_wait_timeout_is_reported_and_context_survives(cuda_device):
    import torch
    from long_context_attn_b200 import lightning_attn as la

    T, H, D = 1024, 8, 128
    q, k, v, g = synth.prefill_inputs(4242, T, H, D, "bf16", 0.5, True)
    dq, dk, dv, dg = (to_dev(a)[None] for a in (q, k, v, g))
    out = torch.zeros((1, T, H * D), dtype=torch.bfloat16, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, 1, T, 0, H, D, 256, la.LA_BF16,
                                                           la.LA_OUT_RMSNORM_GATE))
    hdr = ws[:256].view(torch.int32)
    hdr[4] = 50   # bounded-wait limit in ms
    hdr[5] = 1    # inject: CTA 0 skips publishing
    la.lightning_attn_prefill(dq, dk, dv, dg, out, workspace=ws)
    assert la.lightning_attn_last_path() == "tcgen05"
    st, detail = la.lightning_attn_check(ws, raise_on_error=False)
    assert st == la.LA_ERR_TIMEOUT, (st, detail)
    assert detail[1] in TC_SITES, detail

    # the record was cleared by the check; remove the injection and run normally
    hdr[4] = 0
    hdr[5] = 0
    la.lightning_attn_prefill(dq, dk, dv, dg, out, workspace=ws)
    la.lightning_attn_check(ws)
    ref, _, _ = oracle.prefill(q[None], k[None], v[None], g[None])
    assert_close(to_host(out), ref, "bf16")
