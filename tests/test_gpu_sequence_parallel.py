"""GPU parity of the sequence-parallel prefill, with the ranks emulated one after another
on one GPU (the all-gather is a stack of the chunk states; no kernel waits on another):
the chunks' outputs and the last chunk's state must match one oracle prefill of the whole
sequence from the same initial state."""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("C,chunks,mode", [(256, [700, 333, 1000], "rmsnorm_gate"),
                                           (128, [1, 255, 640, 129], "rmsnorm_gate"),
                                           (256, [500, 500], "raw")])
def test_emulated_ranks_match_one_prefill(C, chunks, mode, cuda_device):
    import torch
    from long_context_attn_b200 import lightning_attn as la
    from long_context_attn_b200 import sequence_parallel as sp
    m = {"raw": la.LA_OUT_RAW, "rmsnorm_gate": la.LA_OUT_RMSNORM_GATE}[mode]
    H, D = 8, 128
    T = sum(chunks)
    q, k, v, g = synth.prefill_inputs(1401, T, H, D, "bf16", 0.5, True)
    s0 = synth.normal(1401, 9, (H, D, D), 0.05, "f32")
    bounds = np.cumsum([0] + chunks)
    parts = []
    for r in range(len(chunks)):
        a, b = bounds[r], bounds[r + 1]
        dq, dk, dv = (to_dev(x[a:b])[None] for x in (q, k, v))
        dg = to_dev(g[a:b])[None]
        out = torch.empty((1, b - a, H * D), dtype=torch.bfloat16, device="cuda")
        parts.append((dq, dk, dv, dg, out, sp.workspace_for(b - a, H, D, C, m)))
    # step 1 on every "rank", step 2 as a stack, step 3 on every "rank"
    local = [sp.chunk_state(dk, dv, ws) for dq, dk, dv, dg, out, ws in parts]
    gathered = torch.stack(local)
    final = torch.full((H, D, D), float("nan"), dtype=torch.float32, device="cuda")
    ds0 = to_dev(s0)
    for r, (dq, dk, dv, dg, out, ws) in enumerate(parts):
        sp.finish_chunk(dq, dk, dv, dg, out, gathered, r, ws, state0=ds0,
                        state_out=final if r == len(parts) - 1 else None, block_size=C, mode=m)
        la.lightning_attn_check(ws)
    got = np.concatenate([to_host(p[4])[0] for p in parts])
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], g[None], state_in=s0[None], mode=m)
    assert_close(got[None], ref, "bf16")
    assert_close(to_host(final)[None], ref_st, "bf16", "final state")
