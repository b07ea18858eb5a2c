"""GPU tests of paths composed from calls that the per-kernel files test on their own:
the sequence-parallel prefill of a packed variable-length batch (ranks emulated one after
another on one GPU: a stack stands in for the all-gather, no kernel waits on another) and
the normalised variant continued in place (state_out = state_in, z_out = z_in).  Collected
after the per-kernel files, so a failure here never hides theirs."""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


def _shift(a):
    """q and k shifted by +1 (bf16) so that phi(q) . z stays away from zero."""
    return synth.f32_to_bf16(synth.bf16_to_f32(a) + 1.0)


def test_emulated_ranks_varlen_batch_match_one_packed_prefill(cuda_device):
    """A packed batch cut into five rank slices (one empty; sequences spanning two and three
    ranks; empty sequences; a sequence ending on a slice boundary), the ranks emulated one
    after another: every token's output and every sequence's final state against one
    oracle prefill of the whole batch from the same initial states."""
    import torch
    from long_context_attn_b200 import lightning_attn as la
    from long_context_attn_b200 import sequence_parallel as sp
    H, D, C = 8, 128, 256
    lens = [300, 0, 900, 129, 1000, 0, 257, 0]
    bounds = [0, 500, 500, 1200, 1700, 2586]
    cu = synth.cu_seqlens_of(lens)
    tot = int(cu[-1])
    assert tot == bounds[-1]
    q, k, v, g = synth.prefill_inputs(1411, tot, H, D, "bf16", 0.5, True)
    s0 = synth.normal(1411, 9, (len(lens), H, D, D), 0.05, "f32")
    ds0 = to_dev(s0)
    world = len(bounds) - 1
    ranks = []
    for r in range(world):
        a, b = bounds[r], bounds[r + 1]
        plan = sp.varlen_slice_plan(cu, bounds, r)
        dq, dk, dv, dg = (to_dev(x[a:b]) for x in (q, k, v, g))
        out = torch.full((b - a, H * D), float("nan"), dtype=torch.bfloat16, device="cuda")
        ranks.append((plan, dq, dk, dv, dg, out, sp.varlen_workspace_for(plan, H, D, C)))
    carries = [sp.varlen_carry(dk, dv, plan, ws) for plan, dq, dk, dv, dg, out, ws in ranks]
    gathered = torch.stack(carries)
    finals = {}
    for r, (plan, dq, dk, dv, dg, out, ws) in enumerate(ranks):
        st = sp.varlen_finish(dq, dk, dv, dg, out, gathered, plan, r, ws, state0=ds0, block_size=C)
        la.lightning_attn_check(ws)
        for i, s in enumerate(plan.seq):
            if plan.final[i]:
                assert s not in finals
                finals[s] = to_host(st[i])
    assert sorted(finals) == list(range(len(lens)))
    got = np.concatenate([to_host(p[5]) for p in ranks])
    ref, ref_st, _ = oracle.forward_packed(q, k, v, g, cu, H, D, state_in=s0)
    assert_close(got, ref, "bf16")
    assert_close(np.stack([finals[s] for s in range(len(lens))]), ref_st, "bf16", "final states")


def test_prefill_znorm_continuation_in_place(cuda_device):
    """A 10000-token sequence as two calls, the second continuing from the first with the
    state and z updated in place (state_out = state_in, z_out = z_in; 20 scan chunks, so the
    chunk items span several blocks): output and final state and z against one oracle run."""
    import torch
    from long_context_attn_b200 import lightning_attn as la
    H, D, C, T1, T2 = 8, 128, 256, 4880, 5120
    T = T1 + T2
    q, k, v, g = synth.prefill_inputs(3441, T, H, D, "bf16", 0.5, True)
    q, k = _shift(q), _shift(k)
    S = torch.empty((1, H, D, D), dtype=torch.float32, device="cuda")
    z = torch.empty((1, H, D), dtype=torch.float32, device="cuda")
    outs = []
    for a, b, first in ((0, T1, True), (T1, T, False)):
        shp, gshp = (1, b - a, H, D), (1, b - a, H * D)
        out = torch.empty(gshp, dtype=torch.bfloat16, device="cuda")
        ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_ZNORM, 1, b - a, 0, H, D, C,
                                                               la.LA_BF16, la.LA_OUT_RMSNORM_GATE))
        la.lightning_attn_prefill_znorm(*(to_dev(x[a:b]).reshape(shp) for x in (q, k, v)),
                                        to_dev(g[a:b]).reshape(gshp), out, state_in=None if first else S,
                                        z_in=None if first else z, state_out=S, z_out=z, block_size=C,
                                        workspace=ws)
        la.lightning_attn_check(ws)
        outs.append(to_host(out)[0])
    shp, gshp = (1, T, H, D), (1, T, H * D)
    ref, ref_S, ref_z = oracle.prefill_znorm(q.reshape(shp), k.reshape(shp), v.reshape(shp), g.reshape(gshp))
    assert_close(np.concatenate(outs)[None], ref, "bf16")
    assert_close(to_host(S), ref_S, "bf16", "state")
    assert_close(to_host(z), ref_z, "f32", "z")
