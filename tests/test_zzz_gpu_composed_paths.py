"""GPU tests of paths composed from calls that the per-kernel files test on their own:
the sequence-parallel prefill and backward (one sequence or a packed variable-length batch;
ranks emulated one after another on one GPU: a stack stands in for the all-gather, no
kernel waits on another), the output transform's backward as its own entry point, the
normalised variant continued in place (state_out = state_in, z_out = z_in) and the
host-memory prefill with overlapped copies.  Collected after every other file (the
per-kernel ones and the workspace-free decode), so a failure here never hides theirs."""
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
        st, _ = sp.varlen_finish(dq, dk, dv, dg, out, gathered, plan, r, ws, state0=ds0, block_size=C)
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


@pytest.mark.parametrize("mode", ["raw", "rmsnorm", "rmsnorm_gate"])
def test_output_transform_backward_matches_oracle(mode, cuda_device):
    """lightning_attn_output_transform_backward (the norm/gate backward kernels behind their own
    entry point): dy, dg and dw against the oracle's transform backward over 700 tokens."""
    import torch
    from long_context_attn_b200 import lightning_attn as la
    from tests._helpers import mode_code
    m = mode_code(mode)
    tokens, H, D = 700, 8, 128
    y = synth.normal(3451, 1, (tokens, H * D), 1.0, "bf16")
    g = synth.normal(3451, 2, (tokens, H * D), 1.0, "bf16")
    dout = synth.normal(3451, 3, (tokens, H * D), 1.0, "bf16")
    w = (1.0 + 0.2 * synth.normal(3451, 4, (H * D,), 1.0, "f32")).astype(np.float32)
    gate = m == la.LA_OUT_RMSNORM_GATE
    dy = torch.full((tokens, H * D), float("nan"), dtype=torch.bfloat16, device="cuda")
    dg = torch.full((tokens, H * D), float("nan"), dtype=torch.bfloat16, device="cuda") if gate else None
    dw = torch.full((H * D,), float("nan"), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_OUTPUT_TRANSFORM_BACKWARD, tokens, 0, 0, H, D, 0,
                                                           la.LA_BF16, m))
    la.lightning_attn_output_transform_backward(to_dev(y).view(tokens, H, D), to_dev(g) if gate else None,
                                                to_dev(dout), dy, dg=dg, dnorm_weight=dw, mode=m,
                                                norm_weight=to_dev(w), workspace=ws)
    torch.cuda.synchronize()
    yf = synth.bf16_to_f32(y).astype(np.float64).reshape(tokens, H, D)
    rdy, rdg, rdw = oracle.transform_backward(yf, dout, m, norm_weight=w, g=g if gate else None)
    assert_close(to_host(dy), rdy, "bf16", "dy")
    if gate:
        assert_close(to_host(dg), rdg, "bf16", "dg")
    if m == la.LA_OUT_RAW:
        assert torch.all(dw == 0)
    else:
        assert_close(to_host(dw), rdw, "bf16", "dw")


def test_emulated_ranks_backward_match_one_backward(cuda_device):
    """The sequence-parallel backward over three chunks (a one-token chunk in the middle), the
    ranks emulated one after another (backward_local on every rank, a stack for the
    all-gather, backward_finish on every rank), with an initial state, a final-state
    gradient, a norm weight and the gate: every chunk's dq, dk, dv, dg, the chunks' dw summed
    and the first chunk's initial-state gradient against one oracle backward."""
    import torch
    from long_context_attn_b200 import sequence_parallel as sp
    H, D, C = 8, 128, 256
    chunks = [700, 1, 333]
    T = sum(chunks)
    q, k, v, g = synth.prefill_inputs(1421, T, H, D, "bf16", 0.5, True)
    dout = synth.normal(1421, 11, (T, H * D), 1.0, "bf16")
    s0 = synth.normal(1421, 9, (H, D, D), 0.05, "f32")
    dsT = synth.normal(1421, 10, (H, D, D), 0.05, "f32")
    w = (1.0 + 0.2 * synth.normal(1421, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    bounds = np.cumsum([0] + chunks)
    dw_, ds0_, dsT_ = to_dev(w), to_dev(s0), to_dev(dsT)
    ranks = []
    for r in range(len(chunks)):
        a, b = bounds[r], bounds[r + 1]
        dq, dk, dv = (to_dev(x[a:b])[None] for x in (q, k, v))
        ranks.append((dq, dk, dv, to_dev(g[a:b])[None], to_dev(dout[a:b])[None],
                      sp.backward_workspace_for(b - a, H, D, C)))
    # forward steps (for each chunk's initial state)
    fws = [sp.workspace_for(b - a, H, D, C) for a, b in zip(bounds[:-1], bounds[1:])]
    local = [sp.chunk_state(p[1], p[2], ws) for p, ws in zip(ranks, fws)]
    gathered = torch.stack(local)
    prefixes = []
    for r, (dq, dk, dv, dg, dd, _) in enumerate(ranks):
        out = torch.empty((1, dq.shape[1], H * D), dtype=torch.bfloat16, device="cuda")
        prefixes.append(sp.finish_chunk(dq, dk, dv, dg, out, gathered, r, fws[r], state0=ds0_, block_size=C,
                                        norm_weight=dw_))
    # backward steps
    grads, dys, Gs = [], [], []
    for r, (dq, dk, dv, dg, dd, ws) in enumerate(ranks):
        gq, gk, gv = (torch.full_like(dq, float("nan")) for _ in range(3))
        gg = torch.full_like(dg, float("nan"))
        gw = torch.full((H * D,), float("nan"), dtype=torch.float32, device="cuda")
        gs = torch.full((H, D, D), float("nan"), dtype=torch.float32, device="cuda")
        dy, G = sp.backward_local(dq, dk, dv, dg, dd, prefixes[r], ws, dg=gg, dnorm_weight=gw,
                                  dstate_end=dsT_ if r == len(chunks) - 1 else None, block_size=C, norm_weight=dw_)
        grads.append((gq, gk, gv, gg, gw, gs))
        dys.append(dy)
        Gs.append(G)
    gathered = torch.stack(Gs)
    for r, (dq, dk, dv, dg, dd, ws) in enumerate(ranks):
        gq, gk, gv, gg, gw, gs = grads[r]
        sp.backward_finish(dq, dk, dv, dys[r], gq, gk, gv, gathered, r, prefixes[r], ws,
                           dstate_end=dsT_ if r == len(chunks) - 1 else None, dstate_in=gs, block_size=C)
    torch.cuda.synchronize()
    ref = oracle.backward(q[None], k[None], v[None], g[None], dout[None], state_in=s0[None], norm_weight=w,
                          dstate_out=dsT[None])
    for i, name in enumerate(("dq", "dk", "dv", "dg")):
        got = np.concatenate([to_host(grads[r][i])[0] for r in range(len(chunks))])
        assert_close(got[None], ref[i], "bf16", name)
    assert_close(sum(to_host(grads[r][4]).astype(np.float64) for r in range(len(chunks))), ref[5], "bf16", "dw")
    assert_close(to_host(grads[0][5]), ref[4][0], "bf16", "dS0")


def test_emulated_ranks_varlen_backward_match_one_packed_backward(cuda_device):
    """The packed batch and cuts of the varlen forward test above, backwards, the ranks emulated
    one after another (varlen_backward_local on every rank, a stack for the all-gather,
    varlen_backward_finish on every rank): every token's dq, dk, dv, dg, the ranks' dw summed
    and every sequence's initial-state gradient against one oracle backward of the batch."""
    import torch
    from long_context_attn_b200 import sequence_parallel as sp
    H, D, C = 8, 128, 256
    lens = [300, 0, 900, 129, 1000, 0, 257, 0]
    bounds = [0, 500, 500, 1200, 1700, 2586]
    cu = synth.cu_seqlens_of(lens)
    tot, n = int(cu[-1]), len(lens)
    q, k, v, g = synth.prefill_inputs(1431, tot, H, D, "bf16", 0.5, True)
    dout = synth.normal(1431, 11, (tot, H * D), 1.0, "bf16")
    s0 = synth.normal(1431, 9, (n, H, D, D), 0.05, "f32")
    dsT = synth.normal(1431, 10, (n, H, D, D), 0.05, "f32")
    w = (1.0 + 0.2 * synth.normal(1431, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    ds0_, dsT_, dw_ = to_dev(s0), to_dev(dsT), to_dev(w)
    world = len(bounds) - 1
    ranks = []
    for r in range(world):
        a, b = bounds[r], bounds[r + 1]
        plan = sp.varlen_slice_plan(cu, bounds, r)
        ranks.append((plan, *(to_dev(x[a:b]) for x in (q, k, v, g, dout)),
                      sp.varlen_workspace_for(plan, H, D, C), sp.varlen_backward_workspace_for(plan, H, D, C)))
    # forward: the pieces' initial states
    carries = [sp.varlen_carry(dk, dv, plan, fws) for plan, dq, dk, dv, dg, dd, fws, bws in ranks]
    gathered = torch.stack(carries)
    st_ins = []
    for r, (plan, dq, dk, dv, dg, dd, fws, bws) in enumerate(ranks):
        out = torch.empty((plan.hi - plan.lo, H * D), dtype=torch.bfloat16, device="cuda")
        _, st_in = sp.varlen_finish(dq, dk, dv, dg, out, gathered, plan, r, fws, state0=ds0_, block_size=C,
                                    norm_weight=dw_)
        st_ins.append(st_in)
    # backward
    grads, dys, Gs = [], [], []
    for r, (plan, dq, dk, dv, dg, dd, fws, bws) in enumerate(ranks):
        gq, gk, gv = (torch.full_like(dq, float("nan")) for _ in range(3))
        gg = torch.full_like(dg, float("nan"))
        gw = torch.full((H * D,), float("nan"), dtype=torch.float32, device="cuda")
        gs = torch.full((len(plan.seq), H, D, D), float("nan"), dtype=torch.float32, device="cuda")
        dy, G = sp.varlen_backward_local(dq, dk, dv, dg, dd, plan, st_ins[r], bws, dg=gg, dnorm_weight=gw,
                                         block_size=C, norm_weight=dw_)
        grads.append((gq, gk, gv, gg, gw, gs))
        dys.append(dy)
        Gs.append(G)
    gathered = torch.stack(Gs)
    starts = {}
    for r, (plan, dq, dk, dv, dg, dd, fws, bws) in enumerate(ranks):
        gq, gk, gv, gg, gw, gs = grads[r]
        sp.varlen_backward_finish(dq, dk, dv, dys[r], gq, gk, gv, gathered, plan, cu, bounds, r, st_ins[r], bws,
                                  dstate_out=dsT_, dstate_in=gs, block_size=C)
        for i, s in enumerate(plan.seq):
            if not (i == 0 and plan.first_from is not None):
                assert s not in starts
                starts[s] = gs[i]
    torch.cuda.synchronize()
    assert sorted(starts) == list(range(n))
    ref = oracle.backward_packed(q, k, v, g, dout, cu, H, D, state_in=s0, norm_weight=w, dstate_out=dsT)
    for i, name in enumerate(("dq", "dk", "dv", "dg")):
        got = np.concatenate([to_host(grads[r][i]) for r in range(world)])
        assert_close(got, ref[i], "bf16", name)
    assert_close(sum(to_host(grads[r][4]).astype(np.float64) for r in range(world)), ref[5], "bf16", "dw")
    assert_close(np.stack([to_host(starts[s]) for s in range(n)]), ref[4], "bf16", "dS0")


@pytest.mark.parametrize("chunk", [4096, 20000])
def test_host_prefill_pipeline_matches_one_prefill(chunk, cuda_device):
    """HostPrefill: a 10000-token sequence in pinned host memory, chunks pipelined over three
    streams (4096: three chunks with a ragged last one; 20000: one chunk), from an initial
    state: the host output and the final state against one oracle prefill."""
    import torch
    from long_context_attn_b200.host_stream import HostPrefill
    H, D, T = 8, 128, 10000
    q, k, v, g = synth.prefill_inputs(1441, T, H, D, "bf16", 0.5, True)
    s0 = synth.normal(1441, 9, (H, D, D), 0.05, "f32")
    pin = lambda a, shape: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).reshape(shape).pin_memory()
    hq, hk, hv = (pin(a, (T, H, D)) for a in (q, k, v))
    hg = pin(g, (T, H * D))
    hout = torch.full((T, H * D), float("nan"), dtype=torch.bfloat16).pin_memory()
    st = torch.full((H, D, D), float("nan"), dtype=torch.float32, device="cuda")
    hp = HostPrefill(H, D, chunk_tokens=chunk)
    hp(hq, hk, hv, hg, hout, state_in=to_dev(s0), state_out=st)
    torch.cuda.current_stream().synchronize()
    hp.check()
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], g[None], state_in=s0[None])
    assert_close(hout.float().numpy()[None], ref, "bf16")
    assert_close(to_host(st)[None], ref_st, "bf16", "final state")


def test_sequence_parallel_autograd_single_rank(cuda_device):
    """lightning_attention_sequence_parallel with a group of one (the all-gather a stack of one):
    out, the end state and, under loss.backward(), every input's gradient against the oracle."""
    import torch
    from long_context_attn_b200.autograd import lightning_attention_sequence_parallel
    H, D, T = 8, 128, 700
    q, k, v, g = synth.prefill_inputs(1451, T, H, D, "bf16", 0.5, True)
    dout = synth.f32_to_bf16(synth.normal(1451, 11, (T, H * D), 1.0, "f32"))
    s0 = synth.normal(1451, 9, (H, D, D), 0.05, "f32")
    dsT = synth.normal(1451, 10, (H, D, D), 0.05, "f32")
    w = (1.0 + 0.2 * synth.normal(1451, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    leaf = lambda a, shape: to_dev(a).reshape(shape).clone().requires_grad_(True)
    tq, tk, tv = (leaf(a, (1, T, H, D)) for a in (q, k, v))
    tg, ts0, tw = leaf(g, (1, T, H * D)), leaf(s0, (H, D, D)), leaf(w, (H * D,))
    out, st = lightning_attention_sequence_parallel(tq, tk, tv, tg, state0=ts0, norm_weight=tw, rank=0,
                                                    all_gather=lambda x: x[None])
    loss = (out.float() * to_dev(dout).reshape(1, T, H * D).float()).sum() + (st * to_dev(dsT)).sum()
    loss.backward()
    ref_o, ref_s, _ = oracle.prefill(q[None], k[None], v[None], g[None], state_in=s0[None], norm_weight=w)
    assert_close(to_host(out.detach()), ref_o, "bf16")
    assert_close(to_host(st.detach())[None], ref_s, "bf16", "end state")
    ref = oracle.backward(q[None], k[None], v[None], g[None], dout[None], state_in=s0[None], norm_weight=w,
                          dstate_out=dsT[None])
    for t, want, name in zip((tq, tk, tv, tg), ref[:4], ("dq", "dk", "dv", "dg")):
        assert_close(to_host(t.grad), want, "bf16", name)
    assert_close(to_host(ts0.grad)[None], ref[4], "bf16", "dS0")
    assert_close(to_host(tw.grad), ref[5], "bf16", "dw")


def test_varlen_autograd_matches_oracle(cuda_device):
    """lightning_attention_varlen under loss.backward(): packed sequences (an empty and a
    one-token one among them) with initial states, final-state gradients, a trained norm
    weight and the gate, against the oracle's packed backward."""
    import torch
    from long_context_attn_b200.autograd import lightning_attention_varlen
    H, D = 8, 128
    lens = [300, 0, 257, 1, 129]
    cu = synth.cu_seqlens_of(lens)
    tot, n = int(cu[-1]), len(lens)
    q, k, v, g = synth.prefill_inputs(1461, tot, H, D, "bf16", 0.5, True)
    dout = synth.f32_to_bf16(synth.normal(1461, 11, (tot, H * D), 1.0, "f32"))
    s0 = synth.normal(1461, 9, (n, H, D, D), 0.05, "f32")
    dsT = synth.normal(1461, 10, (n, H, D, D), 0.05, "f32")
    w = (1.0 + 0.2 * synth.normal(1461, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    leaf = lambda a: to_dev(a).clone().requires_grad_(True)
    tq, tk, tv, tg, ts0, tw = (leaf(a) for a in (q, k, v, g, s0, w))
    out, st = lightning_attention_varlen(tq, tk, tv, torch.from_numpy(cu).cuda(), max(lens), g=tg, state_in=ts0,
                                         norm_weight=tw)
    loss = (out.float() * to_dev(dout).float()).sum() + (st * to_dev(dsT)).sum()
    loss.backward()
    ref = oracle.backward_packed(q, k, v, g, dout, cu, H, D, state_in=s0, norm_weight=w, dstate_out=dsT)
    for t, want, name in zip((tq, tk, tv, tg, ts0, tw), ref, ("dq", "dk", "dv", "dg", "dS0", "dw")):
        assert_close(to_host(t.grad), want, "bf16", name)
