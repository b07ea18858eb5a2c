"""Sequence-parallel Lightning Attention prefill: one long sequence split across ranks.

"MiniMax-01系列大模型：超长上下文与多模态能力深度解析与部署指南", section 2.1.3 names LASP+,
the sequence parallelism made for Lightning Attention, without giving its steps.  What it
rests on is the state recurrence of "六十四：MiniMax-01" section 3: S_t = S0 + sum over
i <= t of phi(k_i) v_i^T is a plain sum, so rank r, holding the contiguous chunk r of the
sequence, needs only the sum of the earlier chunks' states:

  1. chunk_state: the state this chunk reaches from a zero state (lightning_attn_chunk_state:
     phi(K)^T V accumulated on the tensor cores from k and v alone, no outputs);
  2. one all-gather of the [H, D, D] fp32 chunk states (NCCL over NVLink in a job);
  3. finish_chunk: the prefix state0 + sum_{j < r} state_j (lightning_attn_state_prefix, in
     rank order), then the chunk's prefill from that prefix with the requested output mode
     (the RMSNorm over the head concatenation is per token, so it needs no exchange).

The last rank's state_out is the state after the whole sequence.

The same section's variable-length batches (sequences of different lengths handed along
the ranks like a relay) take the same three steps over a packed batch: the token stream of
N sequences (cu_seqlens) is cut into contiguous rank slices (`bounds`), so a sequence may
start on one rank and end several ranks later.  Each rank's slice holds pieces of
consecutive sequences; only its first piece can continue a sequence from earlier ranks and
only its last piece can continue onto later ones.  Step 1 is the state that last piece
reaches from a zero state (zero when its sequence ends on this rank); step 2 the same
all-gather; in step 3 the first piece starts from state0 of its sequence plus the gathered
states of the ranks from the one where that sequence starts up to this one (in rank order),
and the slice runs as one varlen prefill with a state per piece.  The relay is one
collective step, not a chain of hops, because every rank's contribution is computed from a
zero state.

The backward (training used LASP+ as well) needs one exchange too: the gradient reaching
the end of chunk r is the final-state gradient plus, for each later chunk, the sum over
its tokens of phi(q_t) dy_t^T, which every rank computes from its own chunk (the chunk-state
kernel with q as keys and dy as values); after one all-gather each rank adds the later
ranks' sums and runs its chunk's backward (backward_sequence_parallel).

Every compute step runs in the library's kernels; this module only orders the calls and
the collective (and allocates or slices the state buffers).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import lightning_attn as la


def workspace_for(T: int, H: int, D: int, block_size: int = 256, mode: int = la.LA_OUT_RMSNORM_GATE,
                  device="cuda", dtype: int = la.LA_BF16) -> torch.Tensor:
    """One workspace that serves both steps of a chunk of T tokens (calls run one after another)."""
    n = max(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, 1, T, 0, H, D, block_size, dtype, mode),
            la.lightning_attn_workspace_size(la.LA_OP_CHUNK_STATE, 1, T, 0, H, D, 0, dtype, 0))
    return la.new_workspace(n, device)


def chunk_state(k, v, workspace, phi: int = la.LA_PHI_SILU, stream=None):
    """Step 1: the chunk's state from a zero state.  k, v [1, T, H, D].  Returns fp32 [H, D, D]."""
    _, T, H, D = k.shape
    state = torch.empty((1, H, D, D), dtype=torch.float32, device=k.device)
    la.lightning_attn_chunk_state(k, v, state, phi=phi, workspace=workspace, stream=stream)
    return state[0]


def finish_chunk(q, k, v, g, out, gathered, rank: int, workspace, state0=None, state_out=None,
                 block_size: int = 256, phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE,
                 eps: float = 1e-6, norm_weight=None, stream=None):
    """Step 3: prefix the gathered chunk states [world, H, D, D] for `rank` and prefill the chunk
    from it.  state0 [H, D, D] is the state before the whole sequence (None: zero).  Returns the
    prefix (fp32 [H, D, D], the state the chunk started from; the backward takes it)."""
    _, T, H, D = q.shape
    prefix = torch.empty((H, D, D), dtype=torch.float32, device=q.device)
    la.lightning_attn_state_prefix(gathered, rank, prefix, state0=state0, stream=stream)
    la.lightning_attn_prefill(q, k, v, g, out, prefix.view(1, H, D, D),
                              None if state_out is None else state_out.view(1, H, D, D), block_size=block_size,
                              phi=phi, mode=mode, eps=eps, norm_weight=norm_weight, workspace=workspace,
                              stream=stream)
    return prefix


def nccl_all_gather(state: torch.Tensor, group=None) -> torch.Tensor:
    """Step 2 over torch.distributed: [H, D, D] per rank -> [world, H, D, D] in rank order
    (one all_gather_into_tensor over NCCL; a list all_gather on other backends)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world,) + tuple(state.shape), dtype=state.dtype, device=state.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, state.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), state.contiguous(), group=group)
    return out


def prefill_sequence_parallel(q, k, v, g, out, rank: int, all_gather=nccl_all_gather, state0=None,
                              state_out=None, block_size: int = 256, phi: int = la.LA_PHI_SILU,
                              mode: int = la.LA_OUT_RMSNORM_GATE, eps: float = 1e-6, norm_weight=None,
                              workspace=None, stream=None):
    """This rank's part of a sequence-parallel prefill (steps 1-3).  Every rank of the group
    calls it with its own chunk, in the same order relative to other collectives.  Returns the
    state the chunk started from (fp32 [H, D, D])."""
    _, T, H, D = q.shape
    if workspace is None:
        workspace = workspace_for(T, H, D, block_size, mode, q.device, la._dtype(q))
    local = chunk_state(k, v, workspace, phi, stream)
    gathered = all_gather(local)
    return finish_chunk(q, k, v, g, out, gathered, rank, workspace, state0, state_out, block_size, phi, mode, eps,
                        norm_weight, stream)


def backward_workspace_for(T: int, H: int, D: int, block_size: int = 256, mode: int = la.LA_OUT_RMSNORM_GATE,
                           device="cuda", dtype: int = la.LA_BF16) -> torch.Tensor:
    """One workspace for every call of backward_sequence_parallel on a chunk of T tokens."""
    n = max(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, 1, T, 0, H, D, block_size, dtype, la.LA_OUT_RAW),
            la.lightning_attn_workspace_size(la.LA_OP_CHUNK_STATE, 1, T, 0, H, D, 0, dtype, 0),
            la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, 1, T, 0, H, D, block_size, dtype, la.LA_OUT_RAW),
            la.lightning_attn_workspace_size(la.LA_OP_OUTPUT_TRANSFORM_BACKWARD, T, 0, 0, H, D, 0, dtype, mode))
    return la.new_workspace(n, device)


def backward_local(q, k, v, g, dout, prefix, workspace, y=None, dg=None, dnorm_weight=None, dstate_end=None,
                   block_size: int = 256, phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE,
                   eps: float = 1e-6, norm_weight=None, stream=None):
    """Backward steps 1-2 on this rank's chunk: dy (and dg, this chunk's terms of dw) from dout
    through the output transform of the chunk's raw output y (given, or recomputed from
    `prefix`), then this rank's contribution to the earlier ranks' end-of-chunk gradients:
    G = dstate_end + sum over the chunk of phi(q_t) dy_t^T (the chunk-state kernel with q as
    the keys, dy as the values and dstate_end, the gradient of the state at the end of this
    chunk from outside, as its initial state).  Returns (dy [1, T, H*D], G fp32 [H, D, D])."""
    _, T, H, D = q.shape
    if mode == la.LA_OUT_RAW:
        dy = dout
        if dnorm_weight is not None:
            dnorm_weight.zero_()
    else:
        if y is None:
            y = torch.empty_like(dout)
            la.lightning_attn_prefill(q, k, v, None, y, prefix.view(1, H, D, D), None, block_size=block_size, phi=phi,
                                      mode=la.LA_OUT_RAW, workspace=workspace, stream=stream)
        dy = torch.empty_like(dout)
        la.lightning_attn_output_transform_backward(y.view(1, T, H, D), g, dout, dy, dg=dg, dnorm_weight=dnorm_weight,
                                                    mode=mode, eps=eps, norm_weight=norm_weight, workspace=workspace,
                                                    stream=stream)
    G = torch.empty((1, H, D, D), dtype=torch.float32, device=q.device)
    la.lightning_attn_chunk_state(q, dy.view(1, T, H, D), G, None if dstate_end is None else dstate_end.view(1, H, D, D),
                                  phi=phi, workspace=workspace, stream=stream)
    return dy, G[0]


def backward_finish(q, k, v, dy, dq, dk, dv, gathered, rank: int, prefix, workspace, dstate_end=None,
                    dstate_in=None, block_size: int = 256, phi: int = la.LA_PHI_SILU, stream=None):
    """Backward steps 3-4: the gradient reaching the end of the chunk, dstate_end + sum_{j > rank}
    of the gathered G_j [world, H, D, D] (added from the last rank down), then the chunk's
    backward in raw mode from dy with its initial state `prefix`."""
    _, T, H, D = q.shape
    world = gathered.shape[0]
    later_first = torch.flip(gathered, dims=[0]).contiguous()   # rank world-1 first
    ds_end = torch.empty((H, D, D), dtype=torch.float32, device=q.device)
    la.lightning_attn_state_prefix(later_first, world - 1 - rank, ds_end, state0=dstate_end, stream=stream)
    st = lambda x: None if x is None else x.view(1, H, D, D)
    la.lightning_attn_backward(q, k, v, None, dy, dq, dk, dv, state_in=st(prefix), dstate_in=st(dstate_in),
                               block_size=block_size, phi=phi, mode=la.LA_OUT_RAW, workspace=workspace,
                               stream=stream, dstate_out=st(ds_end))


def backward_sequence_parallel(q, k, v, g, dout, dq, dk, dv, rank: int, prefix, all_gather=nccl_all_gather,
                               dstate_end=None, y=None, dg=None, dnorm_weight=None, dstate_in=None,
                               block_size: int = 256, phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE,
                               eps: float = 1e-6, norm_weight=None, workspace=None, stream=None):
    """This rank's part of the backward of prefill_sequence_parallel.

    With X_j the gradient that reaches the state at the end of chunk j from outside (on the
    last rank the gradient of the sequence's final state; elsewhere zero unless the caller
    used that state) and G_j = sum over chunk j of phi(q_t) dy_t^T (the part of chunk j's
    initial-state gradient that its own tokens give), the gradient reaching the end of
    chunk r is X_r + sum_{j > r} (G_j + X_j): after one all-gather of the G_j + X_j every rank
    runs its chunk's backward on its own (backward_local, the all-gather, backward_finish).
    q, k, v, dq, dk, dv [1, T, H, D]; g, dout, dg [1, T, H*D]; prefix (the state the chunk
    started from, as prefill_sequence_parallel returns it), dstate_end (X_r, None for zero),
    dstate_in fp32 [H, D, D] (rank 0's dstate_in is the gradient of the sequence's initial
    state); y: the chunk's raw output if kept; dnorm_weight fp32 [H*D] receives this chunk's
    part of the norm weight's gradient (sum it over the ranks)."""
    _, T, H, D = q.shape
    if workspace is None:
        workspace = backward_workspace_for(T, H, D, block_size, mode, q.device, la._dtype(q))
    dy, G = backward_local(q, k, v, g, dout, prefix, workspace, y, dg, dnorm_weight, dstate_end, block_size, phi,
                           mode, eps, norm_weight, stream)
    gathered = all_gather(G)
    backward_finish(q, k, v, dy, dq, dk, dv, gathered, rank, prefix, workspace, dstate_end, dstate_in, block_size,
                    phi, stream)


@dataclass
class VarlenSlice:
    """One rank's share of a packed batch cut into contiguous rank slices.

    lo, hi        the slice's tokens [lo, hi) of the packed stream
    seq           the sequences with a piece here (consecutive indices, in order)
    local_cu      int32 [len(seq) + 1]: the pieces' boundaries relative to lo
    max_len       the longest piece
    first_from    the rank where the first piece's sequence starts, when that is an earlier
                  rank (the piece continues it), else None
    carries       True when the last piece's sequence goes on past hi
    final         per piece: its sequence ends on this rank (its state after the piece is
                  the sequence's final state)
    """
    lo: int
    hi: int
    seq: list
    local_cu: np.ndarray
    max_len: int
    first_from: int | None
    carries: bool
    final: list


def varlen_slice_plan(cu_seqlens, bounds, rank: int) -> VarlenSlice:
    """Host-side plan of rank `rank`'s slice.  cu_seqlens [N + 1] (host, non-decreasing from
    0) packs N sequences; bounds [world + 1] (non-decreasing from 0 to cu_seqlens[-1]) gives
    rank r the tokens [bounds[r], bounds[r + 1]).  An empty sequence belongs to the rank whose
    slice holds its position (the last rank when it sits at the end of the stream)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    b = np.asarray(bounds, dtype=np.int64)
    if cu.ndim != 1 or cu.size < 1 or cu[0] != 0 or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must be non-decreasing from 0")
    if b.ndim != 1 or b.size < 2 or b[0] != 0 or b[-1] != cu[-1] or np.any(np.diff(b) < 0):
        raise ValueError("bounds must be non-decreasing from 0 to the total token count")
    world = b.size - 1
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    lo, hi = int(b[rank]), int(b[rank + 1])

    def owner(pos):   # the rank whose slice holds token position pos
        return min(int(np.searchsorted(b, pos, side="right")) - 1, world - 1)

    seq, edges, final = [], [], []
    first_from, carries = None, False
    for s in range(cu.size - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        if a == e:
            if owner(a) == rank:
                seq.append(s)
                edges.append((a, a))
                final.append(True)
            continue
        x, y = max(a, lo), min(e, hi)
        if x >= y:
            continue
        if not seq and a < lo:
            first_from = owner(a)
        seq.append(s)
        edges.append((x, y))
        final.append(e <= hi)
    if seq and not final[-1]:
        carries = True
    local_cu = np.array([0] + [y - lo for _, y in edges], dtype=np.int32)
    max_len = max([y - x for x, y in edges], default=0)
    return VarlenSlice(lo, hi, seq, local_cu, max_len, first_from, carries, final)


def varlen_workspace_for(plan: VarlenSlice, H: int, D: int, block_size: int = 256,
                         mode: int = la.LA_OUT_RMSNORM_GATE, device="cuda", dtype: int = la.LA_BF16):
    """One workspace for the slice's chunk-state call and its varlen prefill."""
    n = 256
    if plan.seq:
        n = max(n, la.lightning_attn_workspace_size(la.LA_OP_PREFILL_VARLEN, len(plan.seq), plan.max_len,
                                                    plan.hi - plan.lo, H, D, block_size, dtype, mode))
    if plan.carries:
        last = int(plan.local_cu[-1] - plan.local_cu[-2])
        n = max(n, la.lightning_attn_workspace_size(la.LA_OP_CHUNK_STATE, 1, last, 0, H, D, 0, dtype, 0))
    return la.new_workspace(n, device)


def varlen_carry(k, v, plan: VarlenSlice, workspace, phi: int = la.LA_PHI_SILU, stream=None):
    """Step 1: the state the slice's last piece reaches from a zero state when its sequence
    continues on a later rank, else zero.  k, v [L, H, D] (this slice).  Returns fp32 [H, D, D]."""
    _, H, D = k.shape
    state = torch.zeros((1, H, D, D), dtype=torch.float32, device=k.device)
    if plan.carries:
        a, e = int(plan.local_cu[-2]), int(plan.local_cu[-1])
        la.lightning_attn_chunk_state(k[a:e][None], v[a:e][None], state, phi=phi, workspace=workspace,
                                      stream=stream)
    return state[0]


def varlen_initial_states(plan: VarlenSlice, gathered, rank: int, state0=None, device="cuda", stream=None):
    """The initial state of every piece of the slice, fp32 [len(plan.seq), H, D, D] (None when
    all are zero): state0 of its sequence, and for a first piece that continues a sequence,
    plus the gathered states [world, H, D, D] of the ranks from the one where that sequence
    starts up to this one."""
    m = len(plan.seq)
    if m == 0:
        return None
    _, H, D, _ = gathered.shape
    s0 = plan.seq[0]
    st_in = None if state0 is None else state0[s0:s0 + m]
    if plan.first_from is not None:
        st_in = (torch.zeros((m, H, D, D), dtype=torch.float32, device=device) if st_in is None
                 else st_in.clone())
        r0 = plan.first_from
        la.lightning_attn_state_prefix(gathered[r0:rank + 1], rank - r0, st_in[0],
                                       state0=None if state0 is None else state0[s0], stream=stream)
    return st_in


def varlen_finish(q, k, v, g, out, gathered, plan: VarlenSlice, rank: int, workspace, state0=None,
                  block_size: int = 256, phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE,
                  eps: float = 1e-6, norm_weight=None, stream=None):
    """Step 3: the slice's varlen prefill, every piece from its initial state
    (varlen_initial_states).  q, k, v [L, H, D]; g, out [L, H*D]; state0 fp32 [N, H, D, D] (all
    sequences; None: zero).  Returns (the states after each piece, fp32 [len(plan.seq), H, D, D]
    -- the sequences' final states where plan.final --, the pieces' initial states or None)."""
    _, H, D = q.shape
    m = len(plan.seq)
    st_out = torch.empty((m, H, D, D), dtype=torch.float32, device=q.device)
    if m == 0:
        return st_out, None
    st_in = varlen_initial_states(plan, gathered, rank, state0, q.device, stream)
    if plan.hi == plan.lo:   # only empty sequences: each keeps its initial state
        if st_in is None:
            st_out.zero_()
        else:
            st_out.copy_(st_in)
        return st_out, st_in
    cu = torch.from_numpy(plan.local_cu).to(q.device)
    la.lightning_attn_prefill_varlen(q, k, v, g, out, cu, plan.max_len, state_in=st_in, state_out=st_out,
                                     block_size=block_size, phi=phi, mode=mode, eps=eps, norm_weight=norm_weight,
                                     workspace=workspace, stream=stream)
    return st_out, st_in


def prefill_varlen_sequence_parallel(q, k, v, g, out, cu_seqlens, bounds, rank: int, all_gather=nccl_all_gather,
                                     state0=None, block_size: int = 256, phi: int = la.LA_PHI_SILU,
                                     mode: int = la.LA_OUT_RMSNORM_GATE, eps: float = 1e-6, norm_weight=None,
                                     workspace=None, stream=None):
    """This rank's part of a sequence-parallel prefill of a packed batch (steps 1-3).
    cu_seqlens and bounds are host arrays, the same on every rank; q, k, v [L, H, D] and g,
    out [L, H*D] hold this rank's slice.  Returns (plan, the states after each piece, the
    pieces' initial states or None -- the backward takes them)."""
    _, H, D = q.shape
    plan = varlen_slice_plan(cu_seqlens, bounds, rank)
    if q.shape[0] != plan.hi - plan.lo:
        raise ValueError("q holds %d tokens, the slice %d" % (q.shape[0], plan.hi - plan.lo))
    if workspace is None:
        workspace = varlen_workspace_for(plan, H, D, block_size, mode, q.device, la._dtype(q))
    carry = varlen_carry(k, v, plan, workspace, phi, stream)
    gathered = all_gather(carry)
    st_out, st_in = varlen_finish(q, k, v, g, out, gathered, plan, rank, workspace, state0, block_size, phi, mode,
                                  eps, norm_weight, stream)
    return plan, st_out, st_in


def varlen_backward_workspace_for(plan: VarlenSlice, H: int, D: int, block_size: int = 256,
                                  mode: int = la.LA_OUT_RMSNORM_GATE, device="cuda", dtype: int = la.LA_BF16):
    """One workspace for every call of the packed-batch backward on this slice."""
    n, L, m = 256, plan.hi - plan.lo, len(plan.seq)
    if m:
        n = max(n, la.lightning_attn_workspace_size(la.LA_OP_PREFILL_VARLEN, m, plan.max_len, L, H, D, block_size,
                                                    dtype, la.LA_OUT_RAW),
                la.lightning_attn_workspace_size(la.LA_OP_BACKWARD_VARLEN, m, plan.max_len, L, H, D, block_size,
                                                 dtype, la.LA_OUT_RAW),
                la.lightning_attn_workspace_size(la.LA_OP_OUTPUT_TRANSFORM_BACKWARD, L, 0, 0, H, D, 0, dtype, mode))
    if plan.first_from is not None:
        first = int(plan.local_cu[1])
        n = max(n, la.lightning_attn_workspace_size(la.LA_OP_CHUNK_STATE, 1, first, 0, H, D, 0, dtype, 0))
    return la.new_workspace(n, device)


def varlen_backward_local(q, k, v, g, dout, plan: VarlenSlice, st_in, workspace, y=None, dg=None, dnorm_weight=None,
                          block_size: int = 256, phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE,
                          eps: float = 1e-6, norm_weight=None, stream=None):
    """Backward steps 1-2 on this rank's slice of a packed batch: dy (and dg, the slice's terms
    of dw) through the output transform of the slice's raw output y (given, or recomputed from
    the pieces' initial states st_in), then G = sum of phi(q_t) dy_t^T over the first piece
    when it continues a sequence from an earlier rank (zero otherwise: the sums that later
    ranks need only come from pieces that continue a sequence).  q, k, v [L, H, D]; g, dout
    [L, H*D].  Returns (dy [L, H*D], G fp32 [H, D, D])."""
    L, H, D = q.shape
    if mode == la.LA_OUT_RAW:
        dy = dout
        if dnorm_weight is not None:
            dnorm_weight.zero_()
    else:
        if y is None:
            y = torch.empty_like(dout)
            if L:
                cu = torch.from_numpy(plan.local_cu).to(q.device)
                la.lightning_attn_prefill_varlen(q, k, v, None, y, cu, plan.max_len, state_in=st_in,
                                                 block_size=block_size, phi=phi, mode=la.LA_OUT_RAW,
                                                 workspace=workspace, stream=stream)
        dy = torch.empty_like(dout)
        la.lightning_attn_output_transform_backward(y.view(L, H, D), g, dout, dy, dg=dg, dnorm_weight=dnorm_weight,
                                                    mode=mode, eps=eps, norm_weight=norm_weight, workspace=workspace,
                                                    stream=stream)
    G = torch.zeros((1, H, D, D), dtype=torch.float32, device=q.device)
    if plan.first_from is not None:
        e = int(plan.local_cu[1])
        la.lightning_attn_chunk_state(q[:e][None], dy[:e].view(1, e, H, D), G, phi=phi, workspace=workspace,
                                      stream=stream)
    return dy, G[0]


def varlen_backward_finish(q, k, v, dy, dq, dk, dv, gathered, plan: VarlenSlice, cu_seqlens, bounds, rank: int, st_in,
                           workspace, dstate_out=None, dstate_in=None, block_size: int = 256,
                           phi: int = la.LA_PHI_SILU, stream=None):
    """Backward steps 3-4: each piece's end-of-piece gradient -- dstate_out of its sequence
    (fp32 [N, H, D, D] for all sequences, None: zero), plus, for a last piece whose sequence
    goes on, the gathered sums [world, H, D, D] of the later ranks up to the one holding the
    sequence's last token -- then the slice's backward in raw mode from dy with the pieces'
    initial states st_in.  dstate_in (fp32 [len(plan.seq), H, D, D] or None) receives each
    piece's initial-state gradient (for a piece that starts its sequence, the gradient of
    that sequence's initial state)."""
    L, H, D = q.shape
    m = len(plan.seq)
    if m == 0:
        return
    s0 = plan.seq[0]
    ds_end = None if dstate_out is None else dstate_out[s0:s0 + m]
    if plan.carries:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        b = np.asarray(bounds, dtype=np.int64)
        s_last = plan.seq[-1]
        r_end = int(np.searchsorted(b, cu[s_last + 1] - 1, side="right")) - 1   # holds the last token
        later = gathered[rank + 1:r_end + 1]
        ds_end = (torch.zeros((m, H, D, D), dtype=torch.float32, device=q.device) if ds_end is None
                  else ds_end.clone())
        pad = torch.cat([later, torch.zeros((1, H, D, D), dtype=torch.float32, device=q.device)])
        la.lightning_attn_state_prefix(pad, later.shape[0], ds_end[m - 1],
                                       state0=None if dstate_out is None else dstate_out[s_last], stream=stream)
    if L == 0:   # only empty sequences: the initial-state gradient is the final one
        if dstate_in is not None:
            if ds_end is None:
                dstate_in.zero_()
            else:
                dstate_in.copy_(ds_end)
        return
    cu_local = torch.from_numpy(plan.local_cu).to(q.device)
    la.lightning_attn_backward_varlen(q, k, v, None, dy, dq, dk, dv, cu_local, plan.max_len, state_in=st_in,
                                      dstate_in=dstate_in, block_size=block_size, phi=phi, mode=la.LA_OUT_RAW,
                                      workspace=workspace, stream=stream, dstate_out=ds_end)


def backward_varlen_sequence_parallel(q, k, v, g, dout, dq, dk, dv, cu_seqlens, bounds, rank: int, st_in,
                                      all_gather=nccl_all_gather, dstate_out=None, y=None, dg=None,
                                      dnorm_weight=None, dstate_in=None, block_size: int = 256,
                                      phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE,
                                      eps: float = 1e-6, norm_weight=None, workspace=None, stream=None):
    """This rank's part of the backward of prefill_varlen_sequence_parallel: st_in is the
    pieces' initial states it returned; dstate_out fp32 [N, H, D, D] (all sequences, the same
    on every rank) or None; dstate_in fp32 [len(plan.seq), H, D, D] or None; dnorm_weight
    receives this slice's part of the norm weight's gradient (sum it over the ranks).
    Returns the plan."""
    L, H, D = q.shape
    plan = varlen_slice_plan(cu_seqlens, bounds, rank)
    if L != plan.hi - plan.lo:
        raise ValueError("q holds %d tokens, the slice %d" % (L, plan.hi - plan.lo))
    if workspace is None:
        workspace = varlen_backward_workspace_for(plan, H, D, block_size, mode, q.device, la._dtype(q))
    dy, G = varlen_backward_local(q, k, v, g, dout, plan, st_in, workspace, y, dg, dnorm_weight, block_size, phi,
                                  mode, eps, norm_weight, stream)
    gathered = all_gather(G)
    varlen_backward_finish(q, k, v, dy, dq, dk, dv, gathered, plan, cu_seqlens, bounds, rank, st_in, workspace,
                           dstate_out, dstate_in, block_size, phi, stream)
    return plan
