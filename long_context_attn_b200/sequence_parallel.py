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

The last rank's state_out is the state after the whole sequence.  Every compute step runs
in the library's kernels; this module only orders the calls and the collective.
"""
from __future__ import annotations

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
    from it.  state0 [H, D, D] is the state before the whole sequence (None: zero)."""
    _, T, H, D = q.shape
    prefix = torch.empty((H, D, D), dtype=torch.float32, device=q.device)
    la.lightning_attn_state_prefix(gathered, rank, prefix, state0=state0, stream=stream)
    la.lightning_attn_prefill(q, k, v, g, out, prefix.view(1, H, D, D),
                              None if state_out is None else state_out.view(1, H, D, D), block_size=block_size,
                              phi=phi, mode=mode, eps=eps, norm_weight=norm_weight, workspace=workspace,
                              stream=stream)


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
    calls it with its own chunk, in the same order relative to other collectives."""
    _, T, H, D = q.shape
    if workspace is None:
        workspace = workspace_for(T, H, D, block_size, mode, q.device, la._dtype(q))
    local = chunk_state(k, v, workspace, phi, stream)
    gathered = all_gather(local)
    finish_chunk(q, k, v, g, out, gathered, rank, workspace, state0, state_out, block_size, phi, mode, eps,
                 norm_weight, stream)
