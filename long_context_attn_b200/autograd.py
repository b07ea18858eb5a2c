"""torch.autograd integration of the Lightning Attention forward and backward.

`lightning_attention(q, k, v, g, state_in=None, ...)` returns `(out, state_out)` like one
`lightning_attn_prefill` call (`lightning_attention_varlen` likewise for packed sequences,
`lightning_attention_sequence_parallel` for one rank's chunk of a sequence split across
ranks) and is differentiable in q, k, v, g, state_in and the norm weight: its backward is
one `lightning_attn_backward` call (the gradient reaching `state_out`, when the final state
feeds later computation, is passed to it as dstate_out).  When gradients are
needed in a norm mode, the forward runs the prefill in raw mode and then the output
transform, keeping the raw output y, which saves the backward its recompute of y.  This
module only orders the library calls and allocates their outputs; every computation runs
in the library's kernels.
"""
from __future__ import annotations

import torch

from . import lightning_attn as la
from . import sequence_parallel as sp


class _LightningAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, state_in, block_size, phi, mode, eps, norm_weight):
        B, T, H, D = q.shape
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        g = None if g is None else g.contiguous()
        out = torch.empty((B, T, H * D), dtype=q.dtype, device=q.device)
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
        s_in = None if state_in is None else state_in.detach().contiguous()
        keep_y = mode != la.LA_OUT_RAW and (any(ctx.needs_input_grad[:5]) or ctx.needs_input_grad[9])
        y = None
        if keep_y:   # raw prefill, then the norm (and gate) from the kept y
            y = torch.empty_like(out)
            ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, B, T, 0, H, D, block_size,
                                                                   la._dtype(q), la.LA_OUT_RAW), q.device)
            la.lightning_attn_prefill(q, k, v, None, y, s_in, state_out, block_size=block_size, phi=phi,
                                      mode=la.LA_OUT_RAW, workspace=ws)
            la.lightning_attn_output_transform(y.view(B, T, H, D), g, out, mode=mode, eps=eps,
                                               norm_weight=norm_weight)
        else:        # the fused kernel
            ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, B, T, 0, H, D, block_size,
                                                                   la._dtype(q), mode), q.device)
            la.lightning_attn_prefill(q, k, v, g, out, s_in, state_out, block_size=block_size, phi=phi, mode=mode,
                                      eps=eps, norm_weight=norm_weight, workspace=ws)
        ctx.save_for_backward(q, k, v, g, s_in, None if norm_weight is None else norm_weight.detach(), y)
        ctx.cfg = (block_size, phi, mode, eps)
        ctx.has_state = state_in is not None
        return out, state_out

    @staticmethod
    def backward(ctx, dout, dstate_out):
        q, k, v, g, s_in, norm_weight, y = ctx.saved_tensors
        block_size, phi, mode, eps = ctx.cfg
        B, T, H, D = q.shape
        if dout is None:
            dout = torch.zeros((B, T, H * D), dtype=q.dtype, device=q.device)
        dout = dout.to(q.dtype).contiguous()
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        dg = torch.empty_like(g) if mode == la.LA_OUT_RMSNORM_GATE else None
        ds_in = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device) if ctx.has_state else None
        dw = torch.empty((H * D,), dtype=torch.float32, device=q.device) if ctx.needs_input_grad[9] else None
        ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, B, T, 0, H, D, block_size,
                                                               la._dtype(q), mode), q.device)
        la.lightning_attn_backward(q, k, v, g if mode == la.LA_OUT_RMSNORM_GATE else None, dout, dq, dk, dv, dg=dg,
                                   state_in=s_in, dstate_in=ds_in, block_size=block_size, phi=phi, mode=mode,
                                   eps=eps, norm_weight=norm_weight, workspace=ws,
                                   dstate_out=None if dstate_out is None else dstate_out.float().contiguous(), y=y,
                                   dnorm_weight=dw)
        return dq, dk, dv, dg, ds_in, None, None, None, None, dw


def lightning_attention(q, k, v, g=None, state_in=None, block_size: int = 256, phi: int = la.LA_PHI_SILU,
                        mode: int = la.LA_OUT_RMSNORM_GATE, eps: float = 1e-6, norm_weight=None):
    """Differentiable prefill: q, k, v [B, T, H, D]; g [B, T, H*D] (gated mode); state_in fp32
    [B, H, D, D] or None; norm_weight [H*D] or None.  Returns (out [B, T, H*D], state_out
    fp32 [B, H, D, D])."""
    if norm_weight is not None:
        norm_weight = norm_weight.float().contiguous()
    return _LightningAttention.apply(q, k, v, g, state_in, block_size, phi, mode, eps, norm_weight)


class _LightningAttentionVarlen(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, state_in, cu_seqlens, max_seqlen, block_size, phi, mode, eps, norm_weight):
        total, H, D = q.shape
        N = cu_seqlens.numel() - 1
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        g = None if g is None else g.contiguous()
        out = torch.empty((total, H * D), dtype=q.dtype, device=q.device)
        state_out = torch.empty((N, H, D, D), dtype=torch.float32, device=q.device)
        s_in = None if state_in is None else state_in.detach().contiguous()
        keep_y = mode != la.LA_OUT_RAW and (any(ctx.needs_input_grad[:5]) or ctx.needs_input_grad[11])
        y = None
        if keep_y:   # raw prefill, then the norm (and gate) from the kept y
            y = torch.empty_like(out)
            ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_VARLEN, N, max_seqlen, total, H, D,
                                                                   block_size, la._dtype(q), la.LA_OUT_RAW), q.device)
            la.lightning_attn_prefill_varlen(q, k, v, None, y, cu_seqlens, max_seqlen, s_in, state_out,
                                             block_size=block_size, phi=phi, mode=la.LA_OUT_RAW, workspace=ws)
            la.lightning_attn_output_transform(y.view(total, H, D), g, out, mode=mode, eps=eps,
                                               norm_weight=norm_weight)
        else:        # the fused kernel
            ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_VARLEN, N, max_seqlen, total, H, D,
                                                                   block_size, la._dtype(q), mode), q.device)
            la.lightning_attn_prefill_varlen(q, k, v, g, out, cu_seqlens, max_seqlen, s_in, state_out,
                                             block_size=block_size, phi=phi, mode=mode, eps=eps,
                                             norm_weight=norm_weight, workspace=ws)
        ctx.save_for_backward(q, k, v, g, s_in, cu_seqlens, None if norm_weight is None else norm_weight.detach(), y)
        ctx.cfg = (max_seqlen, block_size, phi, mode, eps)
        ctx.has_state = state_in is not None
        return out, state_out

    @staticmethod
    def backward(ctx, dout, dstate_out):
        q, k, v, g, s_in, cu, norm_weight, y = ctx.saved_tensors
        max_seqlen, block_size, phi, mode, eps = ctx.cfg
        total, H, D = q.shape
        N = cu.numel() - 1
        if dout is None:
            dout = torch.zeros((total, H * D), dtype=q.dtype, device=q.device)
        dout = dout.to(q.dtype).contiguous()
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        dg = torch.empty_like(g) if mode == la.LA_OUT_RMSNORM_GATE else None
        ds_in = torch.empty((N, H, D, D), dtype=torch.float32, device=q.device) if ctx.has_state else None
        dw = torch.empty((H * D,), dtype=torch.float32, device=q.device) if ctx.needs_input_grad[11] else None
        ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_BACKWARD_VARLEN, N, max_seqlen, total, H, D,
                                                               block_size, la._dtype(q), mode), q.device)
        la.lightning_attn_backward_varlen(q, k, v, g if mode == la.LA_OUT_RMSNORM_GATE else None, dout, dq, dk, dv, cu,
                                          max_seqlen, dg=dg, state_in=s_in, dstate_in=ds_in, block_size=block_size,
                                          phi=phi, mode=mode, eps=eps, norm_weight=norm_weight, workspace=ws,
                                          dstate_out=None if dstate_out is None else dstate_out.float().contiguous(),
                                          y=y, dnorm_weight=dw)
        return dq, dk, dv, dg, ds_in, None, None, None, None, None, None, dw


def lightning_attention_varlen(q, k, v, cu_seqlens, max_seqlen: int, g=None, state_in=None, block_size: int = 256,
                               phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE, eps: float = 1e-6,
                               norm_weight=None):
    """Differentiable packed prefill: q, k, v [total, H, D] of N sequences (cu_seqlens int32
    device [N + 1], max_seqlen its longest); g [total, H*D] (gated mode); state_in fp32
    [N, H, D, D] or None.  Returns (out [total, H*D], state_out fp32 [N, H, D, D])."""
    if norm_weight is not None:
        norm_weight = norm_weight.float().contiguous()
    return _LightningAttentionVarlen.apply(q, k, v, g, state_in, cu_seqlens, int(max_seqlen), block_size, phi, mode,
                                           eps, norm_weight)


class _SequenceParallelLightningAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, state0, norm_weight, rank, all_gather, block_size, phi, mode, eps):
        _, T, H, D = q.shape
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        g = None if g is None else g.contiguous()
        s0 = None if state0 is None else state0.detach().contiguous()
        w = None if norm_weight is None else norm_weight.detach().contiguous()
        out = torch.empty((1, T, H * D), dtype=q.dtype, device=q.device)
        state_end = torch.empty((H, D, D), dtype=torch.float32, device=q.device)
        ws = sp.workspace_for(T, H, D, block_size, mode, q.device, la._dtype(q))
        y = None
        if mode != la.LA_OUT_RAW and any(ctx.needs_input_grad[:6]):   # keep the raw output for the backward
            y = torch.empty_like(out)
            prefix = sp.prefill_sequence_parallel(q, k, v, None, y, rank, all_gather, state0=s0, state_out=state_end,
                                                  block_size=block_size, phi=phi, mode=la.LA_OUT_RAW, workspace=ws)
            la.lightning_attn_output_transform(y.view(1, T, H, D), g, out, mode=mode, eps=eps, norm_weight=w)
        else:
            prefix = sp.prefill_sequence_parallel(q, k, v, g, out, rank, all_gather, state0=s0, state_out=state_end,
                                                  block_size=block_size, phi=phi, mode=mode, eps=eps, norm_weight=w,
                                                  workspace=ws)
        ctx.save_for_backward(q, k, v, g, prefix, w, y)
        ctx.cfg = (rank, all_gather, block_size, phi, mode, eps, state0 is not None)
        return out, state_end

    @staticmethod
    def backward(ctx, dout, dstate_end):
        q, k, v, g, prefix, w, y = ctx.saved_tensors
        rank, all_gather, block_size, phi, mode, eps, has_s0 = ctx.cfg
        _, T, H, D = q.shape
        if dout is None:
            dout = torch.zeros((1, T, H * D), dtype=q.dtype, device=q.device)
        dout = dout.to(q.dtype).contiguous()
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        dg = torch.empty_like(g) if mode == la.LA_OUT_RMSNORM_GATE else None
        dw = torch.empty((H * D,), dtype=torch.float32, device=q.device) if ctx.needs_input_grad[5] else None
        ds_in = torch.empty((H, D, D), dtype=torch.float32, device=q.device) if has_s0 else None
        sp.backward_sequence_parallel(q, k, v, g, dout, dq, dk, dv, rank, prefix, all_gather,
                                      dstate_end=None if dstate_end is None else dstate_end.float().contiguous(),
                                      y=y, dg=dg, dnorm_weight=dw, dstate_in=ds_in, block_size=block_size, phi=phi,
                                      mode=mode, eps=eps, norm_weight=w)
        # state0 is the same tensor on every rank: rank 0 returns its whole gradient and the
        # others zero, so that adding the ranks' gradients (as for the norm weight's per-chunk
        # parts) gives the total
        if ds_in is not None and rank != 0:
            ds_in.zero_()
        return dq, dk, dv, dg, ds_in, dw, None, None, None, None, None, None


def lightning_attention_sequence_parallel(q, k, v, g=None, state0=None, norm_weight=None, rank: int = 0,
                                          all_gather=sp.nccl_all_gather, block_size: int = 256,
                                          phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE,
                                          eps: float = 1e-6):
    """Differentiable sequence-parallel prefill: this rank's contiguous chunk q, k, v
    [1, T, H, D] (g [1, T, H*D]) of one sequence split across the group's ranks in order.
    Returns (out [1, T, H*D], the state at the end of this chunk fp32 [H, D, D]: on the last
    rank the sequence's final state).  One all-gather in the forward and one in the backward,
    so every rank must call it in the same order and back-propagate through its output.
    Gradients of state0 and the norm weight (the same tensors on every rank) come as per-rank
    parts to be added over the ranks, as data-parallel gradients are."""
    if norm_weight is not None:
        norm_weight = norm_weight.float().contiguous()
    return _SequenceParallelLightningAttention.apply(q, k, v, g, state0, norm_weight, rank, all_gather, block_size,
                                                     phi, mode, eps)
