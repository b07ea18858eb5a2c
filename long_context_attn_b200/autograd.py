"""torch.autograd integration of the Lightning Attention forward and backward.

`lightning_attention(q, k, v, g, state_in=None, ...)` returns `(out, state_out)` like one
`lightning_attn_prefill` call and is differentiable in q, k, v, g, state_in and the norm
weight: its
backward is one `lightning_attn_backward` call (the gradient reaching `state_out`, when the
final state feeds later computation, is passed to it as dstate_out).  When gradients are
needed in a norm mode, the forward runs the prefill in raw mode and then the output
transform, keeping the raw output y, which saves the backward its recompute of y.  This
module only orders the library calls and allocates their outputs; every computation runs
in the library's kernels.
"""
from __future__ import annotations

import torch

from . import lightning_attn as la


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
