"""Prefill of one long sequence that lives in host memory, with the copies overlapped.

A 131072-token, 64-head bf16 prefill reads 8.6 GB of q, k, v and gate and writes 2.1 GB of
output, so a call that starts and ends in host memory is bound by the PCIe link, not by the
4.7 ms kernel.  `HostPrefill` cuts the sequence into chunks and pipelines them over three
CUDA streams: chunk i+1's host-to-device copies, chunk i's prefill (continuing from the
state chunk i-1 left, kept on the device: "六十四：MiniMax-01" section 3's S is carried from
block to block, so a chunk boundary is just a block boundary with the state in HBM) and
chunk i-1's device-to-host copy of its output run at the same time, through two sets of
device buffers.  Host-to-device and device-to-host traffic then overlap (the link is full
duplex), and the kernel time hides behind the copies.

Every compute step is one lightning_attn_prefill call; this module only moves memory and
orders streams.  Host tensors must be pinned (page-locked), or the copies are synchronous;
synchronise the call's stream before dropping a HostPrefill whose copies may be in flight.
"""
from __future__ import annotations

import torch

from . import lightning_attn as la


class HostPrefill:
    """Reusable device buffers and streams for host-memory prefills of H heads of any length.

    chunk_tokens: tokens per pipelined chunk (a multiple of the block size is best; the
    last chunk may be shorter).  Other arguments as lightning_attn_prefill."""

    def __init__(self, H: int, D: int, chunk_tokens: int = 16384, block_size: int = 256,
                 phi: int = la.LA_PHI_SILU, mode: int = la.LA_OUT_RMSNORM_GATE, eps: float = 1e-6,
                 norm_weight=None, dtype=torch.bfloat16, device="cuda"):
        if chunk_tokens < 1:
            raise ValueError("chunk_tokens must be positive")
        self.H, self.D, self.chunk = H, D, chunk_tokens
        self.block_size, self.phi, self.mode, self.eps = block_size, phi, mode, eps
        self.norm_weight = norm_weight
        self.device = torch.device(device)
        n = chunk_tokens
        self.q = [torch.empty((n, H, D), dtype=dtype, device=device) for _ in range(2)]
        self.k = [torch.empty((n, H, D), dtype=dtype, device=device) for _ in range(2)]
        self.v = [torch.empty((n, H, D), dtype=dtype, device=device) for _ in range(2)]
        self.g = [torch.empty((n, H * D), dtype=dtype, device=device) for _ in range(2)]
        self.out = [torch.empty((n, H * D), dtype=dtype, device=device) for _ in range(2)]
        self.state = torch.empty((1, H, D, D), dtype=torch.float32, device=device)
        self.dt = la.LA_BF16 if dtype == torch.bfloat16 else la.LA_F32
        self.ws = la.new_workspace(self._ws_bytes(n), device)
        self.h2d = torch.cuda.Stream(device=self.device)
        self.d2h = torch.cuda.Stream(device=self.device)
        self.last = None   # the stream the previous call ran its prefills on

    def _ws_bytes(self, tokens):
        return la.lightning_attn_workspace_size(la.LA_OP_PREFILL, 1, tokens, 0, self.H, self.D, self.block_size,
                                                self.dt, self.mode)

    def __call__(self, q, k, v, g, out, state_in=None, state_out=None, stream=None):
        """q, k, v [T, H, D] and g, out [T, H*D] in pinned host memory (g None unless the gated
        mode); state_in, state_out fp32 [H, D, D] on the device or None.  Enqueued on `stream`
        (default: the current stream), which waits for every copy: synchronise it before
        reading `out`."""
        T = q.shape[0]
        H, D, n = self.H, self.D, self.chunk
        if q.shape != (T, H, D) or k.shape != q.shape or v.shape != q.shape or out.shape != (T, H * D):
            raise ValueError("q, k, v must be [T, H, D] and out [T, H*D]")
        gated = self.mode == la.LA_OUT_RMSNORM_GATE
        if gated and (g is None or g.shape != (T, H * D)):
            raise ValueError("the gated mode needs g [T, H*D]")
        compute = stream if stream is not None else torch.cuda.current_stream(self.device)
        if T % n and self._ws_bytes(T % n) > self.ws.numel():   # a tail chunk that needs more workspace
            if self.last is not None:
                self.last.synchronize()
            self.ws = la.new_workspace(self._ws_bytes(T % n), self.device)
        # buffers made (and the workspace zero-filled) on the current stream come first
        compute.wait_stream(torch.cuda.current_stream(self.device))
        # the buffers are free once the caller's earlier work and the previous call are done
        for s in (self.h2d, self.d2h):
            s.wait_stream(compute)
            if self.last is not None and self.last != compute:
                s.wait_stream(self.last)
        self.last = compute
        have_state = state_in is not None
        if have_state:
            with torch.cuda.stream(compute):   # before the first chunk, on the compute stream
                self.state.view(H, D, D).copy_(state_in)
        loaded = [torch.cuda.Event() for _ in range(2)]     # chunk's inputs are in buffer b
        consumed = [torch.cuda.Event() for _ in range(2)]   # the prefill has read buffer b / written out b
        drained = [torch.cuda.Event() for _ in range(2)]    # out buffer b is back in host memory
        chunks = (T + n - 1) // n
        for i in range(chunks):
            b, t0 = i % 2, i * n
            t1 = min(T, t0 + n)
            m = t1 - t0
            with torch.cuda.stream(self.h2d):
                if i >= 2:
                    self.h2d.wait_event(consumed[b])
                self.q[b][:m].copy_(q[t0:t1], non_blocking=True)
                self.k[b][:m].copy_(k[t0:t1], non_blocking=True)
                self.v[b][:m].copy_(v[t0:t1], non_blocking=True)
                if gated:
                    self.g[b][:m].copy_(g[t0:t1], non_blocking=True)
                loaded[b].record(self.h2d)
            compute.wait_event(loaded[b])
            if i >= 2:
                compute.wait_event(drained[b])
            la.lightning_attn_prefill(self.q[b][:m][None], self.k[b][:m][None], self.v[b][:m][None],
                                      self.g[b][:m][None] if gated else None, self.out[b][:m][None],
                                      self.state if (i > 0 or have_state) else None, self.state,
                                      block_size=self.block_size, phi=self.phi, mode=self.mode, eps=self.eps,
                                      norm_weight=self.norm_weight, workspace=self.ws, stream=compute)
            consumed[b].record(compute)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(consumed[b])
                out[t0:t1].copy_(self.out[b][:m], non_blocking=True)
                drained[b].record(self.d2h)
        compute.wait_stream(self.d2h)
        compute.wait_stream(self.h2d)
        if state_out is not None:
            with torch.cuda.stream(compute):
                if T == 0 and not have_state:
                    state_out.zero_()
                else:   # T == 0 with a state: the copy of state_in made above
                    state_out.copy_(self.state.view(H, D, D))

    def check(self):
        """Synchronise the last call's stream and raise on a device-side error it recorded."""
        la.lightning_attn_check(self.ws, stream=self.last)
