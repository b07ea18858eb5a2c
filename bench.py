#!/usr/bin/env python
"""Benchmark of the Lightning Attention forward on B200 (one JSON line on rank 0).

Default workload: prefill of one 131072-token sequence, 64 heads of 128, bf16, block 256,
RMSNorm over the head concatenation times sigmoid(gate), final fp32 state returned.
A step is one lightning_attn_prefill call over that batch (the whole hot path: SiLU,
intra- and inter-block products, the fp32 state carry, the norm and the gate).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

* value: tokens/s of the whole job (N ranks, each an independent replica of the workload:
  the sequences/heads of the path are independent, so there is no data-path collective),
  timed with CUDA events on the launching stream, inputs resident in HBM, max over ranks.
  Inputs are larger than L2 (10.7 GB per step at 128K), so no L2 flush is needed.
* roofline: the prefill kernel is bound by HBM; achieved = algorithmic bytes per launch
  (q, k, v, g read + out written, bf16: 5 * H * D * 2 bytes per token, plus the state)
  / mean launch duration from events around each call in the timed region.
* e2e: the same metric through the C ABI with pinned host buffers; every step copies
  q, k, v, g host->device and reads out (and the state) back.
* cpu_baseline: the fp64 oracle timed on this host's cores on a bounded sample.
* --impl reference: the oracle timed as the reference arm (rank 0 only).
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "lightning-attn prefill tokens/s @128K,H64,d128; % tensor/HBM roofline"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------------------------
_CLK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={_CLK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.text = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.text, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.text, _ = self.proc.communicate()
        return False

    def summary(self):
        rows = [r for r in csv.reader(io.StringIO(self.text)) if len(r) >= 10]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(x):
            try:
                return float(x.strip())
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows]
        util = [num(r[4]) for r in rows]
        loaded = [s for s, u in zip(sm, util) if s is not None and (u or 0) >= 50] or [s for s in sm if s]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[6 + j].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": num(rows[0][2]),
                "reasons": reasons, "samples": len(rows), "power_w_max": max((num(r[3]) or 0) for r in rows)}


# ----------------------------------------------------------------------------------------------
# Workloads
# ----------------------------------------------------------------------------------------------
def _bytes_per_token(H, D):
    return 5 * H * D * 2  # q, k, v, g read + out written, bf16


def _flops_per_token(H, D, C):
    """(algorithmic, issued) FLOPs per token over all heads.

    algorithmic: 2 d (C + 1) for the masked intra block (averaged over a block) plus 4 d^2
    for the inter read phi(q)^T S and the state carry phi(k) v^T.
    issued by the tensor-core kernel: 128-row tiles; a query tile multiplies by the key
    tiles of its block up to the diagonal (the zero quarter of a 256-block is skipped);
    each CTA computes a head's full width, so every score is computed once.  The chunk-state
    pass that lets a long sequence run as parallel chunks is not counted.
    """
    algo = H * (2 * D * (C + 1) + 4 * D * D)
    tiles = C // 128
    keys = 128 * (tiles + 1) / 2          # mean keys per query row multiplied
    issued = H * (2 * keys * D            # P = phi(Q) phi(K)^T
                  + 2 * keys * D          # O += P V
                  + 2 * D * D             # O += phi(Q) S
                  + 2 * D * D)            # S += phi(K)^T V
    return algo, issued


class PrefillCase:
    def __init__(self, name, w, device, rank):
        import torch
        from long_context_attn_b200 import lightning_attn as la
        self.la, self.w = la, w
        self.T, self.H, self.D, self.C = w.T, w.H, w.D, w.block_size
        assert w.dtype == "bf16"
        t0 = time.time()
        q, k, v, g = synth.prefill_inputs(w.seed + 1000 * rank, w.T, w.H, w.D, "bf16", w.qkv_scale, True)
        self.gen_s = time.time() - t0

        def pin(a):
            t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
            return t.pin_memory()

        self.h_q, self.h_k, self.h_v, self.h_g = (pin(a) for a in (q, k, v, g))
        del q, k, v, g
        T, H, D = w.T, w.H, w.D
        self.q = self.h_q.to(device).view(1, T, H, D)
        self.k = self.h_k.to(device).view(1, T, H, D)
        self.v = self.h_v.to(device).view(1, T, H, D)
        self.g = self.h_g.to(device).view(1, T, H * D)
        self.out = torch.empty((1, T, H * D), dtype=torch.bfloat16, device=device)
        self.state = torch.empty((1, H, D, D), dtype=torch.float32, device=device)
        self.h_out = torch.empty((1, T, H * D), dtype=torch.bfloat16).pin_memory()
        self.h_state = torch.empty((1, H, D, D), dtype=torch.float32).pin_memory()
        nbytes = la.lightning_attn_workspace_size(la.LA_OP_PREFILL, 1, T, 0, H, D, self.C, la.LA_BF16,
                                                  la.LA_OUT_RMSNORM_GATE)
        self.ws = la.new_workspace(nbytes, device)
        self.tokens = T
        self.alg_bytes = T * _bytes_per_token(H, D) + H * D * D * 4
        self.alg_flops, self.issued_flops = (x * T for x in _flops_per_token(H, D, self.C))
        self.h2d = sum(t.numel() * t.element_size() for t in (self.h_q, self.h_k, self.h_v, self.h_g))
        self.d2h = self.h_out.numel() * 2 + self.h_state.numel() * 4

    def step(self):
        self.la.lightning_attn_prefill(self.q, self.k, self.v, self.g, self.out, None, self.state,
                                       block_size=self.C, workspace=self.ws)

    @property
    def launches_per_step(self):
        # a sequence run as parallel chunks: chunk bounds, chunk states, their split sum, the
        # prefix of initial states and the prefill kernel; else the prefill kernel alone
        return 5 if self.la.lightning_attn_last_path().endswith("+chunks") else 1

    def enable_host_pipeline(self, chunk_tokens):
        """e2e through HostPrefill: the copies in and out overlapped over chunks of the sequence."""
        from long_context_attn_b200.host_stream import HostPrefill
        self.host = HostPrefill(self.H, self.D, chunk_tokens=chunk_tokens, block_size=self.C,
                                device=self.q.device)
        self.host_chunk = chunk_tokens

    def e2e_step(self):
        host = getattr(self, "host", None)
        if host is not None:
            T, H, D = self.T, self.H, self.D
            host(self.h_q.view(T, H, D), self.h_k.view(T, H, D), self.h_v.view(T, H, D), self.h_g.view(T, H * D),
                 self.h_out.view(T, H * D), state_out=self.state.view(H, D, D))
            self.h_state.copy_(self.state, non_blocking=True)
            return
        self.q.view(-1).copy_(self.h_q.view(-1), non_blocking=True)
        self.k.view(-1).copy_(self.h_k.view(-1), non_blocking=True)
        self.v.view(-1).copy_(self.h_v.view(-1), non_blocking=True)
        self.g.view(-1).copy_(self.h_g.view(-1), non_blocking=True)
        self.step()
        self.h_out.copy_(self.out, non_blocking=True)
        self.h_state.copy_(self.state, non_blocking=True)

    def check(self):
        self.la.lightning_attn_check(self.ws)
        if getattr(self, "host", None) is not None:
            self.host.check()

    def oracle_sample(self, tokens):
        """fp64 oracle on the first `tokens` rows of the same workload (all heads)."""
        import oracle
        w = self.w
        q, k, v, g = synth.prefill_inputs(w.seed, tokens, w.H, w.D, "bf16", w.qkv_scale, True)
        t0 = time.perf_counter()
        oracle.prefill(q[None], k[None], v[None], g[None], store=False)
        return time.perf_counter() - t0

    def describe(self):
        return {"workload": self.w.name, "B": 1, "T": self.T, "H": self.H, "D": self.D, "block_size": self.C,
                "mode": "rmsnorm_gate", "state_out": True,
                "l2": "inputs larger than L2 (%.1f GB per step), no flush" % (self.alg_bytes / 1e9)}


class DecodeCase:
    """256 sequences x 64 heads, one token each; S (1 GiB fp32) updated in place."""

    def __init__(self, name, w, device, rank):
        import torch
        from long_context_attn_b200 import lightning_attn as la
        self.la, self.w = la, w
        B, H, D = w.B, w.H, w.D
        t0 = time.time()
        S = synth.decode_state(w.seed + 1000 * rank, B, H, D)
        ring = [synth.decode_tokens(w.seed, s, B, H, D, "bf16", w.qkv_scale) for s in range(16)]
        self.gen_s = time.time() - t0
        self.S = torch.from_numpy(S).to(device)

        def dev(a):
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)

        self.ring = [tuple(dev(a) for a in r) for r in ring]
        self.h_ring = [tuple(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in r)
                       for r in ring]
        self.out = torch.empty((B, H * D), dtype=torch.bfloat16, device=device)
        self.h_out = torch.empty((B, H * D), dtype=torch.bfloat16).pin_memory()
        self.ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_DECODE, B, 0, 0, H, D, 0, la.LA_BF16,
                                                                    la.LA_OUT_RMSNORM_GATE), device)
        self.i = 0
        self.tokens = B
        self.alg_bytes = B * H * (2 * D * D * 4 + 5 * D * 2)
        self.alg_flops = B * H * 4 * D * D
        self.issued_flops = self.alg_flops
        self.h2d = sum(a.numel() * 2 for a in self.h_ring[0])
        self.d2h = self.h_out.numel() * 2

    def step(self):
        q, k, v, g = self.ring[self.i % 16]
        self.i += 1
        self.la.lightning_attn_decode_step(q, k, v, g, self.out, self.S, workspace=self.ws)

    def e2e_step(self):
        q, k, v, g = self.ring[self.i % 16]
        hq, hk, hv, hg = self.h_ring[self.i % 16]
        for d, h in ((q, hq), (k, hk), (v, hv), (g, hg)):
            d.copy_(h, non_blocking=True)
        self.step()
        self.h_out.copy_(self.out, non_blocking=True)

    def check(self):
        self.la.lightning_attn_check(self.ws)

    def oracle_sample(self, seqs):
        import oracle
        w = self.w
        q, k, v, g = synth.decode_tokens(w.seed, 0, w.B, w.H, w.D, "bf16", w.qkv_scale)
        S = synth.decode_state(w.seed, w.B, w.H, w.D)
        t0 = time.perf_counter()
        oracle.decode(q[:seqs], k[:seqs], v[:seqs], g[:seqs], S[:seqs])
        return time.perf_counter() - t0

    def describe(self):
        return {"workload": self.w.name, "B": self.w.B, "H": self.w.H, "D": self.w.D, "mode": "rmsnorm_gate",
                "state": "fp32 [256,64,128,128] in place (1 GiB)",
                "l2": "state larger than L2 (1 GiB read + written per step), no flush"}


class VarlenCase:
    """16 packed sequences (lengths ~ U{1000..32768}), cu_seqlens on the device, block 256
    with 32/64/128 tail pads, gated concat RMSNorm, per-sequence final states."""

    launches_per_step = 2   # the longest-first work plan and the prefill kernel

    def __init__(self, name, w, device, rank):
        import torch
        from long_context_attn_b200 import lightning_attn as la
        self.la, self.w = la, w
        H, D = w.H, w.D
        self.lens = synth.varlen_lengths(w)
        self.n = len(self.lens)
        self.total = int(self.lens.sum())
        self.max_len = int(self.lens.max())
        t0 = time.time()
        q, k, v, g = synth.prefill_inputs(w.seed + 1000 * rank, self.total, H, D, "bf16", w.qkv_scale, True)
        self.gen_s = time.time() - t0

        def pin(a):
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()

        self.h_q, self.h_k, self.h_v, self.h_g = (pin(a) for a in (q, k, v, g))
        del q, k, v, g
        self.q = self.h_q.to(device).view(self.total, H, D)
        self.k = self.h_k.to(device).view(self.total, H, D)
        self.v = self.h_v.to(device).view(self.total, H, D)
        self.g = self.h_g.to(device).view(self.total, H * D)
        self.cu = torch.from_numpy(synth.cu_seqlens_of(self.lens)).to(device)
        self.out = torch.empty((self.total, H * D), dtype=torch.bfloat16, device=device)
        self.state = torch.empty((self.n, H, D, D), dtype=torch.float32, device=device)
        self.h_out = torch.empty((self.total, H * D), dtype=torch.bfloat16).pin_memory()
        self.h_state = torch.empty((self.n, H, D, D), dtype=torch.float32).pin_memory()
        self.ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_VARLEN, self.n, self.max_len,
                                                                    self.total, H, D, w.block_size, la.LA_BF16,
                                                                    la.LA_OUT_RMSNORM_GATE), device)
        self.tokens = self.total
        self.alg_bytes = self.total * _bytes_per_token(H, D) + self.n * H * D * D * 4
        self.alg_flops, self.issued_flops = (x * self.total for x in _flops_per_token(H, D, w.block_size))
        self.h2d = sum(t.numel() * t.element_size() for t in (self.h_q, self.h_k, self.h_v, self.h_g))
        self.d2h = self.h_out.numel() * 2 + self.h_state.numel() * 4
        # Rows the tail pads add (per sequence: the last block's r = L mod C rows run at the
        # smallest of 32/64/128 that holds them, else at C).
        C = w.block_size
        pad = 0
        for L in self.lens.tolist():
            r = L % C
            if r:
                p = next((x for x in (32, 64, 128) if x >= r and x < C), C)
                pad += p - r
        self.padded_rows = pad

    def step(self):
        self.la.lightning_attn_prefill_varlen(self.q, self.k, self.v, self.g, self.out, self.cu, self.max_len,
                                              None, self.state, block_size=self.w.block_size, workspace=self.ws)

    def e2e_step(self):
        self.q.view(-1).copy_(self.h_q.view(-1), non_blocking=True)
        self.k.view(-1).copy_(self.h_k.view(-1), non_blocking=True)
        self.v.view(-1).copy_(self.h_v.view(-1), non_blocking=True)
        self.g.view(-1).copy_(self.h_g.view(-1), non_blocking=True)
        self.step()
        self.h_out.copy_(self.out, non_blocking=True)
        self.h_state.copy_(self.state, non_blocking=True)

    def check(self):
        self.la.lightning_attn_check(self.ws)

    def oracle_sample(self, tokens):
        """fp64 oracle on the first `tokens` rows of the first sequence (all heads)."""
        import oracle
        w = self.w
        n = min(tokens, int(self.lens[0]))
        q, k, v, g = synth.prefill_inputs(w.seed, n, w.H, w.D, "bf16", w.qkv_scale, True)
        t0 = time.perf_counter()
        oracle.prefill(q[None], k[None], v[None], g[None], store=False)
        return time.perf_counter() - t0, n

    def describe(self):
        return {"workload": self.w.name, "N": self.n, "total_tokens": self.total, "max_len": self.max_len,
                "H": self.w.H, "D": self.w.D, "block_size": self.w.block_size, "mode": "rmsnorm_gate",
                "state_out": True, "padded_rows": self.padded_rows,
                "l2": "inputs larger than L2 (%.1f GB per step), no flush" % (self.alg_bytes / 1e9)}


class ZnormCase(PrefillCase):
    """The normalised variant over the 128K prefill's shapes (q, k shifted so phi(q) . z > 0)."""

    launches_per_step = 5   # raw prefill, phi(k) chunk sums, their prefix, denominators, transform

    def __init__(self, name, w, device, rank):
        super().__init__(name, w, device, rank)
        import torch
        T, H, D = self.T, self.H, self.D
        for host, dev in ((self.h_q, self.q), (self.h_k, self.k)):
            a = synth.shifted(host.view(torch.int16).numpy().view(np.uint16), w.qk_shift)
            host.copy_(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16))
            dev.view(-1).copy_(host.view(-1))
        self.z = torch.empty((1, H, D), dtype=torch.float32, device=device)
        self.h_z = torch.empty((1, H, D), dtype=torch.float32).pin_memory()
        nbytes = self.la.lightning_attn_workspace_size(self.la.LA_OP_PREFILL_ZNORM, 1, T, 0, H, D, self.C,
                                                       self.la.LA_BF16, self.la.LA_OUT_RMSNORM_GATE)
        self.ws = self.la.new_workspace(nbytes, device)
        self.alg_bytes += H * D * 4
        self.d2h += H * D * 4

    def step(self):
        self.la.lightning_attn_prefill_znorm(self.q, self.k, self.v, self.g, self.out, None, None, self.state, self.z,
                                             block_size=self.C, workspace=self.ws)

    def e2e_step(self):
        super().e2e_step()
        self.h_z.copy_(self.z, non_blocking=True)

    def oracle_sample(self, tokens):
        import oracle
        w = self.w
        q, k, v, g = synth.prefill_inputs(w.seed, tokens, w.H, w.D, "bf16", w.qkv_scale, True)
        q, k = synth.shifted(q, w.qk_shift), synth.shifted(k, w.qk_shift)
        t0 = time.perf_counter()
        oracle.prefill_znorm(q[None], k[None], v[None], g[None])
        return time.perf_counter() - t0

    def describe(self):
        return dict(super().describe(), variant="normalised (z-denominator)", qk_shift=self.w.qk_shift)


class TinyCase:
    """The small fp32 check: 1 x 512 tokens x 2 heads x d 64, block 64, raw output.  Its
    inputs fit in L2, so each timed step follows a write of a buffer larger than L2 and is
    timed alone."""

    def __init__(self, name, w, device, rank):
        import torch
        from long_context_attn_b200 import lightning_attn as la
        self.la, self.w = la, w
        T, H, D = w.T, w.H, w.D
        q, k, v, _ = synth.prefill_inputs(w.seed + 1000 * rank, T, H, D, "f32", w.qkv_scale, False)
        self.q, self.k, self.v = (torch.from_numpy(a).to(device).view(1, T, H, D) for a in (q, k, v))
        self.out = torch.empty((1, T, H * D), dtype=torch.float32, device=device)
        self.state = torch.empty((1, H, D, D), dtype=torch.float32, device=device)
        self.ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, 1, T, 0, H, D, w.block_size,
                                                                    la.LA_F32, la.LA_OUT_RAW), device)
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.tokens = T
        self.alg_bytes = T * 4 * H * D * 4 + H * D * D * 4   # q, k, v read + out written, fp32; the state
        self.alg_flops, self.issued_flops = (x * T for x in _flops_per_token(H, D, w.block_size))
        self.launches_per_step = 1

    def step(self):
        self.la.lightning_attn_prefill(self.q, self.k, self.v, None, self.out, None, self.state,
                                       block_size=self.w.block_size, mode=self.la.LA_OUT_RAW, workspace=self.ws)

    def check(self):
        self.la.lightning_attn_check(self.ws)

    def oracle_sample(self):
        import oracle
        w = self.w
        q, k, v, _ = synth.prefill_inputs(w.seed, w.T, w.H, w.D, "f32", w.qkv_scale, False)
        t0 = time.perf_counter()
        oracle.prefill(q[None], k[None], v[None], None, mode=oracle.MODE_RAW, store=False)
        return time.perf_counter() - t0

    def describe(self):
        w = self.w
        return {"workload": w.name, "B": 1, "T": w.T, "H": w.H, "D": w.D, "block_size": w.block_size,
                "dtype": "f32", "mode": "raw", "l2": "inputs fit in L2: a 256 MiB write before each timed step"}


class ChunkStateCase:
    """Step 1 of the sequence-parallel prefill: the state of one 128K sequence from k and v."""

    def __init__(self, name, w, device, rank):
        import torch
        from long_context_attn_b200 import lightning_attn as la
        self.la, self.w = la, w
        T, H, D = w.T, w.H, w.D
        self.T, self.H, self.D = T, H, D
        t0 = time.time()
        _, k, v, _ = synth.prefill_inputs(w.seed + 1000 * rank, T, H, D, "bf16", w.qkv_scale, False)
        self.gen_s = time.time() - t0
        self.h_k, self.h_v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in (k, v))
        del k, v
        self.k = self.h_k.to(device).view(1, T, H, D)
        self.v = self.h_v.to(device).view(1, T, H, D)
        self.state = torch.empty((1, H, D, D), dtype=torch.float32, device=device)
        self.h_state = torch.empty((1, H, D, D), dtype=torch.float32).pin_memory()
        self.ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_CHUNK_STATE, 1, T, 0, H, D, 0,
                                                                    la.LA_BF16, 0), device)
        self.tokens = T
        self.alg_bytes = T * 2 * H * D * 2 + H * D * D * 4     # k, v read once; the state written
        self.alg_flops = self.issued_flops = T * H * 2 * D * D
        self.launches_per_step = 2                             # the state kernel and the split sum
        self.h2d = 2 * T * H * D * 2
        self.d2h = H * D * D * 4

    def step(self):
        self.la.lightning_attn_chunk_state(self.k, self.v, self.state, workspace=self.ws)

    def e2e_step(self):
        self.k.view(-1).copy_(self.h_k.view(-1), non_blocking=True)
        self.v.view(-1).copy_(self.h_v.view(-1), non_blocking=True)
        self.step()
        self.h_state.copy_(self.state, non_blocking=True)

    def check(self):
        self.la.lightning_attn_check(self.ws)

    def oracle_sample(self, tokens):
        import oracle
        w = self.w
        q, k, v, _ = synth.prefill_inputs(w.seed, tokens, w.H, w.D, "bf16", w.qkv_scale, False)
        t0 = time.perf_counter()
        oracle.prefill(k[None], k[None], v[None], None, mode=oracle.MODE_RAW, store=False)
        return time.perf_counter() - t0

    def describe(self):
        return {"workload": self.w.name, "B": 1, "T": self.T, "H": self.H, "D": self.D, "output": "final state only",
                "l2": "inputs larger than L2 (%.1f GB per step), no flush" % (self.alg_bytes / 1e9)}


class BackwardCase:
    """The backward of one long prefill: gradients of q, k, v and the gate from dout."""

    def __init__(self, name, w, device, rank):
        import torch
        from long_context_attn_b200 import lightning_attn as la
        self.la, self.w = la, w
        T, H, D, self.C = w.T, w.H, w.D, w.block_size
        self.T, self.H, self.D = T, H, D
        t0 = time.time()
        q, k, v, g = synth.prefill_inputs(w.seed + 1000 * rank, T, H, D, "bf16", w.qkv_scale, True)
        dout = synth.normal(w.seed + 1000 * rank, synth.STREAM_DOUT, (T, H * D), 1.0, "bf16")
        self.gen_s = time.time() - t0

        def pin(a):
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()

        self.h_in = [pin(a) for a in (q, k, v, g, dout)]
        del q, k, v, g, dout
        shapes = [(1, T, H, D)] * 3 + [(1, T, H * D)] * 2
        self.d_in = [h.to(device).view(s) for h, s in zip(self.h_in, shapes)]
        self.d_out = [torch.empty(s, dtype=torch.bfloat16, device=device) for s in shapes[:4]]
        self.h_out = [torch.empty(s, dtype=torch.bfloat16).pin_memory() for s in shapes[:4]]
        nbytes = la.lightning_attn_workspace_size(la.LA_OP_BACKWARD, 1, T, 0, H, D, self.C, la.LA_BF16,
                                                  la.LA_OUT_RMSNORM_GATE)
        self.ws = la.new_workspace(nbytes, device)
        self.tokens = T
        # inputs q, k, v, g, dout read and dq, dk, dv, dg written once: the bytes any backward moves
        self.alg_bytes = T * 9 * H * D * 2
        # the forward recompute plus three passes of the same linear attention
        self.alg_flops, self.issued_flops = (4 * x * T for x in _flops_per_token(H, D, self.C))
        self.launches_per_step = 7      # recompute, norm/gate backward, prep, three passes, post
        self.h2d = sum(t.numel() * 2 for t in self.h_in)
        self.d2h = sum(t.numel() * 2 for t in self.h_out)

    def step(self):
        q, k, v, g, dout = self.d_in
        dq, dk, dv, dg = self.d_out
        self.la.lightning_attn_backward(q, k, v, g, dout, dq, dk, dv, dg=dg, block_size=self.C, workspace=self.ws)

    def e2e_step(self):
        for d, h in zip(self.d_in, self.h_in):
            d.view(-1).copy_(h.view(-1), non_blocking=True)
        self.step()
        for h, d in zip(self.h_out, self.d_out):
            h.copy_(d, non_blocking=True)

    def check(self):
        self.la.lightning_attn_check(self.ws)

    def oracle_sample(self, tokens):
        """fp64 oracle backward on the first `tokens` rows of the same workload (all heads)."""
        import oracle
        w = self.w
        q, k, v, g = synth.prefill_inputs(w.seed, tokens, w.H, w.D, "bf16", w.qkv_scale, True)
        dout = synth.normal(w.seed, synth.STREAM_DOUT, (tokens, w.H * w.D), 1.0, "bf16")
        t0 = time.perf_counter()
        oracle.backward(q[None], k[None], v[None], g[None], dout[None])
        return time.perf_counter() - t0

    def describe(self):
        return {"workload": self.w.name, "B": 1, "T": self.T, "H": self.H, "D": self.D, "block_size": self.C,
                "mode": "rmsnorm_gate", "grads": "dq, dk, dv, dg",
                "l2": "inputs larger than L2 (%.1f GB per step), no flush" % (self.alg_bytes / 1e9)}


class TrainCase(BackwardCase):
    """A training step on one long sequence: the forward keeping its raw output y (prefill in
    raw mode, then the norm and gate), and the backward from dout using that y, with the
    norm weight's gradient as well (the norm weight is a trained parameter)."""

    def __init__(self, name, w, device, rank):
        super().__init__(name, w, device, rank)
        import torch
        T, H, D = self.T, self.H, self.D
        self.y = torch.empty((1, T, H * D), dtype=torch.bfloat16, device=device)
        self.out = torch.empty((1, T, H * D), dtype=torch.bfloat16, device=device)
        self.h_out_fwd = torch.empty((1, T, H * D), dtype=torch.bfloat16).pin_memory()
        self.nw = torch.ones((H * D,), dtype=torch.float32, device=device)
        self.dw = torch.empty((H * D,), dtype=torch.float32, device=device)
        self.h_dw = torch.empty((H * D,), dtype=torch.float32).pin_memory()
        # forward: q, k, v, g read + out written; backward: q, k, v, g, dout read + 4 gradients written
        self.alg_bytes = T * 14 * H * D * 2
        # the forward prefill plus the backward's three passes (the recompute is skipped)
        self.alg_flops, self.issued_flops = (4 * x * T for x in _flops_per_token(H, D, self.C))
        # prefill, transform; backward: dw (two stages), norm/gate, features, three passes, scale
        self.launches_per_step = 10
        self.d2h += self.h_out_fwd.numel() * 2 + self.h_dw.numel() * 4

    def step(self):
        la = self.la
        q, k, v, g, dout = self.d_in
        dq, dk, dv, dg = self.d_out
        B, T, H, D = q.shape
        la.lightning_attn_prefill(q, k, v, None, self.y, None, None, block_size=self.C, mode=la.LA_OUT_RAW,
                                  workspace=self.ws)
        la.lightning_attn_output_transform(self.y.view(B, T, H, D), g, self.out, norm_weight=self.nw)
        la.lightning_attn_backward(q, k, v, g, dout, dq, dk, dv, dg=dg, block_size=self.C, norm_weight=self.nw,
                                   workspace=self.ws, y=self.y, dnorm_weight=self.dw)

    def e2e_step(self):
        super().e2e_step()
        self.h_out_fwd.copy_(self.out, non_blocking=True)
        self.h_dw.copy_(self.dw, non_blocking=True)

    def oracle_sample(self, tokens):
        import oracle
        w = self.w
        q, k, v, g = synth.prefill_inputs(w.seed, tokens, w.H, w.D, "bf16", w.qkv_scale, True)
        dout = synth.normal(w.seed, synth.STREAM_DOUT, (tokens, w.H * w.D), 1.0, "bf16")
        t0 = time.perf_counter()
        oracle.prefill(q[None], k[None], v[None], g[None], store=False)
        oracle.backward(q[None], k[None], v[None], g[None], dout[None])
        return time.perf_counter() - t0

    def describe(self):
        return dict(super().describe(), grads="dq, dk, dv, dg, dw",
                    step="forward (raw prefill + norm/gate, y kept) + backward with y")


class MixedCase:
    """One serving step: 256 sequences decode a token each while 2 others prefill a 4096-token
    chunk from their state; prefill and decode on two streams, states in a pool (slots in a
    seeded shuffled order), updated in place step after step."""

    def __init__(self, name, w, device, rank):
        import torch
        from long_context_attn_b200 import lightning_attn as la
        self.la, self.w = la, w
        H, D = w.H, w.D
        self.lens = synth.mixed_lengths(w)
        self.n = len(self.lens)
        self.total = int(self.lens.sum())
        t0 = time.time()
        q, k, v, g = synth.prefill_inputs(w.seed + 1000 * rank, self.total, H, D, "bf16", w.qkv_scale, True)
        pool = synth.decode_state(w.seed + 1000 * rank, self.n, H, D)
        self.gen_s = time.time() - t0
        perm = np.argsort(synth.uniform_int(w.seed, synth.STREAM_LEN, self.n, 0, 1 << 30), kind="stable")
        self.slots_host = perm.astype(np.int32)

        def pin(a):
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()

        self.h_q, self.h_k, self.h_v, self.h_g = (pin(a) for a in (q, k, v, g))
        del q, k, v, g
        self.q = self.h_q.to(device).view(self.total, H, D)
        self.k = self.h_k.to(device).view(self.total, H, D)
        self.v = self.h_v.to(device).view(self.total, H, D)
        self.g = self.h_g.to(device).view(self.total, H * D)
        self.pool = torch.from_numpy(pool).to(device)
        self.cu_host = synth.cu_seqlens_of(self.lens)
        self.cu = torch.from_numpy(self.cu_host).to(device)
        self.slots = torch.from_numpy(self.slots_host).to(device)
        self.out = torch.empty((self.total, H * D), dtype=torch.bfloat16, device=device)
        self.h_out = torch.empty((self.total, H * D), dtype=torch.bfloat16).pin_memory()
        max_pre = int(self.lens[self.lens > 1].max()) if (self.lens > 1).any() else 0
        self.ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_MIXED, self.n, max_pre, self.total, H, D,
                                                                    w.block_size, la.LA_BF16, la.LA_OUT_RMSNORM_GATE),
                                   device)
        self.ps, self.ds = torch.cuda.Stream(device), torch.cuda.Stream(device)
        self.tokens = self.total
        # this library's kernels per step: the prefill, the one-token gather and the decode
        self.launches_per_step = int((self.lens > 1).any()) + 2 * int((self.lens == 1).any())
        n_dec = int((self.lens == 1).sum())
        n_pre_tok = int(self.lens[self.lens > 1].sum())
        n_pre_seq = int((self.lens > 1).sum())
        self.alg_bytes = (n_dec * H * (2 * D * D * 4 + 5 * D * 2) + n_pre_tok * _bytes_per_token(H, D) +
                          n_pre_seq * H * D * D * 4 * 2)
        algo_pt, issued_pt = _flops_per_token(H, D, w.block_size)
        self.alg_flops = n_dec * H * 4 * D * D + n_pre_tok * algo_pt
        self.issued_flops = n_dec * H * 4 * D * D + n_pre_tok * issued_pt
        self.h2d = sum(t.numel() * t.element_size() for t in (self.h_q, self.h_k, self.h_v, self.h_g))
        self.d2h = self.h_out.numel() * 2

    def step(self):
        import torch
        cur = torch.cuda.current_stream()
        self.ps.wait_stream(cur)
        self.ds.wait_stream(cur)
        self.la.lightning_attn_mixed_step(self.q, self.k, self.v, self.g, self.out, self.cu, self.cu_host.tolist(),
                                          self.pool, self.slots, block_size=self.w.block_size, workspace=self.ws,
                                          prefill_stream=self.ps, decode_stream=self.ds)
        cur.wait_stream(self.ps)
        cur.wait_stream(self.ds)

    def e2e_step(self):
        self.q.view(-1).copy_(self.h_q.view(-1), non_blocking=True)
        self.k.view(-1).copy_(self.h_k.view(-1), non_blocking=True)
        self.v.view(-1).copy_(self.h_v.view(-1), non_blocking=True)
        self.g.view(-1).copy_(self.h_g.view(-1), non_blocking=True)
        self.step()
        self.h_out.copy_(self.out, non_blocking=True)

    def check(self):
        self.ps.synchronize()
        self.ds.synchronize()
        self.la.lightning_attn_check(self.ws)

    def oracle_sample(self):
        """fp64 oracle over the whole step (every sequence from its pooled state)."""
        import oracle
        w = self.w
        q, k, v, g = synth.prefill_inputs(w.seed, self.total, w.H, w.D, "bf16", w.qkv_scale, True)
        pool = synth.decode_state(w.seed, self.n, w.H, w.D)
        t0 = time.perf_counter()
        oracle.forward_packed(q, k, v, g, self.cu_host, w.H, w.D, state_in=pool[self.slots_host], store=False)
        return time.perf_counter() - t0

    def describe(self):
        return {"workload": self.w.name, "decode_seqs": int((self.lens == 1).sum()),
                "prefill_chunks": int((self.lens > 1).sum()), "chunk_tokens": self.w.T, "H": self.w.H,
                "D": self.w.D, "block_size": self.w.block_size, "mode": "rmsnorm_gate",
                "streams": "prefill and decode on two streams",
                "l2": "state pool larger than L2 (%.2f GB per step), no flush" % (self.alg_bytes / 1e9)}


def _make_case(name, device, rank):
    w = synth.WORKLOADS[name]
    if w.kind == "prefill" and w.dtype == "bf16":
        return PrefillCase(name, w, device, rank)
    if w.kind == "varlen":
        return VarlenCase(name, w, device, rank)
    if w.kind == "mixed":
        return MixedCase(name, w, device, rank)
    if w.kind == "decode":
        return DecodeCase(name, w, device, rank)
    if w.kind == "backward":
        return BackwardCase(name, w, device, rank)
    if w.kind == "train":
        return TrainCase(name, w, device, rank)
    if w.kind == "znorm":
        return ZnormCase(name, w, device, rank)
    if w.kind == "chunk_state":
        return ChunkStateCase(name, w, device, rank)
    if w.kind == "prefill" and w.dtype == "f32":
        return TinyCase(name, w, device, rank)
    raise SystemExit(f"workload {name} is not a bench workload")


# ----------------------------------------------------------------------------------------------
# Multi-rank helpers (one process per GPU; the job's time is its slowest rank's)
# ----------------------------------------------------------------------------------------------
def _max_over_ranks(vals, world, device=None):
    """Element-wise maximum of `vals` over all ranks of the default process group."""
    import torch
    t = torch.tensor([float(x) for x in vals], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def _job_value(units_per_rank_step, steps, world, elapsed_ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank_step * steps * world / (elapsed_ms / 1e3)


# ----------------------------------------------------------------------------------------------
# Arms
# ----------------------------------------------------------------------------------------------
def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    case = _make_case(args.workload, device, rank)
    if args.e2e_chunk:
        if not hasattr(case, "enable_host_pipeline"):
            raise SystemExit(f"--e2e-chunk applies to the single-sequence prefill workloads, not {args.workload}")
        case.enable_host_pipeline(args.e2e_chunk)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        case.step()
    case.check()
    torch.cuda.synchronize()

    # ---- device-resident timing ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        # A device-side spin ahead of the first event lets the host queue the first steps, so
        # the events see the GPU's time and not the first call's marshalling; a host that
        # cannot keep up in steady state still shows in the timing (and e2e has no hold).
        torch.cuda._sleep(HOLD_CYCLES)
        e0.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            case.step()
            ends[i].record(stream)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    case.check()
    elapsed_ms = e0.elapsed_time(e1)
    launch_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    elapsed_ms, launch_ms = _max_over_ranks([elapsed_ms, launch_ms], world, device)

    # ---- end-to-end through the C ABI with pinned host buffers ----
    for _ in range(min(2, args.warmup)):
        case.e2e_step()
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        case.e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    case.check()
    e2e_ms = _max_over_ranks([f0.elapsed_time(f1)], world, device)[0]

    if rank == 0:
        peaks = _peaks()
        value = _job_value(case.tokens, args.steps, world, elapsed_ms)
        achieved_gbs = case.alg_bytes / (launch_ms / 1e3) / 1e9
        line = {
            "metric": METRIC if args.workload == "prefill_128k" else f"lightning-attn {args.workload} tokens/s",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded SplitMix64/Box-Muller)",
            "config": dict(case.describe(), parallelism=f"replicas x{world} (independent sequences, no collective)"),
            "roofline": dict({"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": _traffic(args.workload),
                              "peak_source": peaks["source"], "launch_ms": launch_ms,
                              "algorithmic_bytes_per_launch": case.alg_bytes},
                             **({"scope": "one training step (forward + backward with dw, 10 kernels); algorithmic "
                                          "bytes = both calls' inputs read and outputs written once"}
                                if isinstance(case, TrainCase) else
                                {"scope": "one backward call (7 kernels); algorithmic bytes = its inputs "
                                          "read and gradients written once"}
                                if isinstance(case, BackwardCase) else
                                {"scope": "one normalised-variant call (5 kernels); algorithmic bytes as the "
                                          "prefill's plus z"}
                                if isinstance(case, ZnormCase) else
                                {"scope": "one chunk-state call (state kernel + split sum); algorithmic bytes = k, "
                                          "v read once + the state"}
                                if isinstance(case, ChunkStateCase) else {})),
            "tensor": {"algorithmic_tflops": case.alg_flops / (launch_ms / 1e3) / 1e12,
                       "issued_tflops": case.issued_flops / (launch_ms / 1e3) / 1e12,
                       "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                       "frac_algorithmic": case.alg_flops / (launch_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                       "frac_issued": case.issued_flops / (launch_ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
            "e2e": dict({"value": _job_value(case.tokens, args.steps, world, e2e_ms), "unit": "tokens/s",
                         "h2d_bytes_per_step": case.h2d, "d2h_bytes_per_step": case.d2h},
                        **({"pipeline": f"HostPrefill, chunks of {args.e2e_chunk} tokens"} if args.e2e_chunk else {})),
            "gpu_launches": args.steps * getattr(case, "launches_per_step", 1),
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = _cpu_baseline(case)
        if world == 1 and args.workload == "prefill_128k" and not args.no_secondary:
            del case
            torch.cuda.empty_cache()
            for name in SECONDARY_STEPS:
                line[name] = _measure_secondary(name, device, peaks)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


HOLD_CYCLES = 4_000_000   # about 2 ms at the B200's 1965 MHz SM clock

# The other configurations, measured in the same process after the headline (one GPU) and
# reported as keys of the same line: steps timed per configuration.
SECONDARY_STEPS = {"decode_256": 1000, "varlen_16": 10, "prefill_8k": 50, "tiny_f32": 200}


def _measure_secondary(name, device, peaks):
    """ms per step, tokens/s, the HBM roofline fraction and the clocks of one configuration."""
    import torch
    case = _make_case(name, device, 0)
    steps = SECONDARY_STEPS[name]
    for _ in range(3):
        case.step()
    case.check()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    per_step = isinstance(case, TinyCase)   # inputs inside L2: flush, then time each step alone
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        if per_step:
            total = 0.0
            for _ in range(steps):
                case.flush.fill_(1)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                case.step()
                b.record(stream)
                torch.cuda.synchronize()
                total += a.elapsed_time(b)
            ms = total / steps
        else:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(HOLD_CYCLES)
            a.record(stream)
            for _ in range(steps):
                case.step()
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / steps
    case.check()
    gbs = case.alg_bytes / (ms / 1e3) / 1e9
    out = {"ms_per_step": ms, "tokens_per_s": case.tokens / (ms / 1e3), "steps": steps,
           "config": case.describe(),
           "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_step": case.alg_bytes},
           "tensor": {"algorithmic_tflops": case.alg_flops / (ms / 1e3) / 1e12,
                      "frac_algorithmic": case.alg_flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
           "gpu_launches": steps * case.launches_per_step if hasattr(case, "launches_per_step") else steps,
           "clocks": clk.summary()}
    if hasattr(case, "lens"):
        out["path"] = case.la.lightning_attn_last_path()
    del case
    torch.cuda.empty_cache()
    return out

# Source files each measured kernel is built from (a traffic figure is tied to their hash).
KERNEL_SOURCES = {
    "prefill": ("la_prefill_pair.cu", "la_state_tc.cu", "la_tc_util.cuh", "la_sm100.cuh", "la_common.cuh"),
    "decode": ("la_decode.cu", "la_common.cuh"),
    "backward": ("la_backward.cu", "la_api.cu", "la_prefill_pair.cu", "la_state_tc.cu", "la_tc_util.cuh",
                 "la_sm100.cuh", "la_common.cuh"),
}


def kernel_source_hash(kind):
    """Hash of the CUDA sources of one kernel; committed DRAM traffic is used only while it matches."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_attn_b200", "csrc")
    for fn in KERNEL_SOURCES[kind]:
        h.update(fn.encode())
        h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def _traffic(workload):
    """DRAM bytes per launch of the dominant kernel (from ncu), or None once the kernel changed."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    entry = json.load(open(path)).get(workload)
    kind = next((k for k in ("decode", "backward") if workload.startswith(k)), "prefill")
    if not entry or entry.get("kernel_source_hash") != kernel_source_hash(kind):
        return None
    return entry["bytes_per_launch"]


def _cpu_baseline(case):
    import oracle
    if isinstance(case, ZnormCase):
        n = min(16384, case.T)
        dt = case.oracle_sample(n)
        return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"first {n} tokens of the {case.w.name} workload, all {case.H} heads, fp64 normalised "
                          f"recurrence + norm + gate ({dt:.1f} s)"}
    if isinstance(case, PrefillCase):
        n = min(131072, case.T)
        dt = case.oracle_sample(n)
        return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"first {n} tokens of the {case.w.name} workload, all {case.H} heads, fp64, "
                          f"recurrence + norm + gate ({dt:.1f} s)"}
    if isinstance(case, TinyCase):
        dt = case.oracle_sample()
        return {"value": case.tokens / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"the whole {case.w.name} workload ({case.tokens} tokens, {case.w.H} heads), fp64 raw "
                          f"recurrence ({dt:.2f} s)"}
    if isinstance(case, MixedCase):
        dt = case.oracle_sample()
        return {"value": case.total / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"the whole {case.w.name} step ({case.total} tokens, all {case.w.H} heads), fp64 "
                          f"({dt:.1f} s)"}
    if isinstance(case, ChunkStateCase):
        n = min(32768, case.T)
        dt = case.oracle_sample(n)
        return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"first {n} tokens of the {case.w.name} workload, all {case.H} heads, fp64 recurrence "
                          f"(final state) ({dt:.1f} s)"}
    if isinstance(case, BackwardCase):
        n = min(16384, case.T)
        dt = case.oracle_sample(n)
        what = "forward + backward" if isinstance(case, TrainCase) else \
            "backward (forward recompute, norm/gate backward, both scans)"
        return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"first {n} tokens of the {case.w.name} workload, all {case.H} heads, fp64 {what} "
                          f"({dt:.1f} s)"}
    if isinstance(case, VarlenCase):
        dt, n = case.oracle_sample(131072)
        return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                "sample": f"first {n} tokens of sequence 0 of the {case.w.name} workload, all {case.w.H} heads, "
                          f"fp64, recurrence + norm + gate ({dt:.1f} s)"}
    n = 64
    dt = case.oracle_sample(n)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {n} of {case.w.B} sequences of one decode step, all heads, fp64 ({dt:.1f} s)"}


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, on bounded samples of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = synth.WORKLOADS[args.workload]
    if w.kind == "train":
        n = 512
        q, k, v, g = synth.prefill_inputs(w.seed, n, w.H, w.D, w.dtype, w.qkv_scale, True)
        dout = synth.normal(w.seed, synth.STREAM_DOUT, (n, w.H * w.D), 1.0, w.dtype)

        def step():
            oracle.prefill(q[None], k[None], v[None], g[None], store=False)
            oracle.backward(q[None], k[None], v[None], g[None], dout[None])
        unit_per_step = n
        sample = f"first {n} tokens of {w.name} (all {w.H} heads) per step, fp64 forward + backward"
    elif w.kind == "chunk_state":
        n = 1024
        _, k, v, _ = synth.prefill_inputs(w.seed, n, w.H, w.D, w.dtype, w.qkv_scale, False)

        def step():
            oracle.prefill(k[None], k[None], v[None], None, mode=oracle.MODE_RAW, store=False)
        unit_per_step = n
        sample = f"first {n} tokens of {w.name} (all {w.H} heads) per step, fp64 recurrence (final state)"
    elif w.kind == "znorm":
        n = 1024
        q, k, v, g = synth.prefill_inputs(w.seed, n, w.H, w.D, w.dtype, w.qkv_scale, True)
        q, k = synth.shifted(q, w.qk_shift), synth.shifted(k, w.qk_shift)

        def step():
            oracle.prefill_znorm(q[None], k[None], v[None], g[None])
        unit_per_step = n
        sample = f"first {n} tokens of {w.name} (all {w.H} heads) per step, fp64 normalised recurrence + norm + gate"
    elif w.kind == "backward":
        n = 512
        q, k, v, g = synth.prefill_inputs(w.seed, n, w.H, w.D, w.dtype, w.qkv_scale, True)
        dout = synth.normal(w.seed, synth.STREAM_DOUT, (n, w.H * w.D), 1.0, w.dtype)

        def step():
            oracle.backward(q[None], k[None], v[None], g[None], dout[None])
        unit_per_step = n
        sample = f"first {n} tokens of {w.name} (all {w.H} heads) per step, fp64 backward"
    elif w.kind in ("prefill", "varlen", "mixed"):
        n = 1024
        q, k, v, g = synth.prefill_inputs(w.seed, n, w.H, w.D, w.dtype, w.qkv_scale, True)

        def step():
            oracle.prefill(q[None], k[None], v[None], g[None], store=False)
        unit_per_step = n
        sample = f"first {n} tokens of {w.name} (all {w.H} heads) per step, fp64 recurrence + norm + gate"
    else:
        n = 16
        q, k, v, g = synth.decode_tokens(w.seed, 0, w.B, w.H, w.D, "bf16", w.qkv_scale)
        S = synth.decode_state(w.seed, n, w.H, w.D)

        def step():
            oracle.decode(q[:n], k[:n], v[:n], g[:n], S)
        unit_per_step = n
        sample = f"{n} of {w.B} sequences of one decode step per step, fp64"
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = unit_per_step * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC if args.workload == "prefill_128k" else f"lightning-attn {args.workload} tokens/s",
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded SplitMix64/Box-Muller)",
        "config": {"workload": w.name, "T": w.T, "H": w.H, "D": w.D, "block_size": w.block_size},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_128k",
                    choices=["prefill_8k", "prefill_32k", "prefill_128k", "varlen_16", "decode_256", "mixed_256",
                             "backward_8k", "tiny_f32",
                             "backward_128k", "train_128k", "znorm_128k", "chunk_state_128k", "prefill_128k_h8"])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (profiling runs)")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other configurations after the headline (profiling runs)")
    ap.add_argument("--e2e-chunk", type=int, default=0,
                    help="e2e through HostPrefill with chunks of this many tokens (0: copy in, step, copy out)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        print("note: fewer than 3 warm-up steps; this run is not a valid bench line", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
