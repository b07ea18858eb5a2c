"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module draws numbers only; it holds none of the attention arithmetic.  The
generator itself is C (``synth.c``: SplitMix64 words + Box-Muller normals, a pure
function of (seed, stream, element index)); this file loads it with ctypes and
describes the bench and test workloads (shapes, value distributions, seeds).

Workload recipes (the Lightning Attention forward of MiniMax-01; the pages give
no data, so every input is synthetic):
  * q, k, v ~ scale * N(0, 1), g ~ N(0, 1), rounded to the tensor dtype;
  * prior decode state S ~ N(0, 1) / sqrt(head_dim), fp32;
  * varlen lengths ~ U{1000..32768};
  * the backward's output gradient dout ~ N(0, 1) (bf16);
  * config k uses seed 1000 + k; streams q=0, k=1, v=2, g=3, S=4, lengths=5, dout=6.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libla_synth.so")
_lib = None

STREAM_Q, STREAM_K, STREAM_V, STREAM_G, STREAM_S, STREAM_LEN, STREAM_DOUT = 0, 1, 2, 3, 4, 5, 6


def build(force: bool = False) -> str:
    """Compile synth.c into libla_synth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _get():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.synth_normal_f32.argtypes = [u64, u64, u64, i64, dbl, vp]
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, i64, dbl, vp]
        lib.synth_uniform_int.argtypes = [u64, u64, u64, i64, i64, i64, vp]
        lib.synth_ternary.argtypes = [u64, u64, u64, i64, dbl, vp, vp]
        lib.synth_bf16_to_f32.argtypes = [vp, i64, vp]
        for f in (lib.synth_normal_f32, lib.synth_normal_bf16, lib.synth_uniform_int,
                  lib.synth_ternary, lib.synth_bf16_to_f32):
            f.restype = None
        _lib = lib
    return _lib


def normal(seed: int, stream: int, shape, scale: float = 1.0, dtype: str = "bf16",
           offset: int = 0, out: np.ndarray | None = None) -> np.ndarray:
    """scale * N(0,1) elements [offset, offset + prod(shape)) of (seed, stream).

    dtype 'bf16' returns uint16 bit patterns; 'f32' returns float32.
    """
    n = int(np.prod(shape))
    if dtype == "bf16":
        a = out if out is not None else np.empty(shape, dtype=np.uint16)
        assert a.dtype == np.uint16 and a.flags.c_contiguous and a.size == n
        _get().synth_normal_bf16(seed, stream, offset, n, scale, a.ctypes.data)
    elif dtype == "f32":
        a = out if out is not None else np.empty(shape, dtype=np.float32)
        assert a.dtype == np.float32 and a.flags.c_contiguous and a.size == n
        _get().synth_normal_f32(seed, stream, offset, n, scale, a.ctypes.data)
    else:
        raise ValueError(dtype)
    return a


def uniform_int(seed: int, stream: int, n: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    a = np.empty(n, dtype=np.int64)
    _get().synth_uniform_int(seed, stream, offset, n, lo, hi, a.ctypes.data)
    return a


def ternary(seed: int, stream: int, shape, density: float, dtype: str = "bf16") -> np.ndarray:
    """Sparse values in {-1, 0, +1} (nonzero with probability `density`)."""
    n = int(np.prod(shape))
    if dtype == "bf16":
        a = np.empty(shape, dtype=np.uint16)
        _get().synth_ternary(seed, stream, 0, n, density, a.ctypes.data, None)
    else:
        a = np.empty(shape, dtype=np.float32)
        _get().synth_ternary(seed, stream, 0, n, density, None, a.ctypes.data)
    return a


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.uint16)
    out = np.empty(a.shape, dtype=np.float32)
    _get().synth_bf16_to_f32(a.ctypes.data, a.size, out.ctypes.data)
    return out


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 bit patterns (nearest even)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


# ----------------------------------------------------------------------------------------------
# Workloads
# ----------------------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str              # prefill varlen decode mixed backward train znorm chunk_state
    seed: int
    B: int                 # batch (prefill), number of sequences (varlen / decode)
    T: int                 # tokens per sequence (prefill); 0 otherwise
    H: int
    D: int
    block_size: int
    dtype: str             # 'f32' | 'bf16'
    mode: str              # 'raw' | 'rmsnorm_gate'
    qkv_scale: float
    len_lo: int = 0
    len_hi: int = 0
    eps: float = 1e-6
    n_prefill: int = 0     # mixed: number of prefill chunks (of T tokens) among B decode sequences
    qk_shift: float = 0.0  # added to q and k (before rounding) to keep phi(q) . z away from zero


# The workloads of the Lightning Attention forward and its backward (seed 1000 + k).
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", "prefill", 1001, 1, 512, 2, 64, 64, "f32", "raw", 1.0),
    "prefill_8k": Workload("prefill_8k", "prefill", 1002, 1, 8192, 64, 128, 256, "bf16", "rmsnorm_gate", 0.5),
    "prefill_128k": Workload("prefill_128k", "prefill", 1003, 1, 131072, 64, 128, 256, "bf16", "rmsnorm_gate", 0.5),
    "varlen_16": Workload("varlen_16", "varlen", 1004, 16, 0, 64, 128, 256, "bf16", "rmsnorm_gate", 0.5,
                          len_lo=1000, len_hi=32768),
    "decode_256": Workload("decode_256", "decode", 1005, 256, 0, 64, 128, 0, "bf16", "rmsnorm_gate", 0.5),
    # A serving step: 256 sequences decode one token each while 2 others prefill a 4096-token
    # chunk from their state (chunked prefill), all packed into one batch.
    "mixed_256": Workload("mixed_256", "mixed", 1006, 256, 4096, 64, 128, 256, "bf16", "rmsnorm_gate", 0.5,
                          n_prefill=2),
    # The backward of the 128K prefill (gradients of q, k, v and the gate from dout ~ N(0, 1)),
    # and an 8K version for captures.
    "backward_128k": Workload("backward_128k", "backward", 1007, 1, 131072, 64, 128, 256, "bf16", "rmsnorm_gate",
                              0.5),
    "backward_8k": Workload("backward_8k", "backward", 1008, 1, 8192, 64, 128, 256, "bf16", "rmsnorm_gate", 0.5),
    # The normalised variant at the 128K prefill's shapes; q and k shifted by +1 so the
    # denominators phi(q) . z stay positive.
    "znorm_128k": Workload("znorm_128k", "znorm", 1009, 1, 131072, 64, 128, 256, "bf16", "rmsnorm_gate", 0.5,
                           qk_shift=1.0),
    # The 128K prefill's shapes at 32K tokens: inputs four times L2, small enough for DRAM
    # counter captures of every kernel of one call.
    "prefill_32k": Workload("prefill_32k", "prefill", 1013, 1, 32768, 64, 128, 256, "bf16", "rmsnorm_gate", 0.5),
    # One 128K sequence with 8 heads (a tensor-parallel shard of the 64): the few-heads case.
    "prefill_128k_h8": Workload("prefill_128k_h8", "prefill", 1012, 1, 131072, 8, 128, 256, "bf16", "rmsnorm_gate",
                                0.5),
    # A training step on the 128K prefill's shapes: forward (keeping y) and backward.
    "train_128k": Workload("train_128k", "train", 1011, 1, 131072, 64, 128, 256, "bf16", "rmsnorm_gate", 0.5),
    # Step 1 of the sequence-parallel prefill on the 128K prefill's shapes: the state from k, v.
    "chunk_state_128k": Workload("chunk_state_128k", "chunk_state", 1010, 1, 131072, 64, 128, 0, "bf16", "raw", 0.5),
}


def shifted(a: np.ndarray, shift: float) -> np.ndarray:
    """a + shift rounded back to a's dtype (bf16 bits or fp32); a itself if shift is 0."""
    if shift == 0.0:
        return a
    if a.dtype == np.uint16:
        return f32_to_bf16(bf16_to_f32(a) + np.float32(shift))
    return (a + np.float32(shift)).astype(np.float32)


def mixed_lengths(w: Workload) -> np.ndarray:
    """Sequence lengths of a mixed step: each prefill chunk is followed by its share of the
    one-token (decode) sequences."""
    lens = []
    per = w.B // max(w.n_prefill, 1)
    for i in range(w.n_prefill):
        lens.append(w.T)
        lens.extend([1] * (per if i < w.n_prefill - 1 else w.B - per * (w.n_prefill - 1)))
    if w.n_prefill == 0:
        lens.extend([1] * w.B)
    return np.asarray(lens, dtype=np.int64)


def varlen_lengths(w: Workload) -> np.ndarray:
    return uniform_int(w.seed, STREAM_LEN, w.B, w.len_lo, w.len_hi)


def cu_seqlens_of(lengths) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def prefill_inputs(seed: int, tokens: int, H: int, D: int, dtype: str, qkv_scale: float,
                   with_gate: bool, token_offset: int = 0):
    """q, k, v (and g) of `tokens` rows laid out [tokens, H, D] (g: [tokens, H*D]).

    `token_offset` selects rows [token_offset, token_offset + tokens) of the same
    seeded stream, so a sample of a large workload has the same bytes as the
    corresponding rows of the full workload.
    """
    n = H * D
    q = normal(seed, STREAM_Q, (tokens, H, D), qkv_scale, dtype, offset=token_offset * n)
    k = normal(seed, STREAM_K, (tokens, H, D), qkv_scale, dtype, offset=token_offset * n)
    v = normal(seed, STREAM_V, (tokens, H, D), qkv_scale, dtype, offset=token_offset * n)
    g = normal(seed, STREAM_G, (tokens, H * D), 1.0, dtype, offset=token_offset * n) if with_gate else None
    return q, k, v, g


def decode_state(seed: int, B: int, H: int, D: int, out: np.ndarray | None = None) -> np.ndarray:
    """Prior decode state S ~ N(0,1)/sqrt(D), fp32, [B, H, D, D]."""
    return normal(seed, STREAM_S, (B, H, D, D), 1.0 / np.sqrt(D), "f32", out=out)


def decode_tokens(seed: int, step: int, B: int, H: int, D: int, dtype: str, qkv_scale: float):
    """q, k, v [B, H, D] and g [B, H*D] of decode step `step` (one token per sequence)."""
    n = B * H * D
    q = normal(seed, STREAM_Q, (B, H, D), qkv_scale, dtype, offset=step * n)
    k = normal(seed, STREAM_K, (B, H, D), qkv_scale, dtype, offset=step * n)
    v = normal(seed, STREAM_V, (B, H, D), qkv_scale, dtype, offset=step * n)
    g = normal(seed, STREAM_G, (B, H * D), 1.0, dtype, offset=step * n)
    return q, k, v, g
