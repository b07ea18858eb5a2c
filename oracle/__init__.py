"""fp64 CPU oracle for the Lightning Attention forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg
and ``--impl reference`` arm) may import this package.  The product path (the C-ABI
library and its Python binding) never imports, links or calls it, and the oracle
shares no code with the CUDA path; only the seeded input generator (``synth``) feeds
both sides.

The arithmetic lives in ``lightning_oracle.cpp`` (plain C++17, fp64, OpenMP over
heads); this module builds it with gcc and wraps it with ctypes.  What each function
computes, and which passage of the pages it follows, is documented there:
  * ``forward_packed`` / ``prefill`` / ``decode`` -- the token-by-token recurrence
    S_t = S_{t-1} + phi(k_t) v_t^T, y_t = phi(q_t)^T S_t ("六十四：MiniMax-01", section 3)
    followed by RMSNorm over the head concatenation times sigmoid(gate)
    ("MiniMax-Text-01 405B MoE模型架构与训练策略解析", section 2.1);
  * ``quadratic`` -- restatement R1, (phi(Q) phi(K)^T (.) M) V;
  * ``chunked``   -- restatement R2, block-wise intra + inter form for any block size;
  * ``transform`` -- the output transform alone;
  * ``forward_znorm_packed`` / ``prefill_znorm`` -- the normalised variant, y = phi(q)^T S /
    (phi(q) . z) with z_t = z_{t-1} + phi(k_t) ("六十四：MiniMax-01", section 3);
  * ``backward_packed`` / ``backward`` -- the gradients of the forward (chain rule through
    the output transform, the recurrence and the feature map; pinned by finite differences
    of ``forward_packed``).

Parity pins for every function are in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lightning_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liblightning_oracle.so")
_lib = None

DT_F32, DT_BF16 = 0, 1
PHI_SILU, PHI_IDENTITY = 0, 1
MODE_RAW, MODE_RMSNORM, MODE_RMSNORM_GATE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle into liblightning_oracle.so (g++, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-march=x86-64-v3", "-fPIC", "-shared",
                               "-fopenmp", "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _get():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_forward_packed.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, vp, i32, i32, dbl,
                                              vp, vp, vp, vp, vp, vp]
        lib.oracle_prefill.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, i32, i32, dbl, vp,
                                       vp, vp, vp, vp, vp]
        lib.oracle_decode.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, i32, i32, dbl, vp, vp,
                                      vp, vp, vp, vp]
        lib.oracle_quadratic.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp]
        lib.oracle_chunked.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp]
        lib.oracle_transform.argtypes = [vp, i64, i32, i32, i32, dbl, vp, vp, i32, vp]
        lib.oracle_forward_znorm_packed.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, vp, vp, i32, i32, dbl,
                                                    vp, vp, vp, vp]
        lib.oracle_backward_packed.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, vp, vp, i32, i32, dbl,
                                               vp, vp, vp, vp, vp, vp, vp]
        lib.oracle_transform_backward.argtypes = [vp, vp, vp, i32, i64, i32, i32, i32, dbl, vp, vp, vp, vp]
        lib.oracle_backward_znorm_packed.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, vp, vp, vp, vp, i32,
                                                     i32, dbl, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        for f in (lib.oracle_forward_packed, lib.oracle_prefill, lib.oracle_decode,
                  lib.oracle_quadratic, lib.oracle_chunked, lib.oracle_transform, lib.oracle_backward_packed,
                  lib.oracle_forward_znorm_packed, lib.oracle_transform_backward, lib.oracle_backward_znorm_packed):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return DT_BF16
    if a.dtype == np.float32:
        return DT_F32
    raise TypeError(f"inputs must be bf16 bits (uint16) or float32, got {a.dtype}")


def _c(a, dtype=None):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype) if dtype is not None else np.ascontiguousarray(a)


class Stats(dict):
    """max_ref / max_err / argmax / nonfinite for the output and the state."""


def _stats(buf):
    return Stats(out_max_ref=buf[0], out_max_err=buf[1], out_argmax=int(buf[2]), out_nonfinite=int(buf[3]),
                 state_max_ref=buf[4], state_max_err=buf[5], state_argmax=int(buf[6]),
                 state_nonfinite=int(buf[7]))


def forward_packed(q, k, v, g, cu_seqlens, H, D, state_in=None, phi=PHI_SILU, mode=MODE_RMSNORM_GATE,
                   eps=1e-6, norm_weight=None, store=True, cand_out=None, cand_state=None):
    """Packed sequences: q, k, v [tokens, H, D]; g [tokens, H*D]; cu_seqlens [N+1].

    Returns (out fp64 [tokens, H*D] or None, state fp64 [N, H, D, D], stats or None).
    """
    q, k, v, g = _c(q), _c(k), _c(v), _c(g)
    dt = _dtype_code(q)
    cu = _c(cu_seqlens, np.int32)
    N = cu.size - 1
    tokens = int(cu[-1]) if N > 0 else 0
    out = np.empty((tokens, H * D), dtype=np.float64) if store else None
    st = np.empty((N, H, D, D), dtype=np.float64)
    stats = np.zeros(8, dtype=np.float64) if (cand_out is not None or cand_state is not None) else None
    cand_out = _c(cand_out)
    cand_state = _c(cand_state, np.float32)
    s_in, w = _c(state_in, np.float32), _c(norm_weight, np.float32)   # held until the call returns
    rc = _get().oracle_forward_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), dt, _ptr(cu), N, H, D,
                                      _ptr(s_in), phi, mode, eps,
                                      _ptr(w), _ptr(out), _ptr(st),
                                      _ptr(cand_out), _ptr(cand_state), _ptr(stats))
    if rc != 0:
        raise ValueError("oracle_forward_packed rejected its arguments")
    return out, st, (_stats(stats) if stats is not None else None)


def prefill(q, k, v, g=None, state_in=None, phi=PHI_SILU, mode=MODE_RMSNORM_GATE, eps=1e-6,
            norm_weight=None, store=True, cand_out=None, cand_state=None):
    """Fixed-length batch: q, k, v [B, T, H, D]; g [B, T, H*D]."""
    B, T, H, D = q.shape
    cu = np.arange(B + 1, dtype=np.int32) * T
    out, st, stats = forward_packed(np.reshape(q, (B * T, H, D)), np.reshape(k, (B * T, H, D)),
                                    np.reshape(v, (B * T, H, D)),
                                    None if g is None else np.reshape(g, (B * T, H * D)), cu, H, D,
                                    state_in, phi, mode, eps, norm_weight, store,
                                    None if cand_out is None else np.reshape(cand_out, (B * T, H * D)),
                                    cand_state)
    if out is not None:
        out = out.reshape(B, T, H * D)
    return out, st, stats


def decode(q, k, v, g, state_in, phi=PHI_SILU, mode=MODE_RMSNORM_GATE, eps=1e-6, norm_weight=None,
           cand_out=None, cand_state=None):
    """One decode step: q, k, v [B, H, D]; g [B, H*D]; state_in fp32 [B, H, D, D]."""
    B, H, D = q.shape
    cu = np.arange(B + 1, dtype=np.int32)
    return forward_packed(q, k, v, g, cu, H, D, state_in, phi, mode, eps, norm_weight, True,
                          cand_out, cand_state)


def quadratic(q, k, v, phi=PHI_SILU):
    """R1: raw Y = (phi(Q) phi(K)^T (.) M) V for one sequence [T, H, D] (tiny inputs)."""
    q, k, v = _c(q), _c(k), _c(v)
    T, H, D = q.shape
    y = np.empty((T, H, D), dtype=np.float64)
    if _get().oracle_quadratic(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), T, H, D, phi, _ptr(y)) != 0:
        raise ValueError("oracle_quadratic rejected its arguments")
    return y


def chunked(q, k, v, C, phi=PHI_SILU, s0=None):
    """R2: raw block-wise result (block size C) for one sequence [T, H, D]; returns (y, S_T)."""
    q, k, v = _c(q), _c(k), _c(v)
    T, H, D = q.shape
    y = np.empty((T, H, D), dtype=np.float64)
    st = np.empty((H, D, D), dtype=np.float64)
    s0c = _c(s0, np.float64)   # held until the call returns
    if _get().oracle_chunked(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), T, H, D, C, phi,
                             _ptr(s0c), _ptr(y), _ptr(st)) != 0:
        raise ValueError("oracle_chunked rejected its arguments")
    return y, st


def num_threads() -> int:
    """OpenMP threads the oracle uses (the `cores` of a CPU timing)."""
    return int(_get().oracle_num_threads())


def transform(y, mode, eps=1e-6, norm_weight=None, g=None):
    """Output transform of raw y [tokens, H, D] (fp64); g [tokens, H*D] bf16 bits or fp32."""
    y = _c(y, np.float64)
    tokens, H, D = y.shape
    out = np.empty((tokens, H * D), dtype=np.float64)
    g = _c(g)
    dt = DT_F32 if g is None else _dtype_code(g)
    w = _c(norm_weight, np.float32)
    _get().oracle_transform(_ptr(y), tokens, H, D, mode, eps, _ptr(w), _ptr(g),
                            dt, _ptr(out))
    return out


def transform_backward(y, dout, mode, eps=1e-6, norm_weight=None, g=None):
    """Backward of `transform`: y fp64 [tokens, H, D]; dout, g [tokens, H*D] (bf16 bits or
    fp32, one dtype).  Returns fp64 (dy [tokens, H*D], dg [tokens, H*D] or None, dw [H*D])."""
    y = _c(y, np.float64)
    tokens, H, D = y.shape
    dout, g = _c(dout), _c(g)
    dt = _dtype_code(dout)
    w = _c(norm_weight, np.float32)
    dy = np.empty((tokens, H * D), dtype=np.float64)
    dg = np.empty((tokens, H * D), dtype=np.float64) if mode == MODE_RMSNORM_GATE else None
    dw = np.empty(H * D, dtype=np.float64)
    rc = _get().oracle_transform_backward(_ptr(y), _ptr(dout), _ptr(g), dt, tokens, H, D, mode, eps, _ptr(w),
                                          _ptr(dy), _ptr(dg), _ptr(dw))
    if rc != 0:
        raise ValueError("oracle_transform_backward rejected its arguments")
    return dy, dg, dw


def backward_packed(q, k, v, g, dout, cu_seqlens, H, D, state_in=None, phi=PHI_SILU, mode=MODE_RMSNORM_GATE,
                    eps=1e-6, norm_weight=None, dstate_out=None):
    """Gradients of forward_packed for the loss with output gradient dout [tokens, H*D] and
    final-state gradient dstate_out [N, H, D, D] (fp32, or None for zero).

    q, k, v [tokens, H, D], g and dout [tokens, H*D] (bf16 bits or fp32, all one dtype).
    Returns fp64 (dq, dk, dv [tokens, H, D], dg [tokens, H*D] or None, dstate [N, H, D, D],
    dw [H*D] -- the norm weight's gradient, zeros in raw mode).
    """
    q, k, v, g, dout = _c(q), _c(k), _c(v), _c(g), _c(dout)
    dt = _dtype_code(q)
    cu = _c(cu_seqlens, np.int32)
    N = cu.size - 1
    tokens = int(cu[-1]) if N > 0 else 0
    dq, dk, dv = (np.zeros((tokens, H, D), dtype=np.float64) for _ in range(3))
    dg = np.zeros((tokens, H * D), dtype=np.float64) if mode == MODE_RMSNORM_GATE else None
    dst = np.zeros((N, H, D, D), dtype=np.float64)
    dw = np.zeros(H * D, dtype=np.float64)
    s_in, ds_out, w = _c(state_in, np.float32), _c(dstate_out, np.float32), _c(norm_weight, np.float32)
    rc = _get().oracle_backward_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dout), dt, _ptr(cu), N, H, D,
                                       _ptr(s_in), _ptr(ds_out), phi, mode, eps, _ptr(w), _ptr(dq), _ptr(dk),
                                       _ptr(dv), _ptr(dg), _ptr(dst), _ptr(dw))
    if rc != 0:
        raise ValueError("oracle_backward_packed rejected its arguments")
    return dq, dk, dv, dg, dst, dw


def backward(q, k, v, g, dout, state_in=None, phi=PHI_SILU, mode=MODE_RMSNORM_GATE, eps=1e-6,
             norm_weight=None, dstate_out=None):
    """Fixed-length batch: q, k, v [B, T, H, D]; g, dout [B, T, H*D]; states [B, H, D, D]."""
    B, T, H, D = q.shape
    cu = np.arange(B + 1, dtype=np.int32) * T
    r = lambda a, s: None if a is None else np.reshape(a, s)
    dq, dk, dv, dg, dst, dw = backward_packed(r(q, (B * T, H, D)), r(k, (B * T, H, D)), r(v, (B * T, H, D)),
                                          r(g, (B * T, H * D)), r(dout, (B * T, H * D)), cu, H, D, state_in,
                                          phi, mode, eps, norm_weight, dstate_out)
    return (dq.reshape(B, T, H, D), dk.reshape(B, T, H, D), dv.reshape(B, T, H, D),
            None if dg is None else dg.reshape(B, T, H * D), dst, dw)


def forward_znorm_packed(q, k, v, g, cu_seqlens, H, D, state_in=None, z_in=None, phi=PHI_SILU,
                         mode=MODE_RMSNORM_GATE, eps=1e-6, norm_weight=None):
    """Normalised variant over packed sequences: q, k, v [tokens, H, D]; g [tokens, H*D];
    state_in [N, H, D, D], z_in [N, H, D] (fp32 or None).  Returns fp64 (out [tokens, H*D],
    state [N, H, D, D], z [N, H, D])."""
    q, k, v, g = _c(q), _c(k), _c(v), _c(g)
    dt = _dtype_code(q)
    cu = _c(cu_seqlens, np.int32)
    N = cu.size - 1
    tokens = int(cu[-1]) if N > 0 else 0
    out = np.empty((tokens, H * D), dtype=np.float64)
    st = np.empty((N, H, D, D), dtype=np.float64)
    z = np.empty((N, H, D), dtype=np.float64)
    s_in, zz, w = _c(state_in, np.float32), _c(z_in, np.float32), _c(norm_weight, np.float32)
    rc = _get().oracle_forward_znorm_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), dt, _ptr(cu), N, H, D,
                                            _ptr(s_in), _ptr(zz), phi, mode, eps, _ptr(w), _ptr(out), _ptr(st),
                                            _ptr(z))
    if rc != 0:
        raise ValueError("oracle_forward_znorm_packed rejected its arguments")
    return out, st, z


def backward_znorm_packed(q, k, v, g, dout, cu_seqlens, H, D, state_in=None, z_in=None, phi=PHI_SILU,
                          mode=MODE_RMSNORM_GATE, eps=1e-6, norm_weight=None, dstate_out=None, dz_out=None):
    """Gradients of forward_znorm_packed for the loss with output gradient dout [tokens, H*D]
    and final-state gradients dstate_out [N, H, D, D], dz_out [N, H, D] (fp32 or None).
    Returns fp64 (dq, dk, dv [tokens, H, D], dg [tokens, H*D] or None, dstate [N, H, D, D],
    dz [N, H, D], dw [H*D])."""
    q, k, v, g, dout = _c(q), _c(k), _c(v), _c(g), _c(dout)
    dt = _dtype_code(q)
    cu = _c(cu_seqlens, np.int32)
    N = cu.size - 1
    tokens = int(cu[-1]) if N > 0 else 0
    dq, dk, dv = (np.zeros((tokens, H, D), dtype=np.float64) for _ in range(3))
    dg = np.zeros((tokens, H * D), dtype=np.float64) if mode == MODE_RMSNORM_GATE else None
    dst = np.zeros((N, H, D, D), dtype=np.float64)
    dz = np.zeros((N, H, D), dtype=np.float64)
    dw = np.zeros(H * D, dtype=np.float64)
    s_in, z0, w = _c(state_in, np.float32), _c(z_in, np.float32), _c(norm_weight, np.float32)
    ds_out, dz_o = _c(dstate_out, np.float32), _c(dz_out, np.float32)
    rc = _get().oracle_backward_znorm_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dout), dt, _ptr(cu), N, H, D,
                                             _ptr(s_in), _ptr(z0), _ptr(ds_out), _ptr(dz_o), phi, mode, eps, _ptr(w),
                                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dst), _ptr(dz), _ptr(dw))
    if rc != 0:
        raise ValueError("oracle_backward_znorm_packed rejected its arguments")
    return dq, dk, dv, dg, dst, dz, dw


def prefill_znorm(q, k, v, g=None, state_in=None, z_in=None, phi=PHI_SILU, mode=MODE_RMSNORM_GATE, eps=1e-6,
                  norm_weight=None):
    """Fixed-length batch of the normalised variant: q, k, v [B, T, H, D]; g [B, T, H*D]."""
    B, T, H, D = q.shape
    cu = np.arange(B + 1, dtype=np.int32) * T
    out, st, z = forward_znorm_packed(np.reshape(q, (B * T, H, D)), np.reshape(k, (B * T, H, D)),
                                      np.reshape(v, (B * T, H, D)),
                                      None if g is None else np.reshape(g, (B * T, H * D)), cu, H, D, state_in,
                                      z_in, phi, mode, eps, norm_weight)
    return out.reshape(B, T, H * D), st, z
