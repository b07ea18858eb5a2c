"""Thin ctypes binding of liblightning_attn.so (argument marshalling only).

The functions carry the names of the C ABI in include/lightning_attn.h.  They take
torch tensors (device memory and streams come from PyTorch), pass raw pointers and
sizes to the library, and raise LightningAttnError on a non-OK status.  Every step of
the computation runs in the library's CUDA kernels; there is no Python or CPU path, and
a missing library raises at import.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblightning_attn.so")

LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA, LA_ERR_TIMEOUT, LA_ERR_DEVICE = range(6)
LA_F32, LA_BF16 = 0, 1
LA_OUT_RAW, LA_OUT_RMSNORM, LA_OUT_RMSNORM_GATE = 0, 1, 2
LA_PHI_SILU, LA_PHI_IDENTITY = 0, 1
(LA_OP_PREFILL, LA_OP_PREFILL_VARLEN, LA_OP_DECODE, LA_OP_MIXED, LA_OP_BACKWARD, LA_OP_BACKWARD_VARLEN,
 LA_OP_PREFILL_ZNORM, LA_OP_PREFILL_ZNORM_VARLEN, LA_OP_CHUNK_STATE, LA_OP_OUTPUT_TRANSFORM_BACKWARD) = range(10)

# The symbols include/lightning_attn.h declares (checked by tests/test_abi.py).
EXPORTED = (
    "lightning_attn_prefill",
    "lightning_attn_prefill_varlen",
    "lightning_attn_prefill_znorm",
    "lightning_attn_prefill_znorm_varlen",
    "lightning_attn_backward",
    "lightning_attn_backward_varlen",
    "lightning_attn_decode_step_znorm",
    "lightning_attn_decode_step",
    "lightning_attn_decode_step_noalloc",
    "lightning_attn_mixed_step",
    "lightning_attn_state_prefix",
    "lightning_attn_chunk_state",
    "lightning_attn_output_transform",
    "lightning_attn_output_transform_backward",
    "lightning_attn_workspace_size",
    "lightning_attn_check",
    "lightning_attn_status_string",
    "lightning_attn_last_path",
)


class LightningAttnError(RuntimeError):
    def __init__(self, status: int, where: str, detail=None):
        self.status = status
        self.detail = detail
        super().__init__(f"{where}: {status_string(status)}" + (f" detail={detail}" if detail else ""))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m long_context_attn_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.lightning_attn_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                           f32, vp, vp, sz, vp]
    lib.lightning_attn_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                  i32, i32, i32, f32, vp, vp, sz, vp]
    lib.lightning_attn_prefill_znorm.argtypes = [vp] * 9 + [i32] * 8 + [f32, vp, vp, sz, vp]
    lib.lightning_attn_prefill_znorm_varlen.argtypes = [vp] * 10 + [i32] * 9 + [f32, vp, vp, sz, vp]
    lib.lightning_attn_decode_step_znorm.argtypes = [vp] * 7 + [i32] * 6 + [f32, vp, vp, sz, vp]
    lib.lightning_attn_backward.argtypes = [vp] * 14 + [i32] * 8 + [f32, vp, vp, sz, vp]
    lib.lightning_attn_backward_varlen.argtypes = [vp] * 15 + [i32] * 9 + [f32, vp, vp, sz, vp]
    lib.lightning_attn_output_transform.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, vp]
    lib.lightning_attn_output_transform_backward.argtypes = [vp] * 6 + [i32] * 5 + [f32, vp, vp, sz, vp]
    lib.lightning_attn_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp,
                                               sz, vp]
    lib.lightning_attn_decode_step_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32,
                                                       vp, vp]
    lib.lightning_attn_mixed_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                              f32, vp, vp, sz, vp, vp]
    lib.lightning_attn_state_prefix.argtypes = [vp, i32, i32, vp, vp, i32, i32, vp]
    lib.lightning_attn_chunk_state.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, sz, vp]
    lib.lightning_attn_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32]
    lib.lightning_attn_workspace_size.restype = sz
    lib.lightning_attn_check.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint * 4)]
    lib.lightning_attn_status_string.argtypes = [i32]
    lib.lightning_attn_status_string.restype = ctypes.c_char_p
    lib.lightning_attn_last_path.argtypes = []
    lib.lightning_attn_last_path.restype = ctypes.c_char_p
    for f in ("lightning_attn_prefill", "lightning_attn_prefill_varlen", "lightning_attn_backward",
              "lightning_attn_backward_varlen", "lightning_attn_prefill_znorm", "lightning_attn_prefill_znorm_varlen",
              "lightning_attn_decode_step_znorm", "lightning_attn_decode_step",
              "lightning_attn_decode_step_noalloc", "lightning_attn_mixed_step", "lightning_attn_state_prefix", "lightning_attn_chunk_state",
              "lightning_attn_output_transform", "lightning_attn_output_transform_backward",
              "lightning_attn_check"):
        getattr(lib, f).restype = i32
    return lib


_lib = _load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LA_BF16
    if t.dtype == torch.float32:
        return LA_F32
    raise TypeError(f"q/k/v/g/out must be bfloat16 or float32, got {t.dtype}")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _f32_or_none(t):
    if t is None:
        return None
    if t.dtype != torch.float32 or not t.is_contiguous():
        raise TypeError("states and norm_weight must be contiguous float32 tensors")
    return t


def _check_contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def status_string(status: int) -> str:
    return _lib.lightning_attn_status_string(int(status)).decode()


def lightning_attn_status_string(status: int) -> str:
    return status_string(status)


def lightning_attn_last_path() -> str:
    return _lib.lightning_attn_last_path().decode()


def lightning_attn_workspace_size(op: int, B_or_N: int, T_or_max: int, total_tokens: int, H: int, D: int,
                                  block_size: int, dtype: int, mode: int) -> int:
    return int(_lib.lightning_attn_workspace_size(op, B_or_N, T_or_max, total_tokens, H, D, block_size, dtype,
                                                  mode))


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled uint8 device buffer (the caching allocator aligns it to >= 512 bytes)."""
    ws = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def lightning_attn_prefill(q, k, v, g, out, state_in=None, state_out=None, block_size=256,
                           phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE, eps=1e-6, norm_weight=None,
                           workspace=None, stream=None):
    """q, k, v [B, T, H, D]; g, out [B, T, H*D]; states fp32 [B, H, D, D]."""
    B, T, H, D = q.shape
    _check_contig(q, k, v, g, out)
    st = _lib.lightning_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out), _ptr(_f32_or_none(state_in)),
                                     _ptr(_f32_or_none(state_out)), B, T, H, D, block_size, _dtype(q), phi, mode,
                                     eps, _ptr(_f32_or_none(norm_weight)), _ptr(workspace),
                                     0 if workspace is None else workspace.numel(), _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_prefill")


def lightning_attn_prefill_varlen(q, k, v, g, out, cu_seqlens, max_seqlen, state_in=None, state_out=None,
                                  block_size=256, phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE, eps=1e-6,
                                  norm_weight=None, workspace=None, stream=None):
    """q, k, v [total, H, D]; g, out [total, H*D]; cu_seqlens int32 device [N + 1]."""
    total, H, D = q.shape
    _check_contig(q, k, v, g, out, cu_seqlens)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    n = cu_seqlens.numel() - 1
    st = _lib.lightning_attn_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out),
                                            _ptr(_f32_or_none(state_in)), _ptr(_f32_or_none(state_out)),
                                            _ptr(cu_seqlens), n, int(max_seqlen), total, H, D, block_size, _dtype(q),
                                            phi, mode, eps, _ptr(_f32_or_none(norm_weight)), _ptr(workspace),
                                            0 if workspace is None else workspace.numel(), _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_prefill_varlen")


def lightning_attn_prefill_znorm(q, k, v, g, out, state_in=None, z_in=None, state_out=None, z_out=None,
                                 block_size=256, phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE, eps=1e-6,
                                 norm_weight=None, workspace=None, stream=None):
    """Normalised variant: q, k, v [B, T, H, D]; g, out [B, T, H*D]; S fp32 [B, H, D, D]; z fp32 [B, H, D]."""
    B, T, H, D = q.shape
    _check_contig(q, k, v, g, out)
    st = _lib.lightning_attn_prefill_znorm(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out),
                                           _ptr(_f32_or_none(state_in)), _ptr(_f32_or_none(z_in)),
                                           _ptr(_f32_or_none(state_out)), _ptr(_f32_or_none(z_out)), B, T, H, D,
                                           block_size, _dtype(q), phi, mode, eps, _ptr(_f32_or_none(norm_weight)),
                                           _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                           _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_prefill_znorm")


def lightning_attn_prefill_znorm_varlen(q, k, v, g, out, cu_seqlens, max_seqlen, state_in=None, z_in=None,
                                        state_out=None, z_out=None, block_size=256, phi=LA_PHI_SILU,
                                        mode=LA_OUT_RMSNORM_GATE, eps=1e-6, norm_weight=None, workspace=None,
                                        stream=None):
    """Normalised variant over packed sequences: q, k, v [total, H, D]; g, out [total, H*D]."""
    total, H, D = q.shape
    _check_contig(q, k, v, g, out, cu_seqlens)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    n = cu_seqlens.numel() - 1
    st = _lib.lightning_attn_prefill_znorm_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out),
                                                  _ptr(_f32_or_none(state_in)), _ptr(_f32_or_none(z_in)),
                                                  _ptr(_f32_or_none(state_out)), _ptr(_f32_or_none(z_out)),
                                                  _ptr(cu_seqlens), n, int(max_seqlen), total, H, D, block_size,
                                                  _dtype(q), phi, mode, eps, _ptr(_f32_or_none(norm_weight)),
                                                  _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                                  _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_prefill_znorm_varlen")


def lightning_attn_decode_step_znorm(q, k, v, g, out, state, z, phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE,
                                     eps=1e-6, norm_weight=None, workspace=None, stream=None):
    """Normalised-variant decode: q, k, v [B, H, D]; g, out [B, H*D]; state [B, H, D, D] and z [B, H, D]
    fp32, both updated in place."""
    B, H, D = q.shape
    _check_contig(q, k, v, g, out, state, z)
    st = _lib.lightning_attn_decode_step_znorm(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out),
                                               _ptr(_f32_or_none(state)), _ptr(_f32_or_none(z)), B, H, D, _dtype(q),
                                               phi, mode, eps, _ptr(_f32_or_none(norm_weight)), _ptr(workspace),
                                               0 if workspace is None else workspace.numel(), _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_decode_step_znorm")


def lightning_attn_backward(q, k, v, g, dout, dq, dk, dv, dg=None, state_in=None, dstate_in=None, block_size=256,
                            phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE, eps=1e-6, norm_weight=None, workspace=None,
                            stream=None, dstate_out=None, y=None, dnorm_weight=None):
    """q, k, v, dq, dk, dv [B, T, H, D]; g, dout, dg [B, T, H*D]; states fp32 [B, H, D, D]
    (dstate_out: the gradient reaching the final states; y: the forward's raw output, saved;
    dnorm_weight: fp32 [H*D] receiving the norm weight's gradient)."""
    B, T, H, D = q.shape
    _check_contig(q, k, v, g, dout, dq, dk, dv, dg, dstate_out, y)
    st = _lib.lightning_attn_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dout), _ptr(_f32_or_none(state_in)),
                                      _ptr(_f32_or_none(dstate_out)), _ptr(y), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                                      _ptr(_f32_or_none(dstate_in)), _ptr(_f32_or_none(dnorm_weight)), B, T, H,
                                      D, block_size, _dtype(q), phi, mode, eps, _ptr(_f32_or_none(norm_weight)),
                                      _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                      _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_backward")


def lightning_attn_backward_varlen(q, k, v, g, dout, dq, dk, dv, cu_seqlens, max_seqlen, dg=None, state_in=None,
                                   dstate_in=None, block_size=256, phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE,
                                   eps=1e-6, norm_weight=None, workspace=None, stream=None, dstate_out=None,
                                   y=None, dnorm_weight=None):
    """q, k, v, dq, dk, dv [total, H, D]; g, dout, dg [total, H*D]; cu_seqlens int32 device [N + 1]."""
    total, H, D = q.shape
    _check_contig(q, k, v, g, dout, dq, dk, dv, dg, cu_seqlens, dstate_out, y)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    n = cu_seqlens.numel() - 1
    st = _lib.lightning_attn_backward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dout),
                                             _ptr(_f32_or_none(state_in)), _ptr(_f32_or_none(dstate_out)), _ptr(y),
                                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                                             _ptr(_f32_or_none(dstate_in)), _ptr(_f32_or_none(dnorm_weight)),
                                             _ptr(cu_seqlens), n, int(max_seqlen),
                                             total, H, D, block_size, _dtype(q), phi, mode, eps,
                                             _ptr(_f32_or_none(norm_weight)), _ptr(workspace),
                                             0 if workspace is None else workspace.numel(), _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_backward_varlen")


def lightning_attn_decode_step(q, k, v, g, out, state, phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE, eps=1e-6,
                               norm_weight=None, workspace=None, stream=None):
    """q, k, v [B, H, D]; g, out [B, H*D]; state fp32 [B, H, D, D] updated in place."""
    B, H, D = q.shape
    _check_contig(q, k, v, g, out, state)
    st = _lib.lightning_attn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out), _ptr(_f32_or_none(state)),
                                         B, H, D, _dtype(q), phi, mode, eps, _ptr(_f32_or_none(norm_weight)),
                                         _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                         _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_decode_step")


def lightning_attn_decode_step_noalloc(q, k, v, g, out, state, phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE,
                                       eps=1e-6, norm_weight=None, stream=None):
    """Decode step without a workspace, for callers that cannot allocate device memory.

    Same arguments and results as lightning_attn_decode_step; the scratch is a fixed array
    inside the library shared by every call (calls that overlap on the GPU race), and
    batches that do not fit it raise with LA_ERR_UNSUPPORTED.
    """
    B, H, D = q.shape
    _check_contig(q, k, v, g, out, state)
    dev = torch.cuda.current_device()
    for t in (q, k, v, g, out, state, norm_weight):
        if t is not None and (t.device.type != "cuda" or t.device.index != dev):
            raise ValueError(f"tensors must be on the current CUDA device cuda:{dev}, got {t.device}")
    st = _lib.lightning_attn_decode_step_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out),
                                                 _ptr(_f32_or_none(state)), B, H, D, _dtype(q), phi, mode, eps,
                                                 _ptr(_f32_or_none(norm_weight)), _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_decode_step_noalloc")


def lightning_attn_mixed_step(q, k, v, g, out, cu_seqlens, cu_seqlens_host, state_pool, state_slot,
                              block_size=256, phi=LA_PHI_SILU, mode=LA_OUT_RMSNORM_GATE, eps=1e-6, norm_weight=None,
                              workspace=None, prefill_stream=None, decode_stream=None):
    """One serving step over packed sequences: one-token sequences decode, longer ones prefill
    from their state.  q, k, v [total, H, D]; g, out [total, H*D]; cu_seqlens int32 device
    [N + 1] with the same values in `cu_seqlens_host` (a host sequence of ints); state_pool
    fp32 [P, H, D, D] updated in place; state_slot int32 device [N] (distinct slots)."""
    total, H, D = q.shape
    _check_contig(q, k, v, g, out, cu_seqlens, state_pool, state_slot)
    if cu_seqlens.dtype != torch.int32 or state_slot.dtype != torch.int32:
        raise TypeError("cu_seqlens and state_slot must be int32")
    n = cu_seqlens.numel() - 1
    host = (ctypes.c_int * (n + 1))(*[int(x) for x in cu_seqlens_host])
    st = _lib.lightning_attn_mixed_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(out), _ptr(cu_seqlens),
                                        ctypes.cast(host, ctypes.c_void_p), _ptr(_f32_or_none(state_pool)),
                                        _ptr(state_slot), n, H, D, block_size, _dtype(q), phi, mode, eps,
                                        _ptr(_f32_or_none(norm_weight)), _ptr(workspace),
                                        0 if workspace is None else workspace.numel(), _stream(prefill_stream),
                                        _stream(decode_stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_mixed_step")


def lightning_attn_output_transform(y, g, out, mode=LA_OUT_RMSNORM_GATE, eps=1e-6, norm_weight=None, stream=None):
    """out = RMSNorm(y) * w (* sigmoid(g)) per token: y, g, out [..., H*D] with H*D the last axis;
    H and D from y's last two dims when y is [..., H, D], else pass y as [tokens, H, D]."""
    if y.dim() < 2:
        raise ValueError("y must be [..., H, D]")
    H, D = y.shape[-2], y.shape[-1]
    tokens = y.numel() // (H * D)
    _check_contig(y, g, out)
    st = _lib.lightning_attn_output_transform(_ptr(y), _ptr(g), _ptr(out), tokens, H, D, _dtype(y), mode, eps,
                                              _ptr(_f32_or_none(norm_weight)), _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_output_transform")


def lightning_attn_output_transform_backward(y, g, dout, dy, dg=None, dnorm_weight=None, mode=LA_OUT_RMSNORM_GATE,
                                            eps=1e-6, norm_weight=None, workspace=None, stream=None):
    """dy, dg (and the norm weight's gradient) from dout through the output transform of y:
    y, g, dout, dy, dg hold tokens * H * D elements each, H and D taken from the last two dims
    of y viewed as [..., H, D] (of dout when y is None, in raw mode); dnorm_weight fp32 [H*D]."""
    src = y if y is not None else dout
    if src.dim() < 2:
        raise ValueError("y (or dout) must be [..., H, D]")
    H, D = src.shape[-2], src.shape[-1]
    tokens = src.numel() // (H * D)
    _check_contig(y, g, dout, dy, dg)
    st = _lib.lightning_attn_output_transform_backward(_ptr(y), _ptr(g), _ptr(dout), _ptr(dy), _ptr(dg),
                                                       _ptr(_f32_or_none(dnorm_weight)), tokens, H, D, _dtype(dout),
                                                       mode, eps, _ptr(_f32_or_none(norm_weight)), _ptr(workspace),
                                                       0 if workspace is None else workspace.numel(),
                                                       _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_output_transform_backward")


def lightning_attn_chunk_state(k, v, state_out, state_in=None, phi=LA_PHI_SILU, workspace=None, stream=None):
    """state_out = state_in + sum_t phi(k_t) v_t^T: k, v [B, T, H, D]; states fp32 [B, H, D, D]."""
    B, T, H, D = k.shape
    _check_contig(k, v, state_out, state_in)
    st = _lib.lightning_attn_chunk_state(_ptr(k), _ptr(v), _ptr(_f32_or_none(state_in)),
                                         _ptr(_f32_or_none(state_out)), B, T, H, D, _dtype(k), phi, _ptr(workspace),
                                         0 if workspace is None else workspace.numel(), _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_chunk_state")


def lightning_attn_state_prefix(gathered, rank, out, state0=None, stream=None):
    """out[H, D, D] = state0 + sum over ranks j < rank of gathered[j] (rank order)."""
    world, H, D, _ = gathered.shape
    _check_contig(gathered, out)
    st = _lib.lightning_attn_state_prefix(_ptr(_f32_or_none(gathered)), world, int(rank),
                                          _ptr(_f32_or_none(state0)), _ptr(_f32_or_none(out)), H, D,
                                          _stream(stream))
    if st != LA_OK:
        raise LightningAttnError(st, "lightning_attn_state_prefix")


def lightning_attn_check(workspace, stream=None, raise_on_error=True):
    """Synchronise the stream and read/clear the device error record of `workspace`."""
    detail = (ctypes.c_uint * 4)()
    st = _lib.lightning_attn_check(_ptr(workspace), _stream(stream), ctypes.byref(detail))
    if st != LA_OK and raise_on_error:
        raise LightningAttnError(st, "lightning_attn_check", tuple(detail))
    return st, tuple(detail)
