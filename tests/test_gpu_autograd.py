"""The autograd integration (long_context_attn_b200.autograd.lightning_attention): gradients
from loss.backward() against the oracle's fp64 backward.  The second case runs a sequence
as two chunks, the second starting from the first's state, so the gradients of the first
chunk flow back through the carried state (the backward's final-state gradient)."""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


def _leaf(a, shape):
    t = to_dev(a).reshape(shape).clone()
    t.requires_grad_(True)
    return t


def test_autograd_matches_oracle(cuda_device):
    import torch
    from long_context_attn_b200.autograd import lightning_attention
    B, T, H, D = 1, 700, 8, 128
    q, k, v, g = synth.prefill_inputs(3701, T, H, D, "bf16", 0.5, True)
    dout = synth.normal(3701, 21, (T, H * D), 1.0, "f32")
    s0 = synth.normal(3701, 22, (B, H, D, D), 0.05, "f32")
    dsT = synth.normal(3701, 24, (B, H, D, D), 0.05, "f32")
    shp, gshp = (B, T, H, D), (B, T, H * D)
    tq, tk, tv = (_leaf(a, shp) for a in (q, k, v))
    tg = _leaf(g, gshp)
    ts = torch.from_numpy(s0).cuda().requires_grad_(True)
    out, st = lightning_attention(tq, tk, tv, tg, ts)
    loss = (out.float() * torch.from_numpy(dout).cuda().reshape(gshp)).sum() + (st * torch.from_numpy(dsT).cuda()).sum()
    loss.backward()
    dout_b = synth.f32_to_bf16(dout)   # the backward sees dout in the activations' dtype
    ref = oracle.backward(q.reshape(shp), k.reshape(shp), v.reshape(shp), g.reshape(gshp), dout_b.reshape(gshp),
                          state_in=s0, dstate_out=dsT)
    for t, want, name in zip((tq, tk, tv, tg, ts), ref, ("dq", "dk", "dv", "dg", "dstate")):
        assert_close(to_host(t.grad), want.reshape(to_host(t.grad).shape), "bf16", name)


def test_autograd_through_the_carried_state(cuda_device):
    import torch
    from long_context_attn_b200.autograd import lightning_attention
    H, D, T1, T2 = 8, 128, 400, 333
    T = T1 + T2
    q, k, v, g = synth.prefill_inputs(3711, T, H, D, "bf16", 0.5, True)
    dout = synth.f32_to_bf16(synth.normal(3711, 21, (T, H * D), 1.0, "f32"))
    tq, tk, tv = (_leaf(a, (1, T, H, D)) for a in (q, k, v))
    tg = _leaf(g, (1, T, H * D))
    out1, s1 = lightning_attention(tq[:, :T1], tk[:, :T1], tv[:, :T1], tg[:, :T1])
    out2, _ = lightning_attention(tq[:, T1:], tk[:, T1:], tv[:, T1:], tg[:, T1:], state_in=s1)
    dd = to_dev(dout).reshape(1, T, H * D).float()
    loss = (out1.float() * dd[:, :T1]).sum() + (out2.float() * dd[:, T1:]).sum()
    loss.backward()
    ref = oracle.backward(q[None], k[None], v[None], g[None], dout[None])
    for t, want, name in zip((tq, tk, tv, tg), ref, ("dq", "dk", "dv", "dg")):
        assert_close(to_host(t.grad), want.reshape(to_host(t.grad).shape), "bf16", name)


def test_autograd_norm_weight_gradient(cuda_device):
    """A norm weight that requires grad gets dw = sum_t dout_t * y_t * r_t * sigmoid(g_t)."""
    import torch
    from long_context_attn_b200.autograd import lightning_attention
    B, T, H, D = 1, 520, 8, 128
    q, k, v, g = synth.prefill_inputs(3721, T, H, D, "bf16", 0.5, True)
    dout = synth.f32_to_bf16(synth.normal(3721, 21, (T, H * D), 1.0, "f32"))
    w = (1.0 + 0.2 * synth.normal(3721, 23, (H * D,), 1.0, "f32")).astype(np.float32)
    shp, gshp = (B, T, H, D), (B, T, H * D)
    tq, tk, tv = (_leaf(a, shp) for a in (q, k, v))
    tg = _leaf(g, gshp)
    tw = torch.from_numpy(w).cuda().requires_grad_(True)
    out, _ = lightning_attention(tq, tk, tv, tg, norm_weight=tw)
    (out.float() * to_dev(dout).reshape(gshp).float()).sum().backward()
    ref = oracle.backward(q.reshape(shp), k.reshape(shp), v.reshape(shp), g.reshape(gshp), dout.reshape(gshp),
                          norm_weight=w)
    for t, want, name in zip((tq, tk, tv, tg, tw), ref[:4] + ref[5:], ("dq", "dk", "dv", "dg", "dw")):
        assert_close(to_host(t.grad), want.reshape(to_host(t.grad).shape), "bf16", name)
