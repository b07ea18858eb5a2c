"""The autograd functions' host logic on CPU, the library calls replaced by the oracle
(each call first bound to the real binding's signature): the packed-sequence function's
gradients under loss.backward() against the oracle's backward, with initial states, a
final-state gradient, a trained norm weight and the gate, in the raw and gated modes."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_sequence_parallel_gloo import _OracleBackend


@pytest.fixture
def fake_la(monkeypatch):
    from long_context_attn_b200 import autograd as ag
    fake = _OracleBackend()
    fake.lightning_attn_workspace_size = lambda *a: 256
    fake.new_workspace = lambda n, device=None: torch.zeros(n, dtype=torch.uint8)
    for name in ("LA_OP_PREFILL_VARLEN", "LA_OP_BACKWARD_VARLEN"):
        setattr(fake, name, 0)
    monkeypatch.setattr(ag, "la", fake)
    return ag


@pytest.mark.parametrize("mode", [oracle.MODE_RAW, oracle.MODE_RMSNORM_GATE])
def test_varlen_autograd_matches_oracle(mode, fake_la):
    ag = fake_la
    H, D = 2, 16
    lens = [9, 0, 1, 14]
    cu = synth.cu_seqlens_of(lens)
    tot, n = int(cu[-1]), len(lens)
    q, k, v, g = synth.prefill_inputs(1551, tot, H, D, "f32", 0.5, True)
    dout = synth.normal(1551, 11, (tot, H * D), 1.0, "f32")
    s0 = synth.normal(1551, 9, (n, H, D, D), 0.1, "f32")
    dsT = synth.normal(1551, 10, (n, H, D, D), 0.1, "f32")
    w = (1.0 + 0.2 * synth.normal(1551, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    leaf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).requires_grad_(True)
    tq, tk, tv, tg, ts0, tw = (leaf(a) for a in (q, k, v, g, s0, w))
    gate = mode == oracle.MODE_RMSNORM_GATE
    out, st = ag.lightning_attention_varlen(tq, tk, tv, torch.from_numpy(cu), max(lens), g=tg if gate else None,
                                            state_in=ts0, mode=mode, norm_weight=tw if gate else None)
    loss = (out * torch.from_numpy(dout)).sum() + (st * torch.from_numpy(dsT)).sum()
    loss.backward()
    ref = oracle.backward_packed(q, k, v, g if gate else None, dout, cu, H, D, state_in=s0, mode=mode,
                                 norm_weight=w if gate else None, dstate_out=dsT)
    for t, want, name in zip((tq, tk, tv, tg, ts0), ref[:5], ("dq", "dk", "dv", "dg", "dS0")):
        if want is None:
            assert t.grad is None, name
            continue
        np.testing.assert_allclose(t.grad.numpy(), want, rtol=0, atol=1e-5 * np.abs(want).max(), err_msg=name)
    if gate:
        np.testing.assert_allclose(tw.grad.numpy(), ref[5], rtol=0, atol=1e-5 * np.abs(ref[5]).max(), err_msg="dw")
