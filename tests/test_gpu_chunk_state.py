"""GPU parity of lightning_attn_chunk_state (the state a prefill ends with, from k and v
alone) against the oracle's final state, and against the prefill kernel's own state."""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


def _la():
    from long_context_attn_b200 import lightning_attn as la
    return la


def _run(k, v, s0, dtype_la, phi=0):
    import torch
    la = _la()
    B, T, H, D = k.shape
    out = torch.full((B, H, D, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_CHUNK_STATE, B, T, 0, H, D, 0, dtype_la, 0))
    la.lightning_attn_chunk_state(k, v, out, state_in=s0, phi=phi, workspace=ws)
    path = la.lightning_attn_last_path()
    la.lightning_attn_check(ws)
    return to_host(out), path


@pytest.mark.parametrize("T", [1, 100, 128, 129, 1000, 5000])
@pytest.mark.parametrize("H", [8, 2])
def test_chunk_state_tc(T, H, cuda_device):
    """H = 2 spreads each (sequence, head) over many splits, including splits past the end."""
    la = _la()
    B, D = 2, 128
    q, k, v, _ = synth.prefill_inputs(3601 + T + H, B * T, H, D, "bf16", 0.5, False)
    s0 = synth.normal(3601, 9, (B, H, D, D), 0.05, "f32")
    shp = (B, T, H, D)
    got, path = _run(to_dev(k).reshape(shp), to_dev(v).reshape(shp), to_dev(s0), la.LA_BF16)
    assert path == "tcgen05-state"
    _, ref, _ = oracle.prefill(q.reshape(shp), k.reshape(shp), v.reshape(shp), None, state_in=s0,
                               mode=oracle.MODE_RAW)
    assert_close(got, ref, "bf16", "state")


@pytest.mark.parametrize("T", [300, 4096])
def test_chunk_state_exact_integers(T, cuda_device):
    """Identity features, ternary k and v, integer S0: the state is an integer sum, exact in
    fp32 in any order, so it must equal the oracle's bit for bit."""
    la = _la()
    B, H, D = 1, 4, 128
    k = synth.ternary(3611 + T, 1, (T, H, D), 0.3, "bf16")
    v = synth.ternary(3611 + T, 2, (T, H, D), 0.3, "bf16")
    s0 = np.round(synth.normal(3611, 9, (B, H, D, D), 3.0, "f32")).astype(np.float32)
    shp = (B, T, H, D)
    got, _ = _run(to_dev(k).reshape(shp), to_dev(v).reshape(shp), to_dev(s0), la.LA_BF16, phi=1)
    _, ref, _ = oracle.prefill(k.reshape(shp), k.reshape(shp), v.reshape(shp), None, state_in=s0,
                               phi=oracle.PHI_IDENTITY, mode=oracle.MODE_RAW)
    np.testing.assert_array_equal(got.astype(np.float64), ref)


def test_chunk_state_fp32_and_d64_paths(cuda_device):
    la = _la()
    for dtype, D in (("f32", 64), ("bf16", 64)):
        B, T, H = 2, 300, 4
        q, k, v, _ = synth.prefill_inputs(3621 + D, B * T, H, D, dtype, 0.5, False)
        shp = (B, T, H, D)
        got, path = _run(to_dev(k).reshape(shp), to_dev(v).reshape(shp), None,
                         la.LA_F32 if dtype == "f32" else la.LA_BF16)
        assert path == "simt"
        _, ref, _ = oracle.prefill(k.reshape(shp), k.reshape(shp), v.reshape(shp), None, mode=oracle.MODE_RAW)
        assert_close(got, ref, dtype, "state")


def test_chunk_state_matches_the_prefill_state(cuda_device):
    import torch
    la = _la()
    B, T, H, D = 1, 3000, 8, 128
    q, k, v, g = synth.prefill_inputs(3631, T, H, D, "bf16", 0.5, True)
    dq, dk, dv, dg = (to_dev(a)[None] for a in (q, k, v, g))
    out = torch.empty((1, T, H * D), dtype=torch.bfloat16, device="cuda")
    st = torch.empty((1, H, D, D), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL, 1, T, 0, H, D, 256, la.LA_BF16,
                                                           la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_prefill(dq, dk, dv, dg, out, None, st, workspace=ws)
    la.lightning_attn_check(ws)
    got, _ = _run(dk, dv, None, la.LA_BF16)
    ref = to_host(st)
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()   # same features, other summation order
