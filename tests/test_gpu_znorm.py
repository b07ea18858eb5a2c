"""GPU parity of the normalised variant (y = phi(q)^T S / (phi(q) . z), "六十四：MiniMax-01"
section 3) against the oracle: prefill (fixed and packed, both tensor-core block sizes, the
fp32 path, initial S and z, raw and gated output) and the decode step.  q and k are shifted
by +1 so that phi(q) . z stays away from zero (with SiLU features the denominator can
otherwise vanish); tolerances as the forward's (bf16 2e-2, fp32 1e-4 of max|ref|)."""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import assert_close, mode_code, to_dev, to_host

pytestmark = pytest.mark.gpu


def _la():
    from long_context_attn_b200 import lightning_attn as la
    return la


def _shift(a, dtype):
    if dtype == "bf16":
        return synth.f32_to_bf16(synth.bf16_to_f32(a) + 1.0)
    return (a + 1.0).astype(np.float32)


def _inputs(seed, n, H, D, dtype):
    q, k, v, g = synth.prefill_inputs(seed, n, H, D, dtype, 0.5, True)
    return _shift(q, dtype), _shift(k, dtype), v, g


@pytest.mark.parametrize("C", [128, 256])
@pytest.mark.parametrize("mode", ["raw", "rmsnorm_gate"])
def test_prefill_znorm_tc(C, mode, cuda_device):
    import torch
    la = _la()
    B, T, H, D = 2, 700, 8, 128
    m = mode_code(mode)
    q, k, v, g = _inputs(3401 + C, B * T, H, D, "bf16")
    s0 = np.abs(synth.normal(3401, 22, (B, H, D, D), 0.05, "f32"))
    z0 = np.abs(synth.normal(3401, 23, (B, H, D), 2.0, "f32"))
    shp, gshp = (B, T, H, D), (B, T, H * D)
    dq, dk, dv = (to_dev(a).reshape(shp) for a in (q, k, v))
    dg = to_dev(g).reshape(gshp)
    out = torch.full(gshp, float("nan"), dtype=torch.bfloat16, device="cuda")
    so = torch.empty((B, H, D, D), dtype=torch.float32, device="cuda")
    zo = torch.empty((B, H, D), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_ZNORM, B, T, 0, H, D, C, la.LA_BF16, m))
    la.lightning_attn_prefill_znorm(dq, dk, dv, dg if m == la.LA_OUT_RMSNORM_GATE else None, out, to_dev(s0),
                                    to_dev(z0), so, zo, block_size=C, mode=m, workspace=ws)
    assert la.lightning_attn_last_path() == "tcgen05"
    la.lightning_attn_check(ws)
    ref, ref_s, ref_z = oracle.prefill_znorm(q.reshape(shp), k.reshape(shp), v.reshape(shp),
                                             g.reshape(gshp) if m == la.LA_OUT_RMSNORM_GATE else None,
                                             state_in=s0, z_in=z0, mode=m)
    assert_close(to_host(out), ref, "bf16")
    assert_close(to_host(so), ref_s, "bf16", "state")
    assert_close(to_host(zo), ref_z, "f32", "z")   # z is an fp32 sum of fp32 features


def test_prefill_znorm_varlen(cuda_device):
    import torch
    la = _la()
    H, D, C = 8, 128, 256
    lens = [300, 0, 257, 1, 31, 600]
    tot, n = sum(lens), len(lens)
    cu = synth.cu_seqlens_of(lens)
    q, k, v, g = _inputs(3411, tot, H, D, "bf16")
    z0 = np.abs(synth.normal(3411, 23, (n, H, D), 2.0, "f32"))
    out = torch.full((tot, H * D), float("nan"), dtype=torch.bfloat16, device="cuda")
    zo = torch.empty((n, H, D), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_ZNORM_VARLEN, n, max(lens), tot, H, D, C,
                                                           la.LA_BF16, la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_prefill_znorm_varlen(to_dev(q), to_dev(k), to_dev(v), to_dev(g), out,
                                           torch.from_numpy(cu).cuda(), max(lens), z_in=to_dev(z0), z_out=zo,
                                           block_size=C, workspace=ws)
    la.lightning_attn_check(ws)
    ref, _, ref_z = oracle.forward_znorm_packed(q, k, v, g, cu, H, D, z_in=z0)
    assert_close(to_host(out), ref, "bf16")
    assert_close(to_host(zo), ref_z, "f32", "z")
    np.testing.assert_array_equal(to_host(zo)[1], z0[1])   # the empty sequence keeps its z


def test_prefill_znorm_fp32_path(cuda_device):
    import torch
    la = _la()
    B, T, H, D, C = 2, 150, 4, 64, 64
    q, k, v, g = _inputs(3421, B * T, H, D, "f32")
    shp, gshp = (B, T, H, D), (B, T, H * D)
    out = torch.empty(gshp, dtype=torch.float32, device="cuda")
    zo = torch.empty((B, H, D), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_ZNORM, B, T, 0, H, D, C, la.LA_F32,
                                                           la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_prefill_znorm(*(to_dev(a).reshape(shp) for a in (q, k, v)), to_dev(g).reshape(gshp), out,
                                    z_out=zo, block_size=C, workspace=ws)
    assert la.lightning_attn_last_path() == "simt"
    la.lightning_attn_check(ws)
    ref, _, ref_z = oracle.prefill_znorm(q.reshape(shp), k.reshape(shp), v.reshape(shp), g.reshape(gshp))
    assert_close(to_host(out), ref, "f32")
    assert_close(to_host(zo), ref_z, "f32", "z")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_znorm(dtype, cuda_device):
    la = _la()
    B, H, D = 5, 8, 128
    S = np.abs(synth.normal(3431, 4, (B, H, D, D), 0.1, "f32"))
    z = np.abs(synth.normal(3431, 5, (B, H, D), 3.0, "f32"))
    q, k, v, g = synth.decode_tokens(3431, 0, B, H, D, dtype, 0.5)
    q, k = _shift(q, dtype), _shift(k, dtype)
    dS, dz = to_dev(S), to_dev(z)
    import torch
    out = torch.empty((B, H * D), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_DECODE, B, 0, 0, H, D, 0, la._dtype(out),
                                                           la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_decode_step_znorm(to_dev(q), to_dev(k), to_dev(v), to_dev(g), out, dS, dz, workspace=ws)
    la.lightning_attn_check(ws)
    ref, ref_S, ref_z = oracle.forward_znorm_packed(q, k, v, g, np.arange(B + 1, dtype=np.int32), H, D,
                                                    state_in=S, z_in=z)
    assert_close(to_host(out), ref, dtype)
    assert_close(to_host(dS), ref_S, dtype, "state")
    assert_close(to_host(dz), ref_z, "f32", "z")


@pytest.mark.slow
def test_znorm_128k_full_size_samples(cuda_device):
    """The normalised variant at the bench's full size (znorm_128k): the outputs of the first
    4096 tokens (causal: they depend on nothing later) against the oracle on that prefix, and
    z_out against the fp64 sum of phi(k) over all 131072 tokens."""
    import torch
    la = _la()
    w = synth.WORKLOADS["znorm_128k"]
    T, H, D, n = w.T, w.H, w.D, 4096
    q, k, v, g = synth.prefill_inputs(w.seed, T, H, D, "bf16", w.qkv_scale, True)
    q, k = synth.shifted(q, w.qk_shift), synth.shifted(k, w.qk_shift)
    out = torch.empty((1, T, H * D), dtype=torch.bfloat16, device="cuda")
    zo = torch.empty((1, H, D), dtype=torch.float32, device="cuda")
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_PREFILL_ZNORM, 1, T, 0, H, D, w.block_size,
                                                           la.LA_BF16, la.LA_OUT_RMSNORM_GATE))
    la.lightning_attn_prefill_znorm(*(to_dev(a).reshape(1, T, H, D) for a in (q, k, v)),
                                    to_dev(g).reshape(1, T, H * D), out, z_out=zo, block_size=w.block_size,
                                    workspace=ws)
    la.lightning_attn_check(ws)
    got = to_host(out[0, :n])
    ref, _, _ = oracle.prefill_znorm(q[None, :n], k[None, :n], v[None, :n], g[None, :n])
    assert_close(got[None], ref, "bf16")
    kf = synth.bf16_to_f32(k).astype(np.float64)
    z_ref = (kf / (1.0 + np.exp(-kf))).sum(axis=0)
    # the scan's SiLU is the fast-intrinsic form (a few ulp) summed in fp32 over 131072 tokens
    assert np.abs(to_host(zo)[0] - z_ref).max() <= 1e-4 * np.abs(z_ref).max()
