"""GPU parity of the tcgen05 prefill (bf16, D = 128, block 128 / 256) against the fp64 oracle.

The first tests isolate each tensor-core product with exact integer data (identity
feature map, entries in {-1, 0, 1}, so every partial sum is an integer that bf16 and
fp32 hold exactly) and must match the oracle bit for bit:
  * inter only:  K = 0  ->  out = Q S0, state_out = S0;
  * intra only:  S0 = 0, one tile  ->  out = (Q K^T (.) M) V, state_out = K^T V;
  * several tiles and blocks  ->  the state hand-off between tiles and blocks.
Then SiLU workloads within the bf16 tolerance (2e-2 of max|o|) over lengths that hit
every tail pad (32 / 64 / 128), both block sizes, all output modes and varlen packing.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import as_f64, assert_close, mode_code, record_margin
from tests.test_gpu_prefill_simt import run_prefill, run_varlen

pytestmark = pytest.mark.gpu

H_SMALL = 4


def _tern(seed, shape, density):
    return synth.ternary(seed, 0, shape, density, "bf16"), \
        synth.ternary(seed, 1, shape, density, "bf16"), \
        synth.ternary(seed, 2, shape, density, "bf16")


def _exact(o, ref):
    got = as_f64(o)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} mismatches, first at {bad[:5].tolist()}: got {got[tuple(bad[0])]} " \
                          f"want {ref[tuple(bad[0])]}"


@pytest.mark.parametrize("C", [128, 256])
def test_tc_inter_only_exact(C, cuda_device):
    T, H, D = 128, H_SMALL, 128
    q, _, v = _tern(11, (T, H, D), 0.3)
    k = np.zeros_like(q)
    s0 = np.round(synth.normal(11, 9, (1, H, D, D), 1.5, "f32")).astype(np.float32)
    o, st, path = run_prefill(q[None], k[None], v[None], None, C, oracle.MODE_RAW, phi=1, state_in=s0,
                              want_state=True, expect_path="tcgen05")
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], None, state_in=s0, phi=oracle.PHI_IDENTITY,
                                    mode=oracle.MODE_RAW)
    np.testing.assert_array_equal(st.astype(np.float64), ref_st)
    _exact(o, ref)


@pytest.mark.parametrize("C", [128, 256])
def test_tc_intra_only_exact(C, cuda_device):
    T, H, D = 128, H_SMALL, 128
    q, k, v = _tern(12, (T, H, D), 0.25)
    o, st, _ = run_prefill(q[None], k[None], v[None], None, C, oracle.MODE_RAW, phi=1, want_state=True,
                           expect_path="tcgen05")
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], None, phi=oracle.PHI_IDENTITY, mode=oracle.MODE_RAW)
    np.testing.assert_array_equal(st.astype(np.float64), ref_st)
    _exact(o, ref)


@pytest.mark.parametrize("C", [128, 256])
@pytest.mark.parametrize("T", [256, 640, 1000])
def test_tc_multi_tile_exact(C, T, cuda_device):
    H, D = H_SMALL, 128
    q, k, v = _tern(13 + T, (T, H, D), 0.06)
    s0 = np.round(synth.normal(13, 9, (1, H, D, D), 1.0, "f32")).astype(np.float32)
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], None, state_in=s0, phi=oracle.PHI_IDENTITY,
                                    mode=oracle.MODE_RAW)
    assert np.abs(ref).max() <= 256 and np.abs(ref_st).max() <= 256  # exact in bf16
    o, st, _ = run_prefill(q[None], k[None], v[None], None, C, oracle.MODE_RAW, phi=1, state_in=s0,
                           want_state=True, expect_path="tcgen05")
    np.testing.assert_array_equal(st.astype(np.float64), ref_st)
    _exact(o, ref)


@pytest.mark.parametrize("C", [128, 256])
@pytest.mark.parametrize("T", [1, 31, 32, 33, 64, 65, 127, 128, 129, 200, 255, 256, 257, 383, 1000])
def test_tc_silu_lengths(C, T, cuda_device):
    H, D = H_SMALL, 128
    q, k, v, g = synth.prefill_inputs(500 + T, T, H, D, "bf16", 0.5, True)
    o, st, _ = run_prefill(q[None], k[None], v[None], g[None], C, oracle.MODE_RMSNORM_GATE, want_state=True,
                           expect_path="tcgen05")
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], g[None])
    assert_close(o, ref, "bf16")
    assert_close(st, ref_st, "bf16", "state")


@pytest.mark.parametrize("mode", ["raw", "rmsnorm", "rmsnorm_gate"])
def test_tc_modes_batch_state_in(mode, cuda_device):
    B, T, H, D = 3, 300, 8, 128
    q, k, v, g = synth.prefill_inputs(601, B * T, H, D, "bf16", 0.5, True)
    q, k, v = (a.reshape(B, T, H, D) for a in (q, k, v))
    g = g.reshape(B, T, H * D)
    s0 = synth.normal(601, 9, (B, H, D, D), 0.05, "f32")
    wn = (synth.normal(601, 8, (H * D,), 0.3, "f32") + 1.0) if mode == "rmsnorm" else None
    o, st, _ = run_prefill(q, k, v, g, 256, mode_code(mode), state_in=s0, want_state=True, w=wn,
                           expect_path="tcgen05")
    ref, ref_st, _ = oracle.prefill(q, k, v, g, state_in=s0, mode=mode_code(mode), norm_weight=wn)
    assert_close(o, ref, "bf16")
    assert_close(st, ref_st, "bf16", "state")


def test_tc_varlen_small(cuda_device):
    H, D = H_SMALL, 128
    lens = [0, 300, 1, 128, 0, 257, 77]
    tot = sum(lens)
    q, k, v, g = synth.prefill_inputs(701, tot, H, D, "bf16", 0.5, True)
    s0 = synth.normal(701, 9, (len(lens), H, D, D), 0.05, "f32")
    o, st, _ = run_varlen(q, k, v, g, lens, 256, oracle.MODE_RMSNORM_GATE, state_in=s0, want_state=True,
                          expect_path="tcgen05")
    ref, ref_st, _ = oracle.forward_packed(q, k, v, g, synth.cu_seqlens_of(lens), H, D, state_in=s0)
    assert_close(o, ref, "bf16")
    assert_close(st, ref_st, "bf16", "state")
    np.testing.assert_array_equal(st[0], s0[0])
    np.testing.assert_array_equal(st[4], s0[4])


def test_tc_deterministic(cuda_device):
    T, H, D = 700, 8, 128
    q, k, v, g = synth.prefill_inputs(801, T, H, D, "bf16", 0.5, True)
    o1, s1, _ = run_prefill(q[None], k[None], v[None], g[None], 256, oracle.MODE_RMSNORM_GATE, want_state=True)
    o2, s2, _ = run_prefill(q[None], k[None], v[None], g[None], 256, oracle.MODE_RMSNORM_GATE, want_state=True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_tc_config_8k(cuda_device):
    """B1 H64 T8192 D128 bf16, block 256, RMSNorm over the head concat * sigmoid(G): full compare."""
    w = synth.WORKLOADS["prefill_8k"]
    q, k, v, g = synth.prefill_inputs(w.seed, w.T, w.H, w.D, "bf16", w.qkv_scale, True)
    o, st, _ = run_prefill(q[None], k[None], v[None], g[None], w.block_size, oracle.MODE_RMSNORM_GATE,
                           want_state=True, expect_path="tcgen05+chunks")
    _, _, stats = oracle.prefill(q[None], k[None], v[None], g[None], store=False, cand_out=o, cand_state=st)
    assert stats["out_nonfinite"] == 0 and stats["state_nonfinite"] == 0
    assert stats["out_max_err"] <= 2e-2 * stats["out_max_ref"], stats
    assert stats["state_max_err"] <= 2e-2 * stats["state_max_ref"], stats
    record_margin("test_tc_config_8k", out=stats["out_max_err"] / stats["out_max_ref"],
                  state=stats["state_max_err"] / stats["state_max_ref"])


@pytest.mark.slow
def test_tc_config_128k_full(cuda_device):
    """B1 H64 T131072 D128 bf16, block 256, gated concat RMSNorm, final state: every output
    element and every state element against the fp64 oracle (streamed, not stored)."""
    w = synth.WORKLOADS["prefill_128k"]
    q, k, v, g = synth.prefill_inputs(w.seed, w.T, w.H, w.D, "bf16", w.qkv_scale, True)
    o, st, _ = run_prefill(q[None], k[None], v[None], g[None], w.block_size, oracle.MODE_RMSNORM_GATE,
                           want_state=True, expect_path="tcgen05+chunks")
    _, _, stats = oracle.prefill(q[None], k[None], v[None], g[None], store=False, cand_out=o, cand_state=st)
    assert stats["out_nonfinite"] == 0 and stats["state_nonfinite"] == 0
    assert stats["out_max_err"] <= 2e-2 * stats["out_max_ref"], stats
    assert stats["state_max_err"] <= 2e-2 * stats["state_max_ref"], stats
    record_margin("test_tc_config_128k_full", out=stats["out_max_err"] / stats["out_max_ref"],
                  state=stats["state_max_err"] / stats["state_max_ref"])


@pytest.mark.slow
def test_tc_config_varlen16_full(cuda_device):
    """16 packed sequences, lengths ~ U{1000..32768}, block 256 with 32/64/128 tail pads,
    gated concat RMSNorm, per-sequence final states: full compare against the oracle."""
    w = synth.WORKLOADS["varlen_16"]
    lens = synth.varlen_lengths(w)
    tot = int(lens.sum())
    q, k, v, g = synth.prefill_inputs(w.seed, tot, w.H, w.D, "bf16", w.qkv_scale, True)
    o, st, _ = run_varlen(q, k, v, g, lens, w.block_size, oracle.MODE_RMSNORM_GATE, want_state=True,
                          expect_path="tcgen05")
    _, _, stats = oracle.forward_packed(q, k, v, g, synth.cu_seqlens_of(lens), w.H, w.D, store=False,
                                        cand_out=o, cand_state=st)
    assert stats["out_nonfinite"] == 0 and stats["state_nonfinite"] == 0
    assert stats["out_max_err"] <= 2e-2 * stats["out_max_ref"], stats
    assert stats["state_max_err"] <= 2e-2 * stats["state_max_ref"], stats
    record_margin("test_tc_config_varlen16_full", out=stats["out_max_err"] / stats["out_max_ref"],
                  state=stats["state_max_err"] / stats["state_max_ref"])


@pytest.mark.parametrize("mode,expect", [("rmsnorm_gate", "tcgen05+norm"), ("rmsnorm", "tcgen05+norm"),
                                         ("raw", "tcgen05")])
def test_tc_more_heads_than_resident_pairs(mode, expect, cuda_device):
    """H = 100: more CTA pairs than fit on the GPU at once.  The raw mode runs the tensor-core
    kernel in waves; the norm modes run it raw and then the norm per token in place."""
    H, D, T, C = 100, 128, 300, 256
    q, k, v, g = synth.prefill_inputs(3801, T, H, D, "bf16", 0.5, True)
    m = mode_code(mode)
    o, st, _ = run_prefill(q[None], k[None], v[None], g[None] if m == oracle.MODE_RMSNORM_GATE else None, C, m,
                           want_state=True, expect_path=expect)
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], g[None] if m == oracle.MODE_RMSNORM_GATE else None,
                                    mode=m)
    assert_close(o, ref, "bf16")
    assert_close(st, ref_st, "bf16", "state")


@pytest.mark.parametrize("B,T,H,mode,with_state", [(1, 8192, 8, "rmsnorm_gate", False), (2, 5000, 8, "raw", True),
                                                   (1, 3000, 4, "rmsnorm", True), (1, 2048, 16, "rmsnorm_gate", True)])
def test_tc_long_sequences_few_heads_split_into_chunks(B, T, H, mode, with_state, cuda_device):
    """Few heads, long sequences: each sequence is cut into chunks that run as parallel
    sequence groups, each starting from the state of the chunks before it (chunk-state
    kernel + ordered prefix).  Output and final state against the oracle."""
    D, C = 128, 256
    m = mode_code(mode)
    q, k, v, g = synth.prefill_inputs(3951 + T + H, B * T, H, D, "bf16", 0.5, True)
    q, k, v = (a.reshape(B, T, H, D) for a in (q, k, v))
    g = g.reshape(B, T, H * D) if m == oracle.MODE_RMSNORM_GATE else None
    s0 = synth.normal(3951, 9, (B, H, D, D), 0.05, "f32") if with_state else None
    o, st, _ = run_prefill(q, k, v, g, C, m, state_in=s0, want_state=True, expect_path="tcgen05+chunks")
    ref, ref_st, _ = oracle.prefill(q, k, v, g, state_in=s0, mode=m)
    assert_close(o, ref, "bf16")
    assert_close(st, ref_st, "bf16", "state")
