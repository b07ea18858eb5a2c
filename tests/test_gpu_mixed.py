"""GPU parity of lightning_attn_mixed_step: one-token sequences decode, longer ones prefill
from their pooled state, on two streams.  The reference is the oracle's packed forward with
each sequence's initial state taken from its pool slot (a one-token prefill is exactly the
decode step's update-then-read), so every output row and every touched pool slot is
compared, and untouched slots must be bit-for-bit unchanged."""
import numpy as np
import pytest

import oracle
import synth
from tests._helpers import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


def _step(la, lens, slots, pool, seed, H, D, C, mode, streams):
    import torch
    tot = int(sum(lens))
    cu = synth.cu_seqlens_of(lens)
    q, k, v, g = synth.prefill_inputs(seed, tot, H, D, "bf16", 0.5, True)
    dq, dk, dv, dg = (to_dev(a) for a in (q, k, v, g))
    out = torch.full((tot, H * D), float("nan"), dtype=torch.bfloat16, device="cuda")
    dcu = torch.from_numpy(cu).cuda()
    dslot = torch.tensor(slots, dtype=torch.int32, device="cuda")
    max_pre = max([L for L in lens if L > 1], default=0)
    ws = la.new_workspace(la.lightning_attn_workspace_size(la.LA_OP_MIXED, len(lens), max_pre, tot, H, D, C,
                                                           la.LA_BF16, mode))
    before = to_host(pool).copy()
    ps, ds = streams
    torch.cuda.synchronize()
    la.lightning_attn_mixed_step(dq, dk, dv, dg, out, dcu, cu.tolist(), pool, dslot, block_size=C, mode=mode,
                                 workspace=ws, prefill_stream=ps, decode_stream=ds)
    assert la.lightning_attn_last_path() == "mixed"
    ps.synchronize()
    ds.synchronize()
    la.lightning_attn_check(ws)
    ref, ref_st, _ = oracle.forward_packed(q, k, v, g, cu, H, D, state_in=before[slots], mode=mode)
    assert_close(to_host(out), ref, "bf16")
    after = to_host(pool)
    assert_close(after[slots], ref_st, "bf16", "pooled states")
    untouched = sorted(set(range(pool.shape[0])) - set(slots))
    np.testing.assert_array_equal(after[untouched], before[untouched])
    # decode-only sequences: the fp32 update is exact to fp32 rounding
    dec = [i for i, L in enumerate(lens) if L == 1]
    if dec:
        err = np.abs(after[[slots[i] for i in dec]] - ref_st[dec]).max() / np.abs(ref_st[dec]).max()
        assert err <= 1e-5, err


@pytest.mark.parametrize("mode", ["raw", "rmsnorm_gate"])
@pytest.mark.parametrize("C", [128, 256])
def test_mixed_step_two_streams(mode, C, cuda_device):
    import torch
    from long_context_attn_b200 import lightning_attn as la
    m = {"raw": la.LA_OUT_RAW, "rmsnorm_gate": la.LA_OUT_RMSNORM_GATE}[mode]
    H, D = 8, 128
    P = 12
    pool = to_dev(synth.normal(1301, 4, (P, H, D, D), 0.05, "f32"))
    streams = (torch.cuda.Stream(), torch.cuda.Stream())
    lens = [1, 300, 1, 0, 513, 1, 1, 64]
    slots = [7, 2, 11, 0, 5, 9, 3, 4]
    _step(la, lens, slots, pool, 1302, H, D, C, m, streams)
    # The next step continues the same sequences with the roles swapped.
    lens2 = [257, 1, 40, 1, 1, 200, 1, 1]
    _step(la, lens2, slots, pool, 1303, H, D, C, m, streams)


def test_mixed_step_decode_only_and_prefill_only(cuda_device):
    import torch
    from long_context_attn_b200 import lightning_attn as la
    H, D = 8, 128
    pool = to_dev(synth.normal(1304, 4, (6, H, D, D), 0.05, "f32"))
    s = torch.cuda.current_stream()
    _step(la, [1, 1, 1], [4, 0, 2], pool, 1305, H, D, 256, la.LA_OUT_RMSNORM_GATE, (s, s))
    _step(la, [129, 700], [1, 5], pool, 1306, H, D, 256, la.LA_OUT_RMSNORM_GATE, (s, s))
