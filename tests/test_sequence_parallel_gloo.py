"""The sequence-parallel prefill's host logic across two gloo ranks on CPU.

The kernels are replaced by the fp64 oracle (this checks the ordering of the calls, the
real all-gather over the process group and the prefix arithmetic, not the GPU code):
rank r's chunk output and the last rank's state must equal one oracle prefill of the whole
sequence."""
import json
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
H, D, T = 2, 64, 96
CHUNKS = [40, 56]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _OracleBackend:
    """The three library calls sequence_parallel makes, on the CPU via the oracle."""
    LA_OUT_RAW, LA_OUT_RMSNORM_GATE, LA_PHI_SILU, LA_OP_PREFILL, LA_BF16 = 0, 2, 0, 0, 1

    @staticmethod
    def _dtype(t):
        return 1

    def __init__(self):
        import oracle
        self.oracle = oracle

    def lightning_attn_prefill(self, q, k, v, g, out, state_in, state_out, block_size=256, phi=0, mode=2,
                               eps=1e-6, norm_weight=None, workspace=None, stream=None):
        import torch
        si = None if state_in is None else state_in.numpy()
        o, st, _ = self.oracle.prefill(q.numpy(), k.numpy(), v.numpy(), None if g is None else g.numpy(),
                                       state_in=si, mode=mode)
        out.copy_(torch.from_numpy(o))
        if state_out is not None:
            state_out.copy_(torch.from_numpy(st))

    def lightning_attn_chunk_state(self, k, v, state_out, state_in=None, phi=0, workspace=None, stream=None):
        import torch
        q = k.numpy()   # the state does not depend on q
        _, st, _ = self.oracle.prefill(q, k.numpy(), v.numpy(), None, state_in=None if state_in is None else
                                       state_in.numpy(), phi=phi, mode=self.LA_OUT_RAW)
        state_out.copy_(torch.from_numpy(st))

    def lightning_attn_state_prefix(self, gathered, rank, out, state0=None, stream=None):
        import torch
        acc = np.zeros(out.shape) if state0 is None else state0.numpy().astype(np.float64)
        for r in range(rank):
            acc = acc + gathered[r].numpy()
        out.copy_(torch.from_numpy(acc))


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import synth
    from long_context_attn_b200 import sequence_parallel as sp
    sp.la = _OracleBackend()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, g = synth.prefill_inputs(1501, T, H, D, "f32", 0.5, True)
        s0 = synth.normal(1501, 9, (H, D, D), 0.1, "f32")
        a = sum(CHUNKS[:rank])
        b = a + CHUNKS[rank]
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        out = torch.zeros((1, b - a, H * D), dtype=torch.float64)
        final = torch.zeros((H, D, D), dtype=torch.float64)   # the oracle's state is fp64
        sp.prefill_sequence_parallel(t(q[a:b])[None], t(k[a:b])[None], t(v[a:b])[None], t(g[a:b])[None], out,
                                     rank, state0=t(s0), state_out=final if rank == world - 1 else None,
                                     mode=2, workspace=object())
        np.save(os.path.join(out_dir, f"out{rank}.npy"), out.numpy()[0])
        if rank == world - 1:
            np.save(os.path.join(out_dir, "final.npy"), final.numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_one_prefill(tmp_path):
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    world = len(CHUNKS)
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v, g = synth.prefill_inputs(1501, T, H, D, "f32", 0.5, True)
    s0 = synth.normal(1501, 9, (H, D, D), 0.1, "f32")
    ref, ref_st, _ = oracle.prefill(q[None], k[None], v[None], g[None], state_in=s0[None])
    got = np.concatenate([np.load(tmp_path / f"out{r}.npy") for r in range(world)])
    # the oracle rounds a state it is handed to fp32: 1e-5 of the largest value covers that,
    # while a wrong prefix (a chunk missed, counted twice or taken out of order) is O(1)
    np.testing.assert_allclose(got, ref[0], rtol=0, atol=1e-5 * np.abs(ref).max())
    np.testing.assert_allclose(np.load(tmp_path / "final.npy"), ref_st[0], rtol=0, atol=1e-5 * np.abs(ref_st).max())
