"""The sequence-parallel prefill's host logic across two gloo ranks on CPU.

The kernels are replaced by the fp64 oracle (this checks the ordering of the calls, the
real all-gather over the process group and the prefix arithmetic, not the GPU code):
rank r's chunk output and the last rank's state must equal one oracle prefill of the whole
sequence."""
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
    """The library calls sequence_parallel makes, on the CPU via the oracle.  Each call is
    first bound to the real binding's signature, so a call the real library would reject
    for its arguments fails here too."""
    LA_OUT_RAW, LA_OUT_RMSNORM_GATE, LA_PHI_SILU, LA_OP_PREFILL, LA_BF16 = 0, 2, 0, 0, 1

    @staticmethod
    def _dtype(t):
        return 1

    def __init__(self):
        import oracle
        from long_context_attn_b200 import lightning_attn as real
        self.oracle = oracle
        self.real = real

    def _bind(self, name, *args, **kw):
        import inspect
        inspect.signature(getattr(self.real, name)).bind(*args, **kw)

    def lightning_attn_prefill_varlen(self, q, k, v, g, out, cu_seqlens, max_seqlen, state_in=None, state_out=None,
                                      block_size=256, phi=0, mode=2, eps=1e-6, norm_weight=None, workspace=None,
                                      stream=None):
        import torch
        self._bind("lightning_attn_prefill_varlen", q, k, v, g, out, cu_seqlens, max_seqlen, state_in=state_in,
                   state_out=state_out, block_size=block_size, phi=phi, mode=mode, eps=eps, norm_weight=norm_weight,
                   workspace=workspace, stream=stream)
        cu = cu_seqlens.numpy()
        assert cu.dtype == np.int32 and int(max_seqlen) >= int(np.diff(cu).max())
        assert state_in is None or (state_in.dtype == torch.float32 and state_in.is_contiguous())
        assert state_out is None or (state_out.dtype == torch.float32 and state_out.shape[0] == cu.size - 1)
        _, H, D = q.shape
        o, st, _ = self.oracle.forward_packed(q.numpy(), k.numpy(), v.numpy(), None if g is None else g.numpy(), cu,
                                              H, D, state_in=None if state_in is None else state_in.numpy(),
                                              phi=phi, mode=mode, eps=eps)
        out.copy_(torch.from_numpy(o))
        if state_out is not None:
            state_out.copy_(torch.from_numpy(st))

    def lightning_attn_prefill(self, q, k, v, g, out, state_in, state_out, block_size=256, phi=0, mode=2,
                               eps=1e-6, norm_weight=None, workspace=None, stream=None):
        import torch
        si = None if state_in is None else state_in.numpy()
        o, st, _ = self.oracle.prefill(q.numpy(), k.numpy(), v.numpy(), None if g is None else g.numpy(),
                                       state_in=si, mode=mode)
        out.copy_(torch.from_numpy(o))
        if state_out is not None:
            state_out.copy_(torch.from_numpy(st))

    def lightning_attn_output_transform(self, y, g, out, mode=2, eps=1e-6, norm_weight=None, stream=None):
        import torch
        self._bind("lightning_attn_output_transform", y, g, out, mode=mode, eps=eps, norm_weight=norm_weight,
                   stream=stream)
        H, D = y.shape[-2], y.shape[-1]
        n = y.numel() // (H * D)
        o = self.oracle.transform(y.detach().numpy().reshape(n, H, D), mode, eps=eps,
                                  norm_weight=None if norm_weight is None else norm_weight.numpy(),
                                  g=None if g is None else g.detach().numpy().reshape(n, H * D))
        out.copy_(torch.from_numpy(o).view(out.shape))

    def lightning_attn_output_transform_backward(self, y, g, dout, dy, dg=None, dnorm_weight=None, mode=2, eps=1e-6,
                                                 norm_weight=None, workspace=None, stream=None):
        import torch
        self._bind("lightning_attn_output_transform_backward", y, g, dout, dy, dg=dg, dnorm_weight=dnorm_weight,
                   mode=mode, eps=eps, norm_weight=norm_weight, workspace=workspace, stream=stream)
        H, D = y.shape[-2], y.shape[-1]
        n = y.numel() // (H * D)
        r = lambda t: None if t is None else t.numpy().reshape(n, H * D)
        dyy, dgg, dw = self.oracle.transform_backward(y.numpy().reshape(n, H, D), r(dout), mode, eps=eps,
                                                      norm_weight=None if norm_weight is None else norm_weight.numpy(),
                                                      g=r(g))
        dy.copy_(torch.from_numpy(dyy).view(dy.shape))
        if dg is not None:
            dg.copy_(torch.from_numpy(dgg).view(dg.shape))
        if dnorm_weight is not None:
            dnorm_weight.copy_(torch.from_numpy(dw))

    def lightning_attn_backward(self, q, k, v, g, dout, dq, dk, dv, dg=None, state_in=None, dstate_in=None,
                                block_size=256, phi=0, mode=2, eps=1e-6, norm_weight=None, workspace=None, stream=None,
                                dstate_out=None, y=None, dnorm_weight=None):
        import torch
        self._bind("lightning_attn_backward", q, k, v, g, dout, dq, dk, dv, dg=dg, state_in=state_in,
                   dstate_in=dstate_in, block_size=block_size, phi=phi, mode=mode, eps=eps, norm_weight=norm_weight,
                   workspace=workspace, stream=stream, dstate_out=dstate_out, y=y, dnorm_weight=dnorm_weight)
        assert q.dim() == 4 and dout.shape == (q.shape[0], q.shape[1], q.shape[2] * q.shape[3])
        npy = lambda t: None if t is None else t.numpy()
        ref = self.oracle.backward(q.numpy(), k.numpy(), v.numpy(), npy(g), dout.numpy(), state_in=npy(state_in),
                                   phi=phi, mode=mode, eps=eps, norm_weight=npy(norm_weight),
                                   dstate_out=npy(dstate_out))
        for t, r in zip((dq, dk, dv, dg, dstate_in), ref):
            if t is not None:
                t.copy_(torch.from_numpy(r).view(t.shape))
        if dnorm_weight is not None:
            dnorm_weight.copy_(torch.from_numpy(ref[5]))

    def lightning_attn_backward_varlen(self, q, k, v, g, dout, dq, dk, dv, cu_seqlens, max_seqlen, dg=None,
                                       state_in=None, dstate_in=None, block_size=256, phi=0, mode=2, eps=1e-6,
                                       norm_weight=None, workspace=None, stream=None, dstate_out=None, y=None,
                                       dnorm_weight=None):
        import torch
        self._bind("lightning_attn_backward_varlen", q, k, v, g, dout, dq, dk, dv, cu_seqlens, max_seqlen, dg=dg,
                   state_in=state_in, dstate_in=dstate_in, block_size=block_size, phi=phi, mode=mode, eps=eps,
                   norm_weight=norm_weight, workspace=workspace, stream=stream, dstate_out=dstate_out, y=y,
                   dnorm_weight=dnorm_weight)
        cu = cu_seqlens.numpy()
        assert cu.dtype == np.int32 and int(max_seqlen) >= int(np.diff(cu).max()) and q.dim() == 3
        _, H, D = q.shape
        npy = lambda t: None if t is None else t.numpy()
        ref = self.oracle.backward_packed(q.numpy(), k.numpy(), v.numpy(), npy(g), dout.numpy(), cu, H, D,
                                          state_in=npy(state_in), phi=phi, mode=mode, eps=eps,
                                          norm_weight=npy(norm_weight), dstate_out=npy(dstate_out))
        for t, r in zip((dq, dk, dv, dg, dstate_in), ref):
            if t is not None:
                t.copy_(torch.from_numpy(r).view(t.shape))
        if dnorm_weight is not None:
            dnorm_weight.copy_(torch.from_numpy(ref[5]))

    def lightning_attn_chunk_state(self, k, v, state_out, state_in=None, phi=0, workspace=None, stream=None):
        import torch
        self._bind("lightning_attn_chunk_state", k, v, state_out, state_in=state_in, phi=phi, workspace=workspace,
                   stream=stream)
        assert k.is_contiguous() and v.is_contiguous() and k.dim() == 4
        q = k.numpy()   # the state does not depend on q
        _, st, _ = self.oracle.prefill(q, k.numpy(), v.numpy(), None, state_in=None if state_in is None else
                                       state_in.numpy(), phi=phi, mode=self.LA_OUT_RAW)
        state_out.copy_(torch.from_numpy(st))

    def lightning_attn_state_prefix(self, gathered, rank, out, state0=None, stream=None):
        import torch
        self._bind("lightning_attn_state_prefix", gathered, rank, out, state0=state0, stream=stream)
        assert 0 <= rank < gathered.shape[0] and gathered.is_contiguous() and out.is_contiguous()
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


# A packed batch over five ranks: sequence 2 starts on rank 0, passes over rank 1 (an empty
# slice) and ends exactly on rank 2's upper boundary; sequence 4 spans ranks 3-4; empty
# sequences inside a slice and at the very end of the stream.
VL_LENS = [20, 0, 45, 15, 60, 0, 26, 0]
VL_BOUNDS = [0, 30, 30, 65, 100, 166]


def _varlen_main(rank, world, port, out_dir):
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
        cu = synth.cu_seqlens_of(VL_LENS)
        tot = int(cu[-1])
        q, k, v, g = synth.prefill_inputs(1511, tot, H, D, "f32", 0.5, True)
        s0 = synth.normal(1511, 9, (len(VL_LENS), H, D, D), 0.1, "f32")
        a, b = VL_BOUNDS[rank], VL_BOUNDS[rank + 1]
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        out = torch.zeros((b - a, H * D), dtype=torch.float64)
        plan, st, _ = sp.prefill_varlen_sequence_parallel(t(q[a:b]), t(k[a:b]), t(v[a:b]), t(g[a:b]), out, cu,
                                                       VL_BOUNDS, rank, state0=t(s0), mode=2, workspace=object())
        np.save(os.path.join(out_dir, f"vout{rank}.npy"), out.numpy())
        fin = {int(s): st[i].numpy() for i, s in enumerate(plan.seq) if plan.final[i]}
        np.save(os.path.join(out_dir, f"vfin{rank}.npy"), fin, allow_pickle=True)
    finally:
        dist.destroy_process_group()


def test_varlen_batch_over_five_gloo_ranks_matches_one_packed_prefill(tmp_path):
    """Every token's output and every sequence's final state (from the rank where it ends)
    against one oracle prefill of the whole packed batch."""
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    world = len(VL_BOUNDS) - 1
    mp.start_processes(_varlen_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    cu = synth.cu_seqlens_of(VL_LENS)
    tot = int(cu[-1])
    q, k, v, g = synth.prefill_inputs(1511, tot, H, D, "f32", 0.5, True)
    s0 = synth.normal(1511, 9, (len(VL_LENS), H, D, D), 0.1, "f32")
    ref, ref_st, _ = oracle.forward_packed(q, k, v, g, cu, H, D, state_in=s0)
    got = np.concatenate([np.load(tmp_path / f"vout{r}.npy") for r in range(world)])
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-5 * np.abs(ref).max())
    fins = {}
    for r in range(world):
        part = np.load(tmp_path / f"vfin{r}.npy", allow_pickle=True).item()
        assert not set(part) & set(fins), "a sequence's final state came from two ranks"
        fins.update(part)
    assert sorted(fins) == list(range(len(VL_LENS)))
    for s, st in fins.items():
        np.testing.assert_allclose(st, ref_st[s], rtol=0, atol=1e-5 * np.abs(ref_st).max(), err_msg=f"seq {s}")


def test_varlen_slice_plans_partition_the_batch():
    """Host planning alone, over seeded random batches and cuts: the pieces of all ranks tile
    the stream in order; each sequence ends (final) on exactly one rank, empty ones included;
    a continued first piece names the rank where its sequence starts, which carries it, as
    does every rank in between whose slice is non-empty."""
    sys.path.insert(0, ROOT)
    from long_context_attn_b200.sequence_parallel import varlen_slice_plan
    rng = np.random.default_rng(1521)
    for _ in range(300):
        n = int(rng.integers(1, 8))
        lens = rng.integers(0, 40, size=n) * (rng.random(n) > 0.25)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        tot = int(cu[-1])
        world = int(rng.integers(1, 6))
        bounds = np.concatenate([[0], np.sort(rng.integers(0, tot + 1, size=world - 1)), [tot]])
        plans = [varlen_slice_plan(cu, bounds, r) for r in range(world)]
        pos, finals = 0, []
        for r, p in enumerate(plans):
            assert (p.lo, p.hi) == (bounds[r], bounds[r + 1])
            assert p.seq == list(range(p.seq[0], p.seq[0] + len(p.seq))) if p.seq else True
            assert p.local_cu[0] == 0 and p.local_cu[-1] == p.hi - p.lo and np.all(np.diff(p.local_cu) >= 0)
            pos += p.hi - p.lo
            for i, s in enumerate(p.seq):
                a, e = p.lo + p.local_cu[i], p.lo + p.local_cu[i + 1]
                assert cu[s] <= a <= e <= cu[s + 1]
                assert p.final[i] == (e == cu[s + 1])
                if p.final[i]:
                    finals.append(s)
            if p.first_from is not None:
                s = p.seq[0]
                r0 = p.first_from
                assert r0 < r and bounds[r0] <= cu[s] < bounds[r0 + 1]
                for j in range(r0, r):
                    if bounds[j] < bounds[j + 1]:
                        assert plans[j].carries and plans[j].seq[-1] == s
            if p.carries:
                nxt = next(j for j in range(r + 1, world) if bounds[j] < bounds[j + 1])
                assert plans[nxt].first_from is not None and plans[nxt].seq[0] == p.seq[-1]
        assert pos == tot
        assert sorted(finals) == list(range(n))


# The backward over three ranks (a one-token chunk in the middle), with a final-state
# gradient, a gradient on the state at the end of the middle chunk too, an initial state, a
# trained norm weight and the gate.
BW_CHUNKS = [40, 1, 55]


def _backward_main(rank, world, port, out_dir):
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
        Tt = sum(BW_CHUNKS)
        q, k, v, g = synth.prefill_inputs(1531, Tt, H, D, "f32", 0.5, True)
        dout = synth.normal(1531, 11, (Tt, H * D), 1.0, "f32")
        s0 = synth.normal(1531, 9, (H, D, D), 0.1, "f32")
        dsT = synth.normal(1531, 10, (H, D, D), 0.1, "f32")
        dsM = synth.normal(1531, 14, (H, D, D), 0.1, "f32")
        w = (1.0 + 0.2 * synth.normal(1531, 13, (H * D,), 1.0, "f32")).astype(np.float32)
        a = sum(BW_CHUNKS[:rank])
        b = a + BW_CHUNKS[rank]
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        cq, ck, cv = (t(x[a:b])[None] for x in (q, k, v))
        cg, cd = t(g[a:b])[None], t(dout[a:b])[None]
        out = torch.zeros((1, b - a, H * D), dtype=torch.float64)
        prefix = sp.prefill_sequence_parallel(cq, ck, cv, cg, out, rank, state0=t(s0), mode=2, norm_weight=t(w),
                                              workspace=object())
        dq, dk, dv = (torch.zeros((1, b - a, H, D), dtype=torch.float32) for _ in range(3))
        dg = torch.zeros((1, b - a, H * D), dtype=torch.float32)
        dw = torch.zeros((H * D,), dtype=torch.float32)
        ds0 = torch.zeros((H, D, D), dtype=torch.float32)
        end = {world - 1: dsT, 1: dsM}.get(rank)
        sp.backward_sequence_parallel(cq, ck, cv, cg, cd, dq, dk, dv, rank, prefix,
                                      dstate_end=None if end is None else t(end), dg=dg, dnorm_weight=dw,
                                      dstate_in=ds0, mode=2, norm_weight=t(w), workspace=object())
        np.savez(os.path.join(out_dir, f"bw{rank}.npz"), dq=dq.numpy()[0], dk=dk.numpy()[0], dv=dv.numpy()[0],
                 dg=dg.numpy()[0], dw=dw.numpy(), ds0=ds0.numpy())
    finally:
        dist.destroy_process_group()


def test_backward_over_three_gloo_ranks_matches_one_backward(tmp_path):
    """Each rank's dq, dk, dv, dg, the ranks' dw summed and rank 0's initial-state gradient
    against the oracle: one backward of the whole sequence (with S0, dS_T and a norm weight)
    plus, the backward being linear in its output gradients, one of the tokens up to the
    middle chunk's end with no output gradient and that state's gradient as the final one."""
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    world = len(BW_CHUNKS)
    mp.start_processes(_backward_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    Tt = sum(BW_CHUNKS)
    q, k, v, g = synth.prefill_inputs(1531, Tt, H, D, "f32", 0.5, True)
    dout = synth.normal(1531, 11, (Tt, H * D), 1.0, "f32")
    s0 = synth.normal(1531, 9, (H, D, D), 0.1, "f32")
    dsT = synth.normal(1531, 10, (H, D, D), 0.1, "f32")
    dsM = synth.normal(1531, 14, (H, D, D), 0.1, "f32")
    w = (1.0 + 0.2 * synth.normal(1531, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    ref = list(oracle.backward(q[None], k[None], v[None], g[None], dout[None], state_in=s0[None], norm_weight=w,
                               dstate_out=dsT[None]))
    m = BW_CHUNKS[0] + BW_CHUNKS[1]
    mid = oracle.backward(q[None, :m], k[None, :m], v[None, :m], g[None, :m], np.zeros_like(dout[None, :m]),
                          state_in=s0[None], norm_weight=w, dstate_out=dsM[None])
    for i in range(3):
        ref[i][:, :m] += mid[i]
    ref[4] = ref[4] + mid[4]   # dg and dw get nothing from a state gradient
    parts = [np.load(tmp_path / f"bw{r}.npz") for r in range(world)]
    # states, dy and the partial sums pass through fp32 between the steps: 1e-5 of the largest
    # value covers that, while a missing or misplaced later-chunk sum is O(1)
    for i, name in enumerate(("dq", "dk", "dv", "dg")):
        got = np.concatenate([p[name] for p in parts])
        want = ref[i][0]
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-5 * np.abs(want).max(), err_msg=name)
    np.testing.assert_allclose(sum(p["dw"].astype(np.float64) for p in parts), ref[5], rtol=0,
                               atol=1e-5 * np.abs(ref[5]).max(), err_msg="dw")
    np.testing.assert_allclose(parts[0]["ds0"], ref[4][0], rtol=0, atol=1e-5 * np.abs(ref[4]).max(),
                               err_msg="dS0")



def _varlen_backward_main(rank, world, port, out_dir):
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
        cu = synth.cu_seqlens_of(VL_LENS)
        tot, n = int(cu[-1]), len(VL_LENS)
        q, k, v, g = synth.prefill_inputs(1541, tot, H, D, "f32", 0.5, True)
        dout = synth.normal(1541, 11, (tot, H * D), 1.0, "f32")
        s0 = synth.normal(1541, 9, (n, H, D, D), 0.1, "f32")
        dsT = synth.normal(1541, 10, (n, H, D, D), 0.1, "f32")
        w = (1.0 + 0.2 * synth.normal(1541, 13, (H * D,), 1.0, "f32")).astype(np.float32)
        a, b = VL_BOUNDS[rank], VL_BOUNDS[rank + 1]
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        cq, ck, cv, cg, cd = (t(x[a:b]) for x in (q, k, v, g, dout))
        out = torch.zeros((b - a, H * D), dtype=torch.float32)
        plan, _, st_in = sp.prefill_varlen_sequence_parallel(cq, ck, cv, cg, out, cu, VL_BOUNDS, rank, state0=t(s0),
                                                             mode=2, norm_weight=t(w), workspace=object())
        dq, dk, dv = (torch.zeros((b - a, H, D), dtype=torch.float32) for _ in range(3))
        dg = torch.zeros((b - a, H * D), dtype=torch.float32)
        dw = torch.zeros((H * D,), dtype=torch.float32)
        ds_in = torch.zeros((len(plan.seq), H, D, D), dtype=torch.float32)
        sp.backward_varlen_sequence_parallel(cq, ck, cv, cg, cd, dq, dk, dv, cu, VL_BOUNDS, rank, st_in,
                                             dstate_out=t(dsT), dg=dg, dnorm_weight=dw, dstate_in=ds_in, mode=2,
                                             norm_weight=t(w), workspace=object())
        starts = {int(s): ds_in[i].numpy() for i, s in enumerate(plan.seq) if not (i == 0 and plan.first_from is not None)}
        np.savez(os.path.join(out_dir, f"vbw{rank}.npz"), dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy(), dg=dg.numpy(),
                 dw=dw.numpy())
        np.save(os.path.join(out_dir, f"vbs{rank}.npy"), starts, allow_pickle=True)
    finally:
        dist.destroy_process_group()


def test_varlen_backward_over_five_gloo_ranks_matches_one_packed_backward(tmp_path):
    """The packed batch and cuts of the varlen forward test, backwards: every token's dq, dk,
    dv, dg, the ranks' dw summed and every sequence's initial-state gradient (from the rank
    where the sequence starts) against one oracle backward of the whole batch with initial
    states, final-state gradients and a norm weight."""
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    world = len(VL_BOUNDS) - 1
    mp.start_processes(_varlen_backward_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    cu = synth.cu_seqlens_of(VL_LENS)
    tot, n = int(cu[-1]), len(VL_LENS)
    q, k, v, g = synth.prefill_inputs(1541, tot, H, D, "f32", 0.5, True)
    dout = synth.normal(1541, 11, (tot, H * D), 1.0, "f32")
    s0 = synth.normal(1541, 9, (n, H, D, D), 0.1, "f32")
    dsT = synth.normal(1541, 10, (n, H, D, D), 0.1, "f32")
    w = (1.0 + 0.2 * synth.normal(1541, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    ref = oracle.backward_packed(q, k, v, g, dout, cu, H, D, state_in=s0, norm_weight=w, dstate_out=dsT)
    parts = [np.load(tmp_path / f"vbw{r}.npz") for r in range(world)]
    for i, name in enumerate(("dq", "dk", "dv", "dg")):
        got = np.concatenate([p[name] for p in parts])
        np.testing.assert_allclose(got, ref[i], rtol=0, atol=1e-5 * np.abs(ref[i]).max(), err_msg=name)
    np.testing.assert_allclose(sum(p["dw"].astype(np.float64) for p in parts), ref[5], rtol=0,
                               atol=1e-5 * np.abs(ref[5]).max(), err_msg="dw")
    starts = {}
    for r in range(world):
        part = np.load(tmp_path / f"vbs{r}.npy", allow_pickle=True).item()
        assert not set(part) & set(starts)
        starts.update(part)
    assert sorted(starts) == list(range(n))
    for s, ds in starts.items():
        np.testing.assert_allclose(ds, ref[4][s], rtol=0, atol=1e-5 * np.abs(ref[4]).max(), err_msg=f"dS0 {s}")



def _autograd_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import synth
    from long_context_attn_b200 import autograd as ag
    from long_context_attn_b200 import sequence_parallel as sp
    fake = _OracleBackend()
    fake.lightning_attn_workspace_size = lambda *a: 256
    fake.new_workspace = lambda n, device=None: torch.zeros(n, dtype=torch.uint8)
    for name in ("LA_OP_CHUNK_STATE", "LA_OP_BACKWARD", "LA_OP_OUTPUT_TRANSFORM_BACKWARD"):
        setattr(fake, name, 0)
    sp.la = ag.la = fake
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        Tt = sum(BW_CHUNKS)
        q, k, v, g = synth.prefill_inputs(1531, Tt, H, D, "f32", 0.5, True)
        dout = synth.normal(1531, 11, (Tt, H * D), 1.0, "f32")
        s0 = synth.normal(1531, 9, (H, D, D), 0.1, "f32")
        dsT = synth.normal(1531, 10, (H, D, D), 0.1, "f32")
        dsM = synth.normal(1531, 14, (H, D, D), 0.1, "f32")
        w = (1.0 + 0.2 * synth.normal(1531, 13, (H * D,), 1.0, "f32")).astype(np.float32)
        a = sum(BW_CHUNKS[:rank])
        b = a + BW_CHUNKS[rank]
        leaf = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).requires_grad_(True)
        cq, ck, cv = (leaf(x[a:b][None]) for x in (q, k, v))
        cg, ts0, tw = leaf(g[a:b][None]), leaf(s0), leaf(w)
        out, st_end = ag.lightning_attention_sequence_parallel(cq, ck, cv, cg, state0=ts0, norm_weight=tw, rank=rank)
        loss = (out * torch.from_numpy(dout[a:b][None])).sum()
        end = {world - 1: dsT, 1: dsM}.get(rank)
        if end is not None:
            loss = loss + (st_end * torch.from_numpy(end)).sum()
        loss.backward()
        np.savez(os.path.join(out_dir, f"ag{rank}.npz"), dq=cq.grad.numpy()[0], dk=ck.grad.numpy()[0],
                 dv=cv.grad.numpy()[0], dg=cg.grad.numpy()[0], dw=tw.grad.numpy(), ds0=ts0.grad.numpy())
    finally:
        dist.destroy_process_group()


def test_autograd_over_three_gloo_ranks_matches_one_backward(tmp_path):
    """lightning_attention_sequence_parallel under loss.backward() on three gloo ranks (the
    middle chunk's end state and the last one's in the loss too): the chunks' input gradients
    and the ranks' state0 and norm-weight gradients added up, against the oracle as in the
    test above."""
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    world = len(BW_CHUNKS)
    mp.start_processes(_autograd_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    Tt = sum(BW_CHUNKS)
    q, k, v, g = synth.prefill_inputs(1531, Tt, H, D, "f32", 0.5, True)
    dout = synth.normal(1531, 11, (Tt, H * D), 1.0, "f32")
    s0 = synth.normal(1531, 9, (H, D, D), 0.1, "f32")
    dsT = synth.normal(1531, 10, (H, D, D), 0.1, "f32")
    dsM = synth.normal(1531, 14, (H, D, D), 0.1, "f32")
    w = (1.0 + 0.2 * synth.normal(1531, 13, (H * D,), 1.0, "f32")).astype(np.float32)
    ref = list(oracle.backward(q[None], k[None], v[None], g[None], dout[None], state_in=s0[None], norm_weight=w,
                               dstate_out=dsT[None]))
    m = BW_CHUNKS[0] + BW_CHUNKS[1]
    mid = oracle.backward(q[None, :m], k[None, :m], v[None, :m], g[None, :m], np.zeros_like(dout[None, :m]),
                          state_in=s0[None], norm_weight=w, dstate_out=dsM[None])
    for i in range(3):
        ref[i][:, :m] += mid[i]
    ref[4] = ref[4] + mid[4]
    parts = [np.load(tmp_path / f"ag{r}.npz") for r in range(world)]
    for i, name in enumerate(("dq", "dk", "dv", "dg")):
        got = np.concatenate([p[name] for p in parts])
        np.testing.assert_allclose(got, ref[i][0], rtol=0, atol=1e-5 * np.abs(ref[i]).max(), err_msg=name)
    np.testing.assert_allclose(sum(p["dw"].astype(np.float64) for p in parts), ref[5], rtol=0,
                               atol=1e-5 * np.abs(ref[5]).max(), err_msg="dw")
    np.testing.assert_allclose(sum(p["ds0"].astype(np.float64) for p in parts), ref[4][0], rtol=0,
                               atol=1e-5 * np.abs(ref[4]).max(), err_msg="dS0")
