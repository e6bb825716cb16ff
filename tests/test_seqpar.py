"""Host logic of the sequence sharded along T (seqpar.SeqShard), run as gloo ranks on CPU.

Each rank holds a contiguous slice of the tokens of every sequence; the state and
its gradient cross the rank boundaries as point-to-point messages, micro-batch by
micro-batch.  The ranks' compute here is the fp64 oracle (a test-side runner with
the product runner's interface), so the check is exact: outputs and gradients
gathered from the ranks equal the oracle run over the whole sequence in one
process, to 1e-12, for several slicings, micro-batch counts and world sizes.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case(B, T, H, d, seed):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, d))
    k = r.standard_normal((B, T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, d))
    g = -0.1 * np.log1p(np.exp(r.standard_normal((B, T, H))))
    beta = 1 / (1 + np.exp(-r.standard_normal((B, T, H))))
    dO = r.standard_normal((B, T, H, d))
    S_in = 0.1 * r.standard_normal((B, H, d, d))
    dS_out = 0.1 * r.standard_normal((B, H, d, d))
    return q, k, v, g, beta, dO, S_in, dS_out


class OracleRunner:
    """The ranks' compute for the test: the fp64 oracle over the rank's slice, cut
    into pieces of at most `piece` tokens (the product uses the CUDA keep drivers)."""

    def __init__(self, piece):
        self.piece = piece

    def state_buffer(self, rows, H, dk, dv, like):
        import torch
        return torch.empty((rows, H, dk, dv), dtype=torch.float64)

    def _lens(self, T):
        return [min(self.piece, T - t) for t in range(0, T, self.piece)]

    def fwd(self, q, k, v, g, beta, S_in):
        import torch
        import oracle
        lens = self._lens(q.shape[1])
        a = [x.numpy() for x in (q, k, v, g, beta)]
        o, S_out, saved = oracle.fwd_seq(lens, *a, None if S_in is None else S_in.numpy())
        return torch.from_numpy(o), torch.from_numpy(np.ascontiguousarray(S_out)), (a, saved, lens)

    def bwd(self, ctx, dO, dS_out):
        import torch
        import oracle
        a, saved, lens = ctx
        r = oracle.bwd_seq(lens, *a, saved, dO.numpy(), None if dS_out is None else dS_out.numpy())
        return {n: torch.from_numpy(np.ascontiguousarray(r[n])) for n in
                ("dq", "dk", "dv", "dg", "dbeta", "dS_in")}


def _worker(rank, world, port, cuts, micro, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    from chunked_linear_recurrence_chunkwise_b200.seqpar import SeqShard
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, g, beta, dO, S_in, dS_out = (torch.from_numpy(x) for x in _case(4, cuts[-1], 2, 8, 5))
        t0, t1 = cuts[rank], cuts[rank + 1]
        sl = lambda x: x[:, t0:t1].contiguous()
        shard = SeqShard(OracleRunner(piece=16))
        o, S_out, ctx = shard.forward(sl(q), sl(k), sl(v), sl(g), sl(beta), S_in=S_in, micro=micro)
        gr = shard.backward(ctx, sl(dO), dS_out=dS_out)
        q_out.put((rank, o.numpy(), None if S_out is None else S_out.numpy(),
                   {n: (None if x is None else x.numpy()) for n, x in gr.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts,micro", [
    ((0, 96), 2),               # one rank: no messages, the drivers' own result
    ((0, 40, 96), 1),           # two ranks, uneven slices, one micro-batch
    ((0, 40, 96), 2),           # two ranks, two micro-batches in flight
    ((0, 17, 64, 100), 3),      # three ranks, ragged slices, three micro-batches (of 2, 1, 1 rows)
])
def test_sharded_sequence_equals_the_single_process_oracle(cuts, micro):
    import oracle
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, micro, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q_out.get(timeout=240) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, g, beta, dO, S_in, dS_out = _case(4, cuts[-1], 2, 8, 5)
    o_ref, S_ref, saved = oracle.fwd_seq([cuts[-1]], q, k, v, g, beta, S_in)
    g_ref = oracle.bwd_seq([cuts[-1]], q, k, v, g, beta, saved, dO, dS_out)
    o = np.concatenate([r_[1] for r_ in res], axis=1)
    assert np.abs(o - o_ref).max() <= 1e-12 * np.abs(o_ref).max()
    assert res[-1][2] is not None and all(r_[2] is None for r_ in res[:-1])
    assert np.abs(res[-1][2] - S_ref).max() <= 1e-12 * np.abs(S_ref).max()
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        got = np.concatenate([r_[3][n] for r_ in res], axis=1)
        assert np.abs(got - g_ref[n]).max() <= 1e-12 * np.abs(g_ref[n]).max(), n
    assert res[0][3]["dS_in"] is not None and all(r_[3]["dS_in"] is None for r_ in res[1:])
    assert np.abs(res[0][3]["dS_in"] - g_ref["dS_in"]).max() <= 1e-12 * np.abs(g_ref["dS_in"]).max()


def test_micro_rows_split_the_batch_evenly():
    from chunked_linear_recurrence_chunkwise_b200.seqpar import micro_rows
    assert micro_rows(4, 3) == [(0, 2), (2, 3), (3, 4)]
    assert micro_rows(5, 1) == [(0, 5)]
    with pytest.raises(ValueError):
        micro_rows(2, 3)
