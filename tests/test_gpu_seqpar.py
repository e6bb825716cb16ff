"""The sequence sharded along T (seqpar.SeqShard) with its product compute, the CUDA
keep drivers (seqpar.KeepRunner), on one GPU.

Each rank is a process of a gloo group; every rank's kernels run on cuda:0.  The
boundary states cross between ranks as host tensors (KeepRunner(host_states=True)),
so no kernel of one rank waits on another rank's kernels: a rank launches only after
its message has arrived on the host.  The outputs, final state, gradients and the
initial-state gradient gathered from the ranks are compared with the fp64 oracle run
over the whole sequence in one piece (relative L2 per tensor, 2e-2 for bf16 inputs,
1e-4 for fp32 inputs).
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case(B, T, H, d, seed, dtype):
    """Seeded inputs; bf16 cases round q, k, v, dO to bf16 first, so that the oracle and
    the kernels read the same values."""
    import torch
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = r.standard_normal((B, T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, d))
    g = -0.1 * np.log1p(np.exp(r.standard_normal((B, T, H))))
    beta = 1 / (1 + np.exp(-r.standard_normal((B, T, H))))
    dO = r.standard_normal((B, T, H, d))
    S_in = 0.1 * r.standard_normal((B, H, d, d))
    dS_out = 0.1 * r.standard_normal((B, H, d, d))
    out = [q, k, v, g, beta, dO, S_in, dS_out]
    out = [x.astype(np.float32) for x in out]
    if dtype == "bf16":
        for i in (0, 1, 2, 5):
            out[i] = torch.from_numpy(out[i]).to(torch.bfloat16).float().numpy()
    return out


def _worker(rank, world, port, cuts, micro, piece, dtype, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    import torch.distributed as dist
    from chunked_linear_recurrence_chunkwise_b200.seqpar import KeepRunner, SeqShard
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        io = torch.bfloat16 if dtype == "bf16" else torch.float32
        q, k, v, g, beta, dO, S_in, dS_out = _case(3, cuts[-1], 2, 128 if dtype == "bf16" else 64, 7, dtype)
        t0, t1 = cuts[rank], cuts[rank + 1]
        sl = lambda x, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(x[:, t0:t1])).to("cuda", dt)
        st = lambda x: torch.from_numpy(x).cuda()
        shard = SeqShard(KeepRunner(piece=piece, host_states=True))
        o, S_out, ctx = shard.forward(sl(q, io), sl(k, io), sl(v, io), sl(g), sl(beta), S_in=st(S_in),
                                      micro=micro)
        gr = shard.backward(ctx, sl(dO, io), dS_out=st(dS_out))
        torch.cuda.synchronize()
        h = lambda x: None if x is None else x.float().cpu().numpy()
        q_out.put((rank, h(o), h(S_out), {n: h(x) for n, x in gr.items()}))
    finally:
        dist.destroy_process_group()


def rel_l2(x, ref):
    return float(np.linalg.norm(x.astype(np.float64) - ref) / np.linalg.norm(ref))


@pytest.mark.parametrize("cuts,micro,piece,dtype", [
    ((0, 640 + 17), 2, 256, "bf16"),          # one rank: SeqShard around the drivers, no messages
    ((0, 320, 640 + 17), 1, 192, "bf16"),     # two ranks on one GPU, one micro-batch
    ((0, 256, 640 + 17), 3, 128, "bf16"),     # two ranks, three micro-batches in flight
    ((0, 100, 357), 2, 64, "f32"),            # SIMT path, ragged slices
])
def test_sharded_sequence_on_the_gpu_matches_the_oracle(cuts, micro, piece, dtype):
    import oracle
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, micro, piece, dtype, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q_out.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, g, beta, dO, S_in, dS_out = _case(3, cuts[-1], 2, 128 if dtype == "bf16" else 64, 7, dtype)
    o_ref, S_ref = oracle.fwd(q, k, v, g, beta, S_in)
    g_ref = oracle.bwd(q, k, v, g, beta, S_in, dO, dS_out)
    tol = TOL[dtype]
    errs = {"o": rel_l2(np.concatenate([r_[1] for r_ in res], axis=1), o_ref)}
    assert res[-1][2] is not None and all(r_[2] is None for r_ in res[:-1])
    errs["S_out"] = rel_l2(res[-1][2], S_ref)
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        errs[n] = rel_l2(np.concatenate([r_[3][n] for r_ in res], axis=1), g_ref[n])
    assert res[0][3]["dS_in"] is not None and all(r_[3]["dS_in"] is None for r_ in res[1:])
    errs["dS_in"] = rel_l2(res[0][3]["dS_in"], g_ref["dS_in"])
    bad = {k_: e for k_, e in errs.items() if not e <= tol}
    assert not bad, f"rel-L2 above {tol}: {bad} (all {errs})"
