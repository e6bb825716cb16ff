"""Host logic of the multi-GPU bench path, run as two gloo ranks on CPU.

Heads and batch rows are independent, so ranks share no data-path
collective: each runs its own seeded copy of the workload, and the only
exchange is the max over ranks of the measured step time.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from chunked_linear_recurrence_chunkwise_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w_, lr = bench.dist_env()
        ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        ms_max = bench.reduce_max(ms)
        wl = bench.rank_workload(inputs.WORKLOADS[inputs.BENCH_WORKLOAD], rank)
        q.put((rank, r, w_, lr, ms_max, wl.seed,
               bench.job_tokens_per_s(world, wl.B, wl.T, ms_max)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [x[1] for x in res] == [0, 1] and all(x[2] == world for x in res)
    assert all(x[4] == 15.0 for x in res)           # max over ranks
    assert res[0][5] != res[1][5]                    # independent problems per rank
    assert res[0][6] == res[1][6] == pytest.approx(2 * 65536 / 0.015)
