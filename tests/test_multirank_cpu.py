"""The bench's N > 1 host logic on CPU: two gloo ranks, one replica each; the
step time is the max over ranks and the token count the sum over ranks. No
collective is on the data path (replicas), only the timing reductions."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    import torch.distributed as dist
    r, ws = bench.dist_setup(world)
    try:
        bench.barrier(ws)
        mx = bench.max_over_ranks(10.0 + r, ws)          # rank-dependent "step time"
        tot = bench.sum_over_ranks(8192.0, ws)           # tokens of each replica
        q.put((r, ws, mx, tot))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_replicas_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    for r, ws, mx, tot in res:
        assert ws == 2
        assert mx == 11.0          # the slowest rank sets the time
        assert tot == 2 * 8192.0   # whole-job work
