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


def _worker_one_fails(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port), NSA_PG_TIMEOUT_S="10")
    import time
    import bench
    r, ws = bench.dist_setup(world)
    bench.barrier(ws)
    if r == 1:
        os._exit(3)          # this rank dies between steps, with no collective in flight
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, ws)
        q.put((r, "no error", time.time() - t0))
    except Exception as e:   # the surviving rank learns of it at its next collective
        q.put((r, type(e).__name__, time.time() - t0))
    os._exit(0)


@pytest.mark.timeout(120)
def test_rank_failure_ends_the_next_collective_gloo():
    """Failure detection on the host: when one replica dies between steps, the
    other's next timing reduction ends with an error within the process-group
    limit instead of waiting for good."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_one_fails, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    r, what, dt = q.get(timeout=90)
    for p in procs:
        p.join(timeout=30)
    assert r == 0
    assert what != "no error"
    assert dt < 30.0
    assert procs[1].exitcode == 3 and procs[0].exitcode == 0
