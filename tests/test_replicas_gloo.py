"""Host logic of the multi-GPU path (independent replicas, no collective on the data path) on CPU: two gloo
ranks line up, take the maximum of their times, draw different problems and split units without overlap."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    from exact_io_aware_76_b200 import replicas

    r, w = replicas.init("gloo", timeout_s=60)
    replicas.barrier()
    m = replicas.max_over_ranks(10.0 * (rank + 1))
    seed = replicas.replica_seed(1003, rank)
    span = replicas.shard(13, rank, world)
    replicas.barrier()
    replicas.shutdown()
    q.put((r, w, m, seed, span))


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get() for _ in range(world))
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[2] == 20.0 for r in res)              # max over ranks
    assert res[0][3] != res[1][3]                     # each replica draws its own problem
    spans = [r[4] for r in res]
    assert spans[0][0] == 0 and spans[0][1] == spans[1][0] and spans[1][1] == 13  # contiguous, complete


@pytest.mark.parametrize("n,world", [(0, 3), (5, 1), (7, 4), (128, 8)])
def test_shard_partitions(n, world):
    from exact_io_aware_76_b200 import replicas

    spans = [replicas.shard(n, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for a, b in zip(spans, spans[1:]):
        assert a[1] == b[0]
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
