"""The N>1 bench path on CPU: gloo ranks, max-over-ranks time, summed work, per-rank batches.

Decode shards by sequence with no exchange, so the multi-GPU logic is only
the host-side aggregation; two gloo ranks exercise it without a GPU.
"""
import os
import socket

import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads as W
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        t = bench._max_over_ranks(1.0 + rank, world)
        s = bench._sum_over_ranks(10.0 * (rank + 1), world)
        bench._barrier(world)
        # each rank builds its own batch (weak scaling): different seeds, same shape
        case = W.make_case(2, seed=1000 + 2 + 7919 * rank, batch=3, max_len=300, num_blocks=64)
        q.put((rank, t, s, case.seq_lens.tolist(), case.q.shape))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [2.0, 2.0]        # max over ranks
    assert [r[2] for r in res] == [30.0, 30.0]      # sum over ranks
    assert res[0][3] != res[1][3]                   # distinct per-rank batches
    assert res[0][4] == res[1][4]                   # same shape


def test_single_rank_helpers_are_identity():
    import bench
    assert bench._max_over_ranks(3.5, 1) == 3.5
    assert bench._sum_over_ranks(2.0, 1) == 2.0
    bench._barrier(1)
