"""The multi-rank host logic of bench.py on CPU with two gloo ranks: every rank draws its
own token batch (tokens are sharded, the table is replicated, so no collective touches
the data path), the timing is the max over ranks, and the whole-job value counts every
rank's tokens over the slowest rank's time."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import ngram_inputs as gen
        w = gen.WORKLOADS["mid"]
        ts, hs = bench.rank_seeds(rank, 0)
        toks = gen.tokens_for(w, ts)
        local = [10.0 + rank, 1.0 + 2 * rank, 7.0 - rank]       # elapsed, kernel, e2e (ms)
        agg = bench.max_over_ranks(local, world)
        v = bench.weak_scaling_tokens_per_s(world, w.N, 100, agg[0])
        q.put((rank, toks[0, :64].tolist(), agg, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_tokens_and_take_the_max():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, toks0, agg0, v0), (_, toks1, agg1, v1) = res
    assert toks0 != toks1                                   # each rank its own batch
    assert agg0 == agg1 == [11.0, 3.0, 7.0]                 # element-wise max over ranks
    assert v0 == v1 == pytest.approx(2 * 8192 * 100 / 0.011)
