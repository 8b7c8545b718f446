"""Host logic of the column-sharded table on CPU: the column partition, the exchange
of output-buffer handles between gloo ranks, and the ordering forward_shard puts around
each rank's shard call (the CUDA allocation, IPC and lookup calls are replaced by a
recording fake; the GPU tests run the real ones)."""
import os
import socket
import time

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import hashed_gram_embedding_ngram_b200 as ng
from hashed_gram_embedding_ngram_b200 import shard


@pytest.mark.parametrize("dtype,d_full,world", [(ng.NGRAM_BF16, 2560, 4), (ng.NGRAM_BF16, 2560, 8),
                                                (ng.NGRAM_FP8_E4M3_ROWSCALE, 2560, 2),
                                                (ng.NGRAM_NVFP4, 2560, 4), (ng.NGRAM_INT8_ROWSCALE, 512, 2)])
def test_shard_columns_partition_the_row(dtype, d_full, world):
    parts = [shard.shard_columns(d_full, world, r, dtype) for r in range(world)]
    cols = [c for c0, d in parts for c in range(c0, c0 + d)]
    assert cols == list(range(d_full))
    assert all(d % shard.FORMAT_MULTIPLE[dtype] == 0 and c0 % 8 == 0 for c0, d in parts)


def test_shard_columns_rejects_uneven_splits():
    with pytest.raises(ValueError):
        shard.shard_columns(2560, 3, 0)                       # 853.3 columns
    with pytest.raises(ValueError):
        shard.shard_columns(2560, 32, 0, ng.NGRAM_NVFP4)      # 80 columns: not a multiple of 32
    with pytest.raises(ValueError):
        shard.shard_columns(2560, 2, 2)


class _FakeLib:
    """Records the allocation and IPC calls; rank r's buffer is address 1000 * (r + 1)."""

    def __init__(self, rank):
        self.rank, self.calls = rank, []

    def ngram_device_alloc(self, nbytes):
        self.calls.append(("alloc", nbytes))
        return 1000 * (self.rank + 1)

    def ngram_ipc_get_handle(self, ptr):
        return ("h%d" % ptr).encode().ljust(64, b"\0")

    def ngram_ipc_open(self, handle):
        ptr = int(handle.rstrip(b"\0")[1:])
        self.calls.append(("open", ptr))
        return ptr + 7                                      # the mapping's local address

    def ngram_ipc_close(self, ptr):
        self.calls.append(("close", ptr))

    def ngram_device_free(self, ptr):
        self.calls.append(("free", ptr))

    def ngram_forward_shard(self, ctx, tokens, residual, gate, outs, d_full, col0, history=None):
        t0 = time.time()
        time.sleep(0.4 if self.rank == 1 else 0.0)          # rank 1's lookup is slow
        self.calls.append(("shard", t0, time.time(), list(outs), d_full, col0))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lib = _FakeLib(rank)
        peers = shard.PeerOutputs(max_tokens=16, d_full=64, lib=lib)
        ptrs = list(peers.ptrs)
        peers.close()
        q.put((rank, ptrs, lib.calls))
    finally:
        dist.destroy_process_group()


def test_peer_outputs_exchange_between_three_gloo_ranks():
    world = 3
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
    for rank, ptrs, calls in res:
        # own buffer at its own rank, every other rank's buffer through its IPC mapping
        assert ptrs == [1000 * (p + 1) + (0 if p == rank else 7) for p in range(world)]
        assert calls[0] == ("alloc", 16 * 64 * 2)
        opened = sorted(c[1] for c in calls if c[0] == "open")
        assert opened == [1000 * (p + 1) for p in range(world) if p != rank]
        closed = sorted(c[1] for c in calls if c[0] == "close")
        assert closed == [x + 7 for x in opened]
        assert calls[-1] == ("free", 1000 * (rank + 1))


class _Tokens:
    def __init__(self, n):
        self.n = n

    def numel(self):
        return self.n


def _order_main(rank, world, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lib = _FakeLib(rank)
        peers = shard.PeerOutputs(max_tokens=16, d_full=64, lib=lib)
        col0, _ = shard.shard_columns(64, world, rank)
        steps = []
        for step in range(2):
            time.sleep(0.3 if rank == 0 else 0.0)            # rank 0 arrives late
            t_enter = time.time()
            shard.forward_shard("ctx", peers, _Tokens(16), None, None, col0)
            steps.append((t_enter, time.time()))
        ptrs = list(peers.ptrs)
        peers.close()
        q.put((rank, steps, [c for c in lib.calls if c[0] == "shard"], ptrs, col0))
    finally:
        dist.destroy_process_group()


def test_forward_shard_orders_the_ranks_on_two_gloo_ranks():
    """Every rank's shard call starts only after every rank has entered forward_shard (no
    rank still reads the buffers of the previous step), and forward_shard returns only
    after every rank's shard call has finished (every shard is in).  Each call gets every
    rank's buffer and this rank's first column."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_order_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slack = 0.05                                            # clock reads around a barrier
    for step in range(2):
        enter = max(r[1][step][0] for r in res)
        done = max(r[2][step][2] for r in res)
        for rank, steps, shards, ptrs, col0 in res:
            assert shards[step][1] >= enter - slack, (rank, step)
            assert steps[step][1] >= done - slack, (rank, step)
            assert shards[step][3] == ptrs and shards[step][4] == 64 and shards[step][5] == col0
    assert [r[4] for r in res] == [0, 32]
