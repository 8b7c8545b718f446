"""GPU tests of the column-sharded table (one GPU).

- The shard fill equals the oracle's table restricted to the shard's columns, bit for bit.
- P shards, each its own context over its [R][d_full/P] table, calling
  ngram_forward_shard into one or two full-width buffers, give ngram_forward over the
  whole table bit for bit (every format, per-token gate, grouped order), and the
  assembled output equals the CPU oracle on sampled tokens (bit for bit against its fp32
  mode, within the stated bar of its exact mode).
- Two processes on this GPU, each holding one shard, write into each other's output
  buffer through CUDA IPC (ngram_ipc_*) and end with the full output, equal to the
  unsharded lookup and to the CPU oracle on sampled tokens.  The two processes'
  kernels never wait on each other (a host barrier orders them), so sharing one GPU is
  safe; the same code runs one process per GPU over NVLink.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import ngram_inputs as gen
import oracle
import hashed_gram_embedding_ngram_b200 as ng
from hashed_gram_embedding_ngram_b200 import shard
from parity_helpers import (N_CPU, TABLES, assert_parity, from_dev_bf16, ng_dtype, oracle_dtype,
                            sample_tokens, to_dev_bf16, to_dev_tokens)

pytestmark = pytest.mark.gpu
FMTS = ["bf16", "int8", "fp8", "nvfp4"]


def _hp(vocab, **kw):
    return ng.ngram_default_hash_params(vocab_size=vocab, **kw)


def _shard_table(R, d_full, col0, d, dt, dev, seed=gen.TABLE_SEED):
    table = torch.empty((R, ng.ngram_row_bytes(dt, d)), dtype=torch.uint8, device=dev)
    scale = None
    if dt != ng.NGRAM_BF16:
        scale = torch.empty((1 if dt == ng.NGRAM_NVFP4 else R,), dtype=torch.float32, device=dev)
    ng.ngram_fill_synthetic_cols(table, R, d, col0, dt, seed, row_scale=scale)
    return table, scale


@pytest.mark.parametrize("fmt", FMTS)
def test_shard_fill_is_the_oracle_table_restricted(cuda_device, fmt):
    R, d_full, P = 301, 512, 4
    dt = ng_dtype(fmt)
    for r in range(P):
        col0, d = shard.shard_columns(d_full, P, r, dt)
        table, scale = _shard_table(R, d_full, col0, d, dt, cuda_device, seed=99)
        got = table.cpu().numpy()
        if fmt == "bf16":
            want = oracle.fill_bf16(99, 0, R, d_full).reshape(R, d_full)[:, col0:col0 + d]
            assert np.array_equal(got.view(np.uint16).reshape(R, d), want)
        elif fmt in ("int8", "fp8"):
            q, s = (oracle.fill_int8 if fmt == "int8" else oracle.fill_fp8)(99, 0, R, d_full)
            assert np.array_equal(got.reshape(R, d), q.reshape(R, d_full)[:, col0:col0 + d].view(np.uint8))
            assert np.array_equal(scale.cpu().numpy().view(np.uint32), s.view(np.uint32))
        else:
            full = oracle.fill_fp4(99, 0, R, d_full)
            want = np.zeros((R, ng.ngram_row_bytes(dt, d)), dtype=np.uint8)
            want[:, :d // 2] = full[:, col0 // 2:(col0 + d) // 2]
            want[:, d // 2:d // 2 + d // 16] = full[:, d_full // 2 + col0 // 16:d_full // 2 + (col0 + d) // 16]
            assert np.array_equal(got, want)
            assert scale.item() == oracle.FP4_GLOBAL_SCALE


CASES = [  # fmt, P, n_seq, T, hist, token_gate, n_outs
    ("bf16", 4, 3, 50, True, False, 1),
    ("bf16", 2, 1, 16_384, False, False, 2),      # grouped order
    ("int8", 4, 2, 70, True, False, 2),
    ("fp8", 2, 2, 70, True, True, 1),
    ("nvfp4", 4, 2, 70, True, False, 2),
    ("nvfp4", 2, 2, 70, False, True, 2),
]


@pytest.mark.parametrize("case", CASES)
def test_virtual_shards_equal_the_full_lookup(cuda_device, case):
    fmt, P, n_seq, T, hist, tg, n_outs = case
    R, d_full, V = 65_536, 2560, 151_936
    dt = ng_dtype(fmt)
    w = gen.Workload("shard", R, d_full, fmt, V, n_seq, T, history=hist)
    inp = gen.make_inputs(w, token_seed=81)
    N = w.N
    flags = ng.NGRAM_FLAG_TOKEN_GATE if tg else 0
    tok = to_dev_tokens(inp["tokens"], cuda_device)
    hst = to_dev_tokens(inp["history"], cuda_device)
    res = to_dev_bf16(inp["residual"], cuda_device).view(N, d_full)
    if tg:
        g = np.random.default_rng(5).normal(0.5, 0.25, (N, d_full)).astype(np.float32)
        gate = torch.from_numpy(g).to(cuda_device).to(torch.bfloat16)
    else:
        gate = torch.from_numpy(inp["gate"]).to(cuda_device)
    full_t, full_s = TABLES.get(R, d_full, dt, gen.TABLE_SEED, cuda_device)
    full = ng.ngram_init(full_t, R, d_full, dt, ng.NGRAM_RES_HBM, _hp(V, flags=flags), N, row_scale=full_s)
    want = from_dev_bf16(ng.ngram_forward(full, tok, res, gate, history=hst))
    outs = [torch.full((N, d_full), float("nan"), dtype=torch.bfloat16, device=cuda_device)
            for _ in range(n_outs)]
    keep = []
    for r in range(P):
        col0, d = shard.shard_columns(d_full, P, r, dt)
        t, s = _shard_table(R, d_full, col0, d, dt, cuda_device)
        ctx = ng.ngram_init(t, R, d, dt, ng.NGRAM_RES_HBM, _hp(V, flags=flags), N, row_scale=s)
        ng.ngram_forward_shard(ctx, tok, res, gate, outs, d_full, col0, history=hst)
        keep.append((ctx, t, s))
    torch.cuda.synchronize()
    for o in outs:
        assert np.array_equal(from_dev_bf16(o), want)
    # the assembled full-width output against the CPU oracle (sampled tokens)
    sel = sample_tokens(w, 256)
    kw = dict(R=R, d=d_full, dtype=oracle_dtype(fmt), table_seed=gen.TABLE_SEED, sel=sel,
              n_threads=N_CPU, vocab_size=V)
    gt = from_dev_bf16(gate).reshape(N, d_full) if tg else None
    g = None if tg else inp["gate"]
    got = from_dev_bf16(outs[-1]).reshape(N, d_full)[sel]
    r = assert_parity(got, oracle.forward(inp["tokens"], inp["history"], inp["residual"], g,
                                          gate_tok=gt, acc=oracle.ACC_F32, **kw))
    assert r["exact"] == r["n"]
    want64, _, mag, _ = oracle.forward(inp["tokens"], inp["history"], inp["residual"], g,
                                       gate_tok=gt, acc=oracle.ACC_F64, want_aux=True, **kw)
    assert_parity(got, want64, mag)


def test_shard_arguments(cuda_device):
    R, d_full, V = 1000, 256, 500
    t, s = _shard_table(R, d_full, 128, 128, ng.NGRAM_BF16, cuda_device)
    ctx = ng.ngram_init(t, R, 128, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V), 64)
    tok = torch.zeros((1, 4), dtype=torch.int32, device=cuda_device)
    res = torch.zeros((4, d_full), dtype=torch.bfloat16, device=cuda_device)
    gate = torch.zeros(d_full, device=cuda_device)
    out = torch.zeros_like(res)
    for col0 in (136, 4):                                # beyond d_full; not a multiple of 8
        with pytest.raises(ng.NgramError):
            ng.ngram_forward_shard(ctx, tok, res, gate, [out], d_full, col0)
    with pytest.raises(ValueError):
        ng.ngram_forward_shard(ctx, tok, res, gate, [out] * 9, d_full, 128)
    ng.ngram_forward_shard(ctx, tok, res, gate, [out], d_full, 128)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[:, :128]) == 0        # columns outside the shard untouched


# --------------------------------------------------------------------------- two processes, IPC
def _free_port():
    so = socket.socket()
    so.bind(("127.0.0.1", 0))
    port = so.getsockname()[1]
    so.close()
    return port


def _ipc_rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    peers = None
    try:
        dev = torch.device("cuda:0")
        torch.cuda.set_device(dev)
        R, d_full, V = 65_536, 2560, 151_936
        w = gen.Workload("ipc", R, d_full, "bf16", V, 2, 300, history=True)
        inp = gen.make_inputs(w, token_seed=82)
        N = w.N
        tok = to_dev_tokens(inp["tokens"], dev)
        hst = to_dev_tokens(inp["history"], dev)
        res = to_dev_bf16(inp["residual"], dev).view(N, d_full)
        gate = torch.from_numpy(inp["gate"]).to(dev)
        col0, d = shard.shard_columns(d_full, world, rank)
        t, _ = _shard_table(R, d_full, col0, d, ng.NGRAM_BF16, dev)
        ctx = ng.ngram_init(t, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V), N)
        peers = shard.PeerOutputs(N, d_full, device=dev)
        peers.out.fill_(float("nan"))
        torch.cuda.synchronize()
        got = from_dev_bf16(shard.forward_shard(ctx, peers, tok, res, gate, col0, history=hst))
        full_t = torch.empty((R, 2 * d_full), dtype=torch.uint8, device=dev)
        ng.ngram_fill_synthetic(full_t, R, d_full, ng.NGRAM_BF16, gen.TABLE_SEED)
        full = ng.ngram_init(full_t, R, d_full, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V), N)
        want = from_dev_bf16(ng.ngram_forward(full, tok, res, gate, history=hst))
        # and the assembled output against the CPU oracle on sampled tokens
        sel = sample_tokens(w, 128)
        ref = oracle.forward(inp["tokens"], inp["history"], inp["residual"], inp["gate"], R=R,
                             d=d_full, table_seed=gen.TABLE_SEED, sel=sel, acc=oracle.ACC_F32,
                             n_threads=4, vocab_size=V)
        same_oracle = bool(np.array_equal(got.reshape(N, d_full)[sel], ref))
        q.put((rank, bool(np.array_equal(got, want)) and same_oracle, None))
        dist.barrier()                                   # nobody unmaps while a peer still writes
    except Exception as e:                               # report, never hang the other rank
        q.put((rank, False, repr(e)))
    finally:
        if peers is not None:
            peers.close()
        dist.destroy_process_group()


def test_two_processes_share_their_shards_through_ipc(cuda_device):
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
    assert all(ok for _, ok, _ in res), res
    assert all(p.exitcode == 0 for p in procs)
