"""Column-sharded table over the GPUs of one node (tensor parallel).

The pages' serving stack keeps each rank's shard of the n-gram table on its own GPU at TP4
("Qwen Brought Back N-Grams. All 51 Billion Parameters of Them.", section "Which is why the
offload matters more than the parameter count"; the shard axis is not given).  Here rank r
of P holds columns [col0, col0 + d_full/P) of every row, every rank holds the full-width
residual, and one kernel per rank (ngram_forward_shard) computes its columns of the output
and stores them straight into every rank's output buffer through CUDA IPC peer mappings
over NVLink -- the lookup and the all-gather of its output in one launch.  A one-element
NCCL all-reduce on the same stream then orders the ranks: once it completes on a rank,
every rank's kernel has finished writing.

This module is host plumbing only (buffer allocation, handle exchange, ordering); every
step of the lookup runs in libngram.so.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding as _b

FORMAT_MULTIPLE = {_b.NGRAM_BF16: 8, _b.NGRAM_INT8_ROWSCALE: 16,
                   _b.NGRAM_FP8_E4M3_ROWSCALE: 16, _b.NGRAM_NVFP4: 32}


def shard_columns(d_full: int, world: int, rank: int, dtype: int = _b.NGRAM_BF16) -> tuple[int, int]:
    """(col0, d) of rank `rank`: equal shards whose width meets the format's d rule."""
    m = FORMAT_MULTIPLE[dtype]
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d of %d" % (rank, world))
    if d_full % (world * m) != 0:
        raise ValueError("d_full = %d does not split into %d shards of a multiple of %d columns"
                         % (d_full, world, m))
    d = d_full // world
    return rank * d, d


class _DeviceArray:
    """A device allocation seen through __cuda_array_interface__ (as int16: bf16 bits)."""

    def __init__(self, ptr: int, shape):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": "<i2",
                                         "data": (ptr, False), "version": 3, "strides": None}


class PeerOutputs:
    """One bf16 [max_tokens][d_full] output buffer per rank, each mapped into every rank's
    process.  ptrs[p] is rank p's buffer as this process addresses it (its own allocation
    for p == rank, a CUDA IPC mapping otherwise); `out` is this rank's buffer as a tensor.

    exchange(obj) -> list of every rank's obj (default: dist.all_gather_object over
    `group`); lib: the binding (replaceable for host-side tests)."""

    def __init__(self, max_tokens: int, d_full: int, group=None, device=None, exchange=None,
                 lib=_b):
        self.lib = lib
        self.max_tokens, self.d_full = max_tokens, d_full
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if exchange is None:
            def exchange(obj):
                objs = [None] * self.world
                dist.all_gather_object(objs, obj, group=group)
                return objs
        self.ptr = lib.ngram_device_alloc(max_tokens * d_full * 2)
        self.opened = []
        try:
            handles = exchange(lib.ngram_ipc_get_handle(self.ptr))
            self.ptrs = []
            for p, h in enumerate(handles):
                if p == self.rank:
                    self.ptrs.append(self.ptr)
                else:
                    q = lib.ngram_ipc_open(h)
                    self.opened.append(q)
                    self.ptrs.append(q)
        except Exception:
            self.close()
            raise
        self.out = None
        if device is not None:
            arr = _DeviceArray(self.ptr, (max_tokens, d_full))
            self.out = torch.as_tensor(arr, device=device).view(torch.bfloat16)

    def close(self):
        for q in self.opened:
            self.lib.ngram_ipc_close(q)
        self.opened = []
        if self.ptr:
            self.lib.ngram_device_free(self.ptr)
            self.ptr = 0


def complete(group=None) -> None:
    """Order the ranks after their ngram_forward_shard calls: with NCCL, a one-element
    all-reduce on the current stream (no host synchronisation); otherwise the host waits
    for the stream and meets the other ranks at a barrier."""
    if dist.get_backend(group) == "nccl":
        flag = torch.zeros(1, dtype=torch.int32, device=torch.cuda.current_device())
        dist.all_reduce(flag, group=group)
    else:
        if torch.cuda.is_available():
            torch.cuda.current_stream().synchronize()
        dist.barrier(group=group)


def forward_shard(ctx, peers: PeerOutputs, tokens: torch.Tensor, residual: torch.Tensor,
                  gate: torch.Tensor, col0: int, history: torch.Tensor | None = None,
                  group=None) -> torch.Tensor:
    """The full-width output [N][d_full] on this rank: a barrier (no rank still reads the
    buffers), this rank's shard written into every rank's buffer, a barrier (every shard is
    in).  Returns this rank's buffer, rows 0..N-1."""
    N = tokens.numel()
    if N > peers.max_tokens:
        raise ValueError("N = %d exceeds the buffers' %d tokens" % (N, peers.max_tokens))
    complete(group)
    peers.lib.ngram_forward_shard(ctx, tokens, residual, gate, peers.ptrs, peers.d_full, col0,
                                  history=history)
    complete(group)
    return None if peers.out is None else peers.out[:N]
