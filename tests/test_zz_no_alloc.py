"""ngram_dedup_rows_noalloc: the dedup entry point for callers that cannot call
cudaMalloc (a process whose device memory belongs to another allocator, or a loop that
cannot take the synchronisation an allocation may cause).  It keeps its scratch in a
fixed static device array, so these tests check that its results equal those of
ngram_dedup_rows and of the CPU oracle's dedup on two calls in a row (the second call
must not see the first call's leftovers), that a call takes no device memory, and that
a batch over its fixed limit is refused.

The file is named to be collected last, so that a run stopping at the first failure has
run every other test first; it needs nothing from the other test files.
"""
import ctypes

import numpy as np
import pytest
import torch

import ngram_inputs as gen
import oracle
import hashed_gram_embedding_ngram_b200 as ng

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p
_lib = ng.lib()
_lib.ngram_dedup_rows_noalloc.argtypes = [P, ctypes.c_uint64, P, P, ctypes.c_uint32,
                                          ctypes.c_uint32, P, P, P, P]
_lib.ngram_dedup_rows_noalloc.restype = ctypes.c_int


def _outputs(hp, tokens):
    n_seq, T = tokens.shape
    M = n_seq * T * (hp.n_bigram_heads + hp.n_trigram_heads)
    dev = tokens.device
    return (torch.full((M,), -1, dtype=torch.int32, device=dev),
            torch.full((M,), -1, dtype=torch.int32, device=dev),
            torch.full((1,), -1, dtype=torch.int32, device=dev))


def _noalloc(hp, R, tokens, history, stream, outs=None):
    n_seq, T = tokens.shape
    uniq, inv, count = outs if outs is not None else _outputs(hp, tokens)
    st = _lib.ngram_dedup_rows_noalloc(ctypes.byref(hp), R, P(tokens.data_ptr()),
                                       None if history is None else P(history.data_ptr()),
                                       n_seq, T, P(uniq.data_ptr()), P(inv.data_ptr()),
                                       P(count.data_ptr()), P(stream.cuda_stream))
    assert st == ng.NGRAM_OK, ng.ngram_last_error()
    return uniq, inv, count


def test_noalloc_dedup_equals_dedup_rows_on_two_calls_in_a_row(cuda_device):
    R, V = 20_000_000, 151_936
    hp = ng.ngram_default_hash_params(vocab_size=V)
    buf = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)   # index-only context
    ctx = ng.ngram_init(buf, R, 8, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, hp, 4096)
    stream = torch.cuda.current_stream()
    batches = [   # a large batch, then a smaller one that must not see the first's rows
        (gen.zipf_tokens(4, 1024, V, seed=101), gen.zipf_tokens(4, 2, V, seed=102)),
        (gen.zipf_tokens(3, 50, V, seed=103), None),
    ]
    for toks, hist in batches:
        t = torch.from_numpy(toks).to(cuda_device)
        h = None if hist is None else torch.from_numpy(hist).to(cuda_device)
        u0, v0, c0 = ng.ngram_dedup_rows(ctx, t, h, stream=stream)
        u1, v1, c1 = _noalloc(hp, R, t, h, stream)
        torch.cuda.synchronize()
        U = int(c0.item())
        assert int(c1.item()) == U > 0
        assert torch.equal(u1[:U], u0[:U])          # indices: exact equality
        assert torch.equal(v1, v0)
        assert torch.equal(u1[v1.long()], u0[v0.long()])   # both rebuild the same rows
        # the CPU oracle's dedup (first-appearance order) of the oracle's row ids
        want_u, want_inv = oracle.unique_rows(oracle.indices(toks, hist, R, vocab_size=V))
        assert U == want_u.size
        assert np.array_equal(u1[:U].cpu().numpy().view(np.uint32), want_u)
        assert np.array_equal(v1.cpu().numpy().view(np.uint32), want_inv)
    ctx.close()


def test_noalloc_dedup_takes_no_device_memory(cuda_device):
    """After a first call (which loads the kernels and looks the array up), further
    calls, on another stream too, leave the device's free memory unchanged."""
    R, V = 20_000_000, 151_936
    hp = ng.ngram_default_hash_params(vocab_size=V)
    t = torch.from_numpy(gen.zipf_tokens(4, 1024, V, seed=111)).to(cuda_device)
    side = torch.cuda.Stream()
    _noalloc(hp, R, t, None, torch.cuda.current_stream())
    torch.cuda.synchronize()
    outs = [_outputs(hp, t) for _ in range(2)]           # allocated before the measurement
    free0, _ = torch.cuda.mem_get_info(cuda_device)
    _noalloc(hp, R, t, None, side, outs[0])
    torch.cuda.synchronize()                  # calls that overlap on the GPU would race
    _noalloc(hp, R, t, None, torch.cuda.current_stream(), outs[1])
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(cuda_device)
    assert free1 == free0, (free0, free1)
    assert torch.equal(outs[0][2], outs[1][2]) and torch.equal(outs[0][1], outs[1][1])


def test_noalloc_dedup_refuses_batches_over_its_limit(cuda_device):
    hp = ng.ngram_default_hash_params(vocab_size=1000)
    toks = torch.zeros((1, 4097), dtype=torch.int32, device=cuda_device)   # 4097 x 16 > 65,536
    out = torch.zeros(16, dtype=torch.int32, device=cuda_device)
    st = _lib.ngram_dedup_rows_noalloc(ctypes.byref(hp), 1000, P(toks.data_ptr()), None, 1, 4097,
                                       P(out.data_ptr()), P(out.data_ptr()), P(out.data_ptr()),
                                       None)
    assert st == ng.NGRAM_EINVAL
    assert "65536" in ng.ngram_last_error() or "65,536" in ng.ngram_last_error()
    # n_seq * T * heads = 2^66 wraps to 0 in 64 bits: still refused, before any launch
    st = _lib.ngram_dedup_rows_noalloc(ctypes.byref(hp), 1000, P(toks.data_ptr()), None, 1 << 31,
                                       1 << 31, P(out.data_ptr()), P(out.data_ptr()),
                                       P(out.data_ptr()), None)
    assert st == ng.NGRAM_EINVAL
