"""GPU parity: libngram.so (through the C ABI) against the CPU oracle, element by element.

Indices and table values must match bit for bit.  Outputs must lie within 1 bf16 ulp
of the oracle's fp32-accumulated result, and within 1 ulp plus the near-zero slack of
its exact fp64 result (see parity_helpers).  Sizes: every token at the sizes the
oracle finishes in seconds (tiny: 512 tokens; mid: all 8192 tokens), sampled tokens at
the full 20M x 2560 size in the same launch configuration the benchmark times, and the
edge cases of the method (boundaries, history, collisions, ragged shapes, in place).
"""
import numpy as np
import pytest
import torch

import ngram_inputs as gen
import oracle
import hashed_gram_embedding_ngram_b200 as ng
from parity_helpers import (N_CPU, TABLES, assert_parity, from_dev_bf16, ng_dtype, oracle_dtype, parity_report,
                            sample_tokens, to_dev_bf16, to_dev_tokens, workload_on_device)

pytestmark = pytest.mark.gpu
W = gen.WORKLOADS


def _hp(vocab, nb=8, nt=8, **kw):
    return ng.ngram_default_hash_params(vocab_size=vocab, n_bigram_heads=nb,
                                        n_trigram_heads=nt, **kw)


def _oracle(w, inp, sel=None, acc=oracle.ACC_F32, want_aux=False, **kw):
    return oracle.forward(inp["tokens"], inp["history"], inp["residual"], inp["gate"],
                          R=w.R, d=w.d, dtype=oracle_dtype(w.dtype),
                          table_seed=gen.TABLE_SEED, sel=sel, acc=acc, n_threads=N_CPU,
                          vocab_size=w.vocab, want_aux=want_aux, **kw)


def _run(w, dev, inp_dev, ctx, out=None):
    return ng.ngram_forward(ctx, inp_dev["tokens"], inp_dev["residual"], inp_dev["gate"],
                            out=out, history=inp_dev["history"])


def _ctx_for(w, dev, max_tokens=None):
    dtype = ng_dtype(w.dtype)
    table, scale = TABLES.get(w.R, w.d, dtype, gen.TABLE_SEED, dev)
    return ng.ngram_init(table, w.R, w.d, dtype, ng.NGRAM_RES_HBM, _hp(w.vocab),
                         max_tokens or w.N, row_scale=scale)


def _dummy_ctx(dev, R, d=8, vocab=0x1FFFFF, nb=8, nt=8, max_tokens=1 << 20):
    """A context whose table is never read (index step only)."""
    buf = torch.zeros(16, dtype=torch.bfloat16, device=dev)
    ctx = ng.ngram_init(buf, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(vocab, nb, nt), max_tokens)
    ctx._keep = buf
    return ctx


# --------------------------------------------------------------------------- table values
def test_table_bitexact_every_row_tiny(cuda_device):
    w = W["tiny"]
    table, _ = TABLES.get(w.R, w.d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    got = from_dev_bf16(table)
    assert np.array_equal(got, oracle.fill_bf16(gen.TABLE_SEED, 0, w.R, w.d))


def test_table_bitexact_int8_and_scale(cuda_device):
    R, d = 3000, 512
    q = torch.empty((R, d), dtype=torch.int8, device=cuda_device)
    s = torch.empty((R,), dtype=torch.float32, device=cuda_device)
    ng.ngram_fill_synthetic(q, R, d, ng.NGRAM_INT8_ROWSCALE, 12345, row_scale=s)
    wq, ws = oracle.fill_int8(12345, 0, R, d)
    assert np.array_equal(q.cpu().numpy(), wq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), ws.view(np.uint32))


# --------------------------------------------------------------------------- indices
@pytest.mark.parametrize("name", ["tiny", "mid", "full_prefill", "full_decode_1",
                                  "full_decode_16", "full_decode_64", "full_decode_256",
                                  "int8_uniform"])
def test_indices_bitexact(cuda_device, name):
    w = W[name]
    inp = gen.make_inputs(w)
    ctx = _dummy_ctx(cuda_device, w.R, vocab=w.vocab, max_tokens=w.N)
    got = ng.ngram_hash_indices(ctx, to_dev_tokens(inp["tokens"], cuda_device),
                                to_dev_tokens(inp["history"], cuda_device))
    want = oracle.indices(inp["tokens"], inp["history"], w.R, vocab_size=w.vocab)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want)


@pytest.mark.parametrize("R", [1, 2, 3, 1 << 16, 1 << 31, 20_000_000, 4_294_967_291,
                               4_294_967_295])
def test_indices_exact_remainder_edge_R(cuda_device, R):
    toks = gen.zipf_tokens(5, 97, 151_936, seed=21)
    hist = gen.zipf_tokens(5, 2, 151_936, seed=22)
    ctx = _dummy_ctx(cuda_device, R, vocab=151_936)
    got = ng.ngram_hash_indices(ctx, to_dev_tokens(toks, cuda_device), to_dev_tokens(hist, cuda_device))
    want = oracle.indices(toks, hist, R, vocab_size=151_936)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want)


def test_largest_vocabulary_uses_every_key_bit(cuda_device):
    """Token ids up to 2^21 - 2 with vocab_size = 2^21 - 1 (the largest the 21-bit packing
    allows): the trigram key fills 63 bits.  Indices (R = 2^32 - 1, and R = 20M in the
    forward), the grouped-order path that hashes every token once (20,000 tokens) and the
    forward itself equal the oracle; ids at the top of the range appear on purpose."""
    V = (1 << 21) - 1
    rng = np.random.default_rng(31)
    toks = rng.integers(0, V, (2, 10_000)).astype(np.int32)
    toks[0, :64] = V - 1 - np.arange(64)            # the largest ids, consecutive
    hist = rng.integers(V - 8, V, (2, 2)).astype(np.int32)
    ctx = _dummy_ctx(cuda_device, 4_294_967_295, vocab=V, max_tokens=toks.size)
    got = ng.ngram_hash_indices(ctx, to_dev_tokens(toks, cuda_device), to_dev_tokens(hist, cuda_device))
    want = oracle.indices(toks, hist, 4_294_967_295, vocab_size=V)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want)
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK
    R, d = 20_000_000, 64
    table, _ = TABLES.get(R, d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    w = gen.Workload("vmax", R, d, "bf16", V, 2, 10_000, history=True)
    fctx = ng.ngram_init(table, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V), w.N)
    res = gen.residual_bf16_bits(w.N, d, 32)
    gate = gen.gate_f32(d, 33)
    out = ng.ngram_forward(fctx, to_dev_tokens(toks, cuda_device), to_dev_bf16(res, cuda_device).view(w.N, d),
                           torch.from_numpy(gate).to(cuda_device), history=to_dev_tokens(hist, cuda_device))
    sel = sample_tokens(w, 512)
    ref = oracle.forward(toks, hist, res, gate, R=R, d=d, table_seed=gen.TABLE_SEED, sel=sel,
                         acc=oracle.ACC_F32, n_threads=N_CPU, vocab_size=V)
    r = assert_parity(from_dev_bf16(out).reshape(w.N, d)[sel], ref)
    assert r["exact"] == r["n"]
    assert ng.ngram_get_device_error(fctx)[0] == ng.NGRAM_OK


@pytest.mark.parametrize("nb,nt", [(1, 0), (0, 1), (3, 5), (16, 0), (0, 16), (7, 9)])
def test_indices_head_counts(cuda_device, nb, nt):
    toks = gen.zipf_tokens(3, 50, 32_000, seed=23)
    ctx = _dummy_ctx(cuda_device, 65_536, vocab=32_000, nb=nb, nt=nt)
    got = ng.ngram_hash_indices(ctx, to_dev_tokens(toks, cuda_device))
    want = oracle.indices(toks, None, 65_536, n_bigram=nb, n_trigram=nt, vocab_size=32_000)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want)


# --------------------------------------------------------------------------- forward
def test_forward_tiny_every_token(cuda_device):
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    r32 = assert_parity(got, _oracle(w, inp))
    want64, _, mag, _ = _oracle(w, inp, acc=oracle.ACC_F64, want_aux=True)
    assert_parity(got, want64, mag)
    assert r32["exact"] == r32["n"]          # same operations in the same order
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


def test_forward_mid_every_token(cuda_device):
    w = W["mid"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    r = assert_parity(got, _oracle(w, inp))
    assert r["exact"] == r["n"]


def test_forward_full_prefill_sampled(cuda_device):
    """Full size (20M x 2560, 32,768 tokens) in the benchmark's launch configuration;
    1,024 sampled tokens (boundaries included) against the oracle."""
    w = W["full_prefill"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx)).reshape(w.N, w.d)
    sel = sample_tokens(w, 1024)
    want, _, mag, idx = _oracle(w, inp, sel=sel, acc=oracle.ACC_F64, want_aux=True)
    assert_parity(got[sel], want, mag)
    r = assert_parity(got[sel], _oracle(w, inp, sel=sel))
    assert r["exact"] == r["n"]              # same operations in the same order
    # the same sampled indices straight from the index step
    gi = ng.ngram_hash_indices(ctx, dv["tokens"]).cpu().numpy().view(np.uint32)
    assert np.array_equal(gi[sel], idx)


@pytest.mark.parametrize("name", ["full_decode_1", "full_decode_16", "full_decode_64",
                                  "full_decode_256"])
def test_forward_full_decode_every_token(cuda_device, name):
    w = W[name]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    r = assert_parity(got, _oracle(w, inp))
    assert r["exact"] == r["n"]


@pytest.mark.parametrize("flags", [0, ng.NGRAM_FLAG_TMA_STAGING])
@pytest.mark.parametrize("d,nb,nt,n_seq,T,hist", [
    (8, 8, 8, 3, 37, False),       # one column vector: 31 idle lanes per strip
    (136, 3, 5, 2, 45, True),      # 17 vectors: ragged strip
    (264, 16, 0, 1, 70, True),     # 33 vectors: a full strip plus one lane
    (520, 0, 16, 5, 9, False),     # 65 vectors
    (2568, 8, 8, 2, 33, True),     # 321 vectors: the pages' width plus a ragged tail
    (256, 1, 0, 4, 16, False),     # single head: an embedding lookup
])
def test_forward_ragged_shapes_and_heads(cuda_device, d, nb, nt, n_seq, T, hist, flags):
    """Both bf16 gathers: register loads (default) and TMA bulk staging (flag)."""
    R, V = 4099, 5000
    w = gen.Workload("ragged", R, d, "bf16", V, n_seq, T, history=hist)
    inp = gen.make_inputs(w, token_seed=31)
    table, _ = TABLES.get(R, d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM,
                        _hp(V, nb, nt, flags=flags), w.N)
    dv = {"tokens": to_dev_tokens(inp["tokens"], cuda_device),
          "history": to_dev_tokens(inp["history"], cuda_device),
          "residual": to_dev_bf16(inp["residual"], cuda_device).view(w.N, d),
          "gate": torch.from_numpy(inp["gate"]).to(cuda_device)}
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    want = _oracle(w, inp, n_bigram=nb, n_trigram=nt)
    r = assert_parity(got, want)
    assert r["exact"] == r["n"]


def test_forward_collisions_R2(cuda_device):
    """R = 2: every token's 16 heads collide on two rows; each head still counts."""
    R, d, V = 2, 64, 100
    w = gen.Workload("r2", R, d, "bf16", V, 2, 40)
    inp = gen.make_inputs(w, token_seed=41)
    table, _ = TABLES.get(R, d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V), w.N)
    dv = {"tokens": to_dev_tokens(inp["tokens"], cuda_device), "history": None,
          "residual": to_dev_bf16(inp["residual"], cuda_device).view(w.N, d),
          "gate": torch.from_numpy(inp["gate"]).to(cuda_device)}
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    r = assert_parity(got, _oracle(w, inp))
    assert r["exact"] == r["n"]


def test_forward_large_batch_small_rows(cuda_device):
    """262,144 tokens (grid-stride loop wraps many times) at d = 256; sampled check."""
    w = gen.Workload("bigN", 65_536, 256, "bf16", 32_000, 64, 4096)
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx)).reshape(w.N, w.d)
    sel = sample_tokens(w, 4096)
    r = assert_parity(got[sel], _oracle(w, inp, sel=sel))
    assert r["exact"] == r["n"]


def test_in_place_equals_out_of_place(cuda_device):
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    ref = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    buf = dv["residual"].clone()
    ng.ngram_forward(ctx, dv["tokens"], buf, dv["gate"], out=buf)
    assert np.array_equal(from_dev_bf16(buf), ref)


@pytest.mark.parametrize("fmt,n_seq,T", [("bf16", 256, 1), ("bf16", 1, 20_000), ("bf16", 3, 300),
                                          ("int8", 64, 1), ("fp8", 2, 500), ("nvfp4", 1, 20_000)])
def test_back_to_back_in_place_calls_keep_stream_order(cuda_device, fmt, n_seq, T):
    """The gathers (and the grouped-order kernels) are launched as programmatic dependents:
    each may be scheduled while the previous kernel of the stream still runs and waits for
    it before touching memory.  Six in-place calls in a row, each reading the residual the
    previous one wrote, with no host synchronisation between them -- eagerly and replayed
    from a CUDA graph -- must equal the same calls with a synchronisation after each."""
    R, d, V = 65_536, 2560, 151_936
    w = gen.Workload("chain", R, d, fmt, V, n_seq, T, history=T == 1)
    dt = ng_dtype(fmt)
    table, scale = TABLES.get(R, d, dt, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, dt, ng.NGRAM_RES_HBM, _hp(V), w.N, row_scale=scale)
    batches = [gen.make_inputs(w, token_seed=700 + i) for i in range(6)]
    toks = [torch.from_numpy(b["tokens"]).to(cuda_device) for b in batches]
    hist = [None if b["history"] is None else torch.from_numpy(b["history"]).to(cuda_device) for b in batches]
    res0 = torch.from_numpy(batches[0]["residual"].view(np.int16)).view(torch.bfloat16).view(w.N, d).to(cuda_device)
    gate = torch.from_numpy(batches[0]["gate"]).to(cuda_device)
    ref = res0.clone()
    for i in range(6):
        ng.ngram_forward(ctx, toks[i], ref, gate, out=ref, history=hist[i])
        torch.cuda.synchronize()
    buf = res0.clone()
    for i in range(6):
        ng.ngram_forward(ctx, toks[i], buf, gate, out=buf, history=hist[i])
    torch.cuda.synchronize()
    assert torch.equal(buf.view(torch.int16), ref.view(torch.int16))
    g = torch.cuda.CUDAGraph()
    gbuf = res0.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                          # warm the capture stream
        ng.ngram_forward(ctx, toks[0], gbuf.clone(), gate, history=hist[0], stream=s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        cs = torch.cuda.current_stream()
        for i in range(6):
            ng.ngram_forward(ctx, toks[i], gbuf, gate, out=gbuf, history=hist[i], stream=cs)
    gbuf.copy_(res0)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(gbuf.view(torch.int16), ref.view(torch.int16))
    del g
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


def test_zero_gate_returns_residual_bitwise(cuda_device):
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    out = ng.ngram_forward(ctx, dv["tokens"], dv["residual"], torch.zeros_like(dv["gate"]))
    assert np.array_equal(from_dev_bf16(out), inp["residual"].reshape(w.N, w.d))


def test_chunked_prefill_and_decode_bitexact(cuda_device):
    """history = the two preceding tokens reproduces the full prefill exactly."""
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    full = from_dev_bf16(_run(w, cuda_device, dv, ctx)).reshape(w.n_seq, w.T, w.d)
    toks = dv["tokens"]
    res = dv["residual"].view(w.n_seq, w.T, w.d)
    c = 50
    a = ng.ngram_forward(ctx, toks[:, :c].contiguous(), res[:, :c].contiguous().view(-1, w.d), dv["gate"])
    b = ng.ngram_forward(ctx, toks[:, c:].contiguous(), res[:, c:].contiguous().view(-1, w.d), dv["gate"],
                         history=toks[:, c - 2:c].contiguous())
    got = np.concatenate([from_dev_bf16(a).reshape(w.n_seq, c, w.d),
                          from_dev_bf16(b).reshape(w.n_seq, w.T - c, w.d)], axis=1)
    assert np.array_equal(got, full)
    t = 77                                           # one decode step per sequence
    step = ng.ngram_forward(ctx, toks[:, t:t + 1].contiguous(), res[:, t].contiguous(),
                            dv["gate"], history=toks[:, t - 2:t].contiguous())
    assert np.array_equal(from_dev_bf16(step).reshape(w.n_seq, w.d), full[:, t])


def test_empty_batch_launches_nothing(cuda_device):
    w = W["tiny"]
    ctx = _ctx_for(w, cuda_device)
    toks = torch.zeros((0, 5), dtype=torch.int32, device=cuda_device)
    res = torch.zeros((0, w.d), dtype=torch.bfloat16, device=cuda_device)
    gate = torch.ones(w.d, dtype=torch.float32, device=cuda_device)
    out = ng.ngram_forward(ctx, toks, res, gate)
    assert out.numel() == 0


def test_argument_errors(cuda_device):
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device, max_tokens=100)
    with pytest.raises(ng.NgramError) as ei:                  # N > max_tokens
        _run(w, cuda_device, dv, ctx)
    assert ei.value.status == ng.NGRAM_EINVAL and "max_tokens" in str(ei.value)
    # every pointer below stays inside its buffer, so even a call that slipped past
    # the host checks would only touch memory it owns
    lib = ng.lib()
    base = dv["residual"].data_ptr()                           # 512 x 256 bf16
    other = torch.empty((10, w.d), dtype=torch.bfloat16, device=cuda_device)
    st = lib.ngram_forward(ctx.handle, dv["tokens"].data_ptr(), None, 1, 10, base + 2,
                           dv["gate"].data_ptr(), other.data_ptr(), None)
    assert st == ng.NGRAM_EINVAL and "aligned" in ng.ngram_last_error()
    st = lib.ngram_forward(ctx.handle, dv["tokens"].data_ptr(), None, 1, 10, base,
                           dv["gate"].data_ptr(), base + 16, None)
    assert st == ng.NGRAM_EINVAL and "overlaps" in ng.ngram_last_error()
    torch.cuda.synchronize()


def test_bad_token_ids_flag_the_device_error_word(cuda_device):
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK
    toks = dv["tokens"].clone()
    toks.view(-1)[300] = w.vocab + 5                          # out of vocabulary
    out = ng.ngram_forward(ctx, toks, dv["residual"], dv["gate"])
    st, info = ng.ngram_get_device_error(ctx, clear=True)
    assert st == ng.NGRAM_EDEVICE and info[0] == 1 and info[2] == w.vocab + 5
    assert info[1] == 300                                     # the position of the bad id
    # the bad id reads as PAD: same result as the oracle with PAD there
    t2 = inp["tokens"].copy()
    t2.reshape(-1)[300] = oracle.DEFAULT_PAD_ID
    inp2 = dict(inp, tokens=t2)
    r = assert_parity(from_dev_bf16(out), _oracle(w, inp2))
    assert r["exact"] == r["n"]
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK   # cleared
    hist = torch.full((w.n_seq, 2), -1, dtype=torch.int32, device=cuda_device)
    ng.ngram_forward(ctx, dv["tokens"], dv["residual"], dv["gate"], history=hist)
    st, info = ng.ngram_get_device_error(ctx, clear=True)
    assert st == ng.NGRAM_EDEVICE and (info[1] & 0x80000000)


# --------------------------------------------------------------------------- int8 rows
@pytest.mark.parametrize("d,nb,nt,n_seq,T,hist", [
    (16, 8, 8, 3, 37, False),      # one 16-column vector per row
    (272, 3, 5, 2, 45, True),      # 17 vectors: ragged strip
    (528, 16, 0, 1, 70, True),     # 33 vectors
    (2560, 8, 8, 2, 60, True),     # the pages' width
    (2576, 0, 16, 3, 11, False),   # 161 vectors: ragged tail
    (272, 3, 4, 2, 45, True),      # 7 heads
])
def test_forward_int8_every_token(cuda_device, d, nb, nt, n_seq, T, hist):
    R, V = 5003, 7000
    w = gen.Workload("int8_ragged", R, d, "int8", V, n_seq, T, history=hist)
    inp = gen.make_inputs(w, token_seed=51)
    table, scale = TABLES.get(R, d, ng.NGRAM_INT8_ROWSCALE, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng.NGRAM_INT8_ROWSCALE, ng.NGRAM_RES_HBM, _hp(V, nb, nt),
                        w.N, row_scale=scale)
    dv = {"tokens": to_dev_tokens(inp["tokens"], cuda_device),
          "history": to_dev_tokens(inp["history"], cuda_device),
          "residual": to_dev_bf16(inp["residual"], cuda_device).view(w.N, d),
          "gate": torch.from_numpy(inp["gate"]).to(cuda_device)}
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    r = assert_parity(got, _oracle(w, inp, n_bigram=nb, n_trigram=nt))
    assert r["exact"] == r["n"]
    want64, _, mag, _ = _oracle(w, inp, acc=oracle.ACC_F64, want_aux=True, n_bigram=nb,
                                n_trigram=nt)
    assert_parity(got, want64, mag)


def test_forward_int8_full_sampled(cuda_device):
    """20M x 2560 int8 + row scales (47.8 GiB), 65,536 uniform tokens; 1,024 sampled."""
    w = W["int8_uniform"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx)).reshape(w.N, w.d)
    sel = sample_tokens(w, 1024)
    r = assert_parity(got[sel], _oracle(w, inp, sel=sel))
    assert r["exact"] == r["n"]
    # the stated bar against the exact definition, independent of the fp32 rounding order
    want64, _, mag, _ = _oracle(w, inp, sel=sel, acc=oracle.ACC_F64, want_aux=True)
    assert_parity(got[sel], want64, mag)
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


def test_tma_staging_matches_register_gather_full_size(cuda_device):
    """The TMA-staged gather on the full table equals the default gather bit for bit."""
    w = W["full_prefill"]
    inp, dv = workload_on_device(w, cuda_device)
    table, _ = TABLES.get(w.R, w.d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    a = ng.ngram_init(table, w.R, w.d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(w.vocab), w.N)
    b = ng.ngram_init(table, w.R, w.d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM,
                      _hp(w.vocab, flags=ng.NGRAM_FLAG_TMA_STAGING), w.N)
    oa = _run(w, cuda_device, dv, a)
    ob = _run(w, cuda_device, dv, b)
    assert torch.equal(oa.view(torch.int16), ob.view(torch.int16))
    assert ng.ngram_get_device_error(b)[0] == ng.NGRAM_OK


# --------------------------------------------------------------------------- host buffers
def _host_inputs(inp, w, pinned=True):
    t = torch.from_numpy(np.ascontiguousarray(inp["tokens"]))
    h = None if inp["history"] is None else torch.from_numpy(np.ascontiguousarray(inp["history"]))
    r = torch.from_numpy(inp["residual"].view(np.int16)).view(torch.bfloat16).view(w.N, w.d)
    if pinned:
        t, r = t.pin_memory(), r.pin_memory()
        h = None if h is None else h.pin_memory()
    return t, h, r


@pytest.mark.parametrize("name", ["tiny", "full_prefill", "full_decode_256", "full_decode_1"])
def test_forward_host_buffers_equal_device_forward(cuda_device, name):
    """Chunked, three-stream pipeline over host buffers: the same bits as the device
    call, including contexts that straddle chunk boundaries of one long sequence."""
    w = W[name]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    ref = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    t, h, r = _host_inputs(inp, w)
    out = ng.ngram_forward_host(ctx, t, r, dv["gate"], history=h)
    torch.cuda.current_stream().synchronize()
    assert np.array_equal(out.view(torch.int16).numpy().view(np.uint16), ref)
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


def test_forward_host_back_to_back_and_pageable(cuda_device):
    """Consecutive calls reuse the double buffers; pageable host memory also works."""
    w = W["mid"]
    table, _ = TABLES.get(w.R, w.d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, w.R, w.d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(w.vocab), w.N)
    outs, refs = [], []
    for seed, pinned in ((11, True), (12, True), (13, False)):
        inp, dv = workload_on_device(w, cuda_device, token_seed=seed)
        refs.append(from_dev_bf16(_run(w, cuda_device, dv, ctx)))
        t, h, r = _host_inputs(inp, w, pinned)
        outs.append(ng.ngram_forward_host(ctx, t, r, dv["gate"], history=h))
    torch.cuda.current_stream().synchronize()
    for o, ref in zip(outs, refs):
        assert np.array_equal(o.view(torch.int16).numpy().view(np.uint16), ref)


def test_forward_host_rejects_staged_modes(cuda_device):
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    table, _ = TABLES.get(w.R, w.d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, w.R, w.d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM,
                        _hp(w.vocab, flags=ng.NGRAM_FLAG_DEDUP), w.N)
    t, h, r = _host_inputs(inp, w)
    with pytest.raises(ng.NgramError) as ei:
        ng.ngram_forward_host(ctx, t, r, dv["gate"])
    assert ei.value.status == ng.NGRAM_EUNSUPPORTED


def test_forward_host_rejects_overlapping_buffers(cuda_device):
    """Output chunks are copied back while other chunks' inputs are still being read, on
    other streams: the host output must not overlap the host residual, in place included."""
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    t, h, r = _host_inputs(inp, w)
    with pytest.raises(ng.NgramError) as ei:                       # in place
        ng.ngram_forward_host(ctx, t, r, dv["gate"], out=r, history=h)
    assert ei.value.status == ng.NGRAM_EINVAL
    big = torch.empty(r.numel() + w.d, dtype=torch.bfloat16).pin_memory()
    res, out = big[:r.numel()].view_as(r), big[w.d:].view_as(r)     # one row apart
    res.copy_(r)
    with pytest.raises(ng.NgramError) as ei:
        ng.ngram_forward_host(ctx, t, res, dv["gate"], out=out, history=h)
    assert ei.value.status == ng.NGRAM_EINVAL


# --------------------------------------------------------------------------- grouped order
@pytest.mark.parametrize("name", ["tiny", "mid", "full_prefill", "full_decode_1",
                                  "full_decode_256", "int8_uniform"])
def test_sort_flag_is_bit_identical(cuda_device, name):
    """Tokens processed grouped by bigram context give exactly the batch-order output;
    the default (grouped from NGRAM_SORT_MIN_TOKENS tokens) agrees with both."""
    w = W[name]
    inp, dv = workload_on_device(w, cuda_device)
    dtype = ng_dtype(w.dtype)
    table, scale = TABLES.get(w.R, w.d, dtype, gen.TABLE_SEED, cuda_device)
    ctxs = [ng.ngram_init(table, w.R, w.d, dtype, ng.NGRAM_RES_HBM, _hp(w.vocab, flags=f), w.N,
                          row_scale=scale)
            for f in (ng.NGRAM_FLAG_BATCH_ORDER, ng.NGRAM_FLAG_SORT, 0)]
    ref = _run(w, cuda_device, dv, ctxs[0])
    for ctx in ctxs[1:]:
        for _ in range(2):                   # scratch reuse across calls
            got = _run(w, cuda_device, dv, ctx)
            assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
        assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


def test_sort_flag_ragged_heads(cuda_device):
    R, d, V = 4099, 136, 300                # small vocabulary: many repeated contexts
    w = gen.Workload("ragged_sort", R, d, "bf16", V, 3, 211, history=True)
    inp = gen.make_inputs(w, token_seed=77)
    table, _ = TABLES.get(R, d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM,
                        _hp(V, 3, 5, flags=ng.NGRAM_FLAG_SORT), w.N)
    dv = {"tokens": to_dev_tokens(inp["tokens"], cuda_device),
          "history": to_dev_tokens(inp["history"], cuda_device),
          "residual": to_dev_bf16(inp["residual"], cuda_device).view(w.N, d),
          "gate": torch.from_numpy(inp["gate"]).to(cuda_device)}
    got = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    r = assert_parity(got, _oracle(w, inp, n_bigram=3, n_trigram=5))
    assert r["exact"] == r["n"]


def test_device_wait_gives_up_and_context_survives(cuda_device):
    """The kernels' bounded wait, on an mbarrier nothing completes (the path a TMA-staged
    gather would take if its copies never landed): it gives up after the limit, sets device
    error code 2, and the context keeps working afterwards."""
    w = W["tiny"]
    inp, dv = workload_on_device(w, cuda_device)
    ctx = _ctx_for(w, cuda_device)
    ref = from_dev_bf16(_run(w, cuda_device, dv, ctx))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    ng.ngram_selftest_wait_timeout(ctx, 100)
    t1.record()
    st, info = ng.ngram_get_device_error(ctx, clear=True)
    assert st == ng.NGRAM_EDEVICE and info[0] == 2
    assert 90.0 <= t0.elapsed_time(t1) < 1000.0            # it waited about the limit, then left
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK   # cleared
    assert np.array_equal(from_dev_bf16(_run(w, cuda_device, dv, ctx)), ref)
