"""GPU parity of the backward pass and the per-token gate, through the C ABI, against the
CPU oracle.

Table gradient: the distinct-row list, its length and every gradient row must equal the
oracle's fp32 mode bit for bit (both sum each row's occurrences in ascending order), and
lie within the sequential-sum bound of its fp64 mode.  Gate gradient: per-token values bit
for bit (fp32(dy * e), e the forward's head sum); the shared-gate sum within one fp32 ulp
plus the fp64 rounding slack of the oracle's (both sum exact products in fp64, in
different orders).  Forward with a per-token gate: bit for bit.  Every result must repeat
bit for bit from run to run.
"""
import numpy as np
import pytest
import torch

import ngram_inputs as gen
import oracle
import hashed_gram_embedding_ngram_b200 as ng
from parity_helpers import (N_CPU, TABLES, assert_parity, from_dev_bf16, ng_dtype, oracle_dtype,
                            sample_tokens, to_dev_bf16, to_dev_tokens, workload_on_device)

pytestmark = pytest.mark.gpu
W = gen.WORKLOADS
FMTS = ["bf16", "int8", "fp8", "nvfp4"]


def _hp(vocab, nb=8, nt=8, **kw):
    return ng.ngram_default_hash_params(vocab_size=vocab, n_bigram_heads=nb,
                                        n_trigram_heads=nt, **kw)


def _bf16_bits(x):
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _dy(N, d, seed):
    """Upstream gradient dL/dout: bf16, normal(0, 1) (seeded, from ngram_inputs' stream)."""
    rng = np.random.default_rng(1000 + seed)
    return _bf16_bits(rng.normal(0.0, 1.0, (N, d)))


def _gate_tok(N, d, seed):
    rng = np.random.default_rng(2000 + seed)
    return _bf16_bits(rng.normal(0.5, 0.25, (N, d)))


def _f32_ulp(v):
    v = np.abs(np.asarray(v, dtype=np.float64)).astype(np.float32)
    return np.spacing(v).astype(np.float64)


def _dummy_ctx(dev, R, d, vocab, nb=8, nt=8, max_tokens=1 << 16, flags=0):
    """A context whose table is never read (the table gradient only needs the indices)."""
    buf = torch.zeros(16, dtype=torch.bfloat16, device=dev)
    ctx = ng.ngram_init(buf, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(vocab, nb, nt, flags=flags),
                        max_tokens)
    ctx._keep = buf
    return ctx


# --------------------------------------------------------------------------- table gradient
ROW_CASES = [  # R, d, nb, nt, n_seq, T, hist, token_gate
    (97, 8, 8, 8, 3, 41, False, False),        # many repeats and collisions
    (97, 8, 8, 8, 3, 41, False, True),
    (5003, 264, 3, 5, 2, 77, True, False),     # 33 vectors: ragged strip
    (5003, 264, 3, 5, 2, 77, True, True),
    (1, 16, 8, 8, 2, 9, False, False),         # one row: every occurrence
    (20_000_000, 2560, 8, 8, 2, 300, True, False),
    (65_536, 2560, 16, 0, 4, 257, False, True),
]


@pytest.mark.parametrize("case", ROW_CASES)
def test_backward_rows_every_row(cuda_device, case):
    R, d, nb, nt, n_seq, T, hist, tg = case
    V = 7000
    w = gen.Workload("bw", R, d, "bf16", V, n_seq, T, history=hist)
    inp = gen.make_inputs(w, token_seed=71)
    N = w.N
    dy = _dy(N, d, 1)
    gt = _gate_tok(N, d, 2) if tg else None
    ctx = _dummy_ctx(cuda_device, R, d, V, nb, nt, max_tokens=N,
                     flags=ng.NGRAM_FLAG_TOKEN_GATE if tg else 0)
    tok = to_dev_tokens(inp["tokens"], cuda_device)
    hst = to_dev_tokens(inp["history"], cuda_device)
    dy_d = to_dev_bf16(dy, cuda_device).view(N, d)
    gate_d = to_dev_bf16(gt, cuda_device).view(N, d) if tg else torch.from_numpy(inp["gate"]).to(cuda_device)
    uniq, count, grad = ng.ngram_backward_rows(ctx, tok, dy_d, gate_d, history=hst)
    U = int(count.item())
    kw = dict(R=R, d=d, gate_tok=gt, n_bigram=nb, n_trigram=nt, vocab_size=V, n_threads=N_CPU)
    wu, wg = oracle.backward_rows(inp["tokens"], inp["history"], dy, inp["gate"], acc=oracle.ACC_F32, **kw)
    assert U == wu.size
    assert np.array_equal(uniq[:U].cpu().numpy().view(np.uint32), wu)
    got = grad[:U].cpu().numpy()
    assert np.array_equal(got.view(np.uint32), wg.astype(np.float32).view(np.uint32))
    # within the sequential-sum bound of the exact gradient
    _, g64, mag = oracle.backward_rows(inp["tokens"], inp["history"], dy, inp["gate"],
                                       acc=oracle.ACC_F64, want_mag=True, **kw)
    idx = oracle.indices(inp["tokens"], inp["history"], R=R, n_bigram=nb, n_trigram=nt,
                         vocab_size=V).reshape(-1)
    pos = {int(r): k for k, r in enumerate(wu)}
    n_terms = np.bincount([pos[int(r)] for r in idx], minlength=U)[:, None]
    assert np.all(np.abs(got - g64) <= (n_terms + 1) * 2.0 ** -24 * mag + _f32_ulp(g64))
    # the same bits again
    u2, c2, g2 = ng.ngram_backward_rows(ctx, tok, dy_d, gate_d, history=hst)
    assert torch.equal(g2[:U], grad[:U]) and torch.equal(u2[:U], uniq[:U])


def test_backward_rows_full_prefill_sampled(cuda_device):
    """The full 32,768-token Zipf prefill over 20M rows; 256 distinct rows checked (the 32
    first-seen, which hold the most frequent contexts, and a seeded sample)."""
    w = W["full_prefill"]
    inp = gen.make_inputs(w)
    N, d = w.N, w.d
    dy = _dy(N, d, 3)
    ctx = _dummy_ctx(cuda_device, w.R, d, w.vocab, max_tokens=N)
    tok = to_dev_tokens(inp["tokens"], cuda_device)
    dy_d = to_dev_bf16(dy, cuda_device).view(N, d)
    gate_d = torch.from_numpy(inp["gate"]).to(cuda_device)
    uniq, count, grad = ng.ngram_backward_rows(ctx, tok, dy_d, gate_d)
    U = int(count.item())
    rng = np.random.default_rng(4)
    sel = np.unique(np.concatenate([np.arange(32), rng.choice(U, 223, replace=False), [U - 1]]))
    wu, wg = oracle.backward_rows(inp["tokens"], None, dy, inp["gate"], R=w.R, d=d, sel_u=sel,
                                  vocab_size=w.vocab, n_threads=N_CPU)
    assert U == wu.size
    assert np.array_equal(uniq[:U].cpu().numpy().view(np.uint32), wu)
    got = grad[torch.from_numpy(sel).to(cuda_device)].cpu().numpy()
    assert np.array_equal(got.view(np.uint32), wg.astype(np.float32).view(np.uint32))


def test_backward_rows_empty_and_errors(cuda_device):
    ctx = _dummy_ctx(cuda_device, 1000, 64, 500, max_tokens=64)
    tok = torch.zeros((0, 4), dtype=torch.int32, device=cuda_device)
    count = torch.full((1,), 7, dtype=torch.int32, device=cuda_device)
    ng.ngram_backward_rows(ctx, tok, torch.zeros(0, dtype=torch.bfloat16, device=cuda_device),
                           torch.zeros(64, device=cuda_device), count_out=count)
    assert count.item() == 0
    tok = torch.zeros((2, 40), dtype=torch.int32, device=cuda_device)     # 80 > max_tokens
    with pytest.raises(ng.NgramError):
        ng.ngram_backward_rows(ctx, tok, torch.zeros((80, 64), dtype=torch.bfloat16, device=cuda_device),
                               torch.zeros(64, device=cuda_device))


def test_back_to_back_calls_keep_stream_order(cuda_device):
    """The hash, dedup, radix-sort and backward kernels are launched as programmatic
    dependents: each may be scheduled while the previous kernel of the stream still runs and
    waits for it before touching memory.  Three batches' dedup, table gradient, gate
    gradient and staged forward, issued back to back on one stream with no host
    synchronisation (the calls share the context's scratch), must equal the same calls with
    a synchronisation after each."""
    R, d, V = 65_536, 264, 7000
    w = gen.Workload("bwchain", R, d, "bf16", V, 2, 150, history=True)
    table, _ = TABLES.get(R, d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V), w.N)
    ins = [gen.make_inputs(w, token_seed=900 + i) for i in range(3)]
    toks = [to_dev_tokens(x["tokens"], cuda_device) for x in ins]
    hsts = [to_dev_tokens(x["history"], cuda_device) for x in ins]
    dys = [to_dev_bf16(_dy(w.N, d, 30 + i), cuda_device).view(w.N, d) for i in range(3)]
    res = [to_dev_bf16(x["residual"], cuda_device).view(w.N, d) for x in ins]
    gate = torch.from_numpy(ins[0]["gate"]).to(cuda_device)

    def run(sync):
        outs = []
        for i in range(3):
            uu, inv, cc = ng.ngram_dedup_rows(ctx, toks[i], history=hsts[i])
            u, c, g = ng.ngram_backward_rows(ctx, toks[i], dys[i], gate, history=hsts[i])
            gg = ng.ngram_backward_gate(ctx, toks[i], dys[i], history=hsts[i])
            ng.ngram_prefetch(ctx, i % 2, toks[i], history=hsts[i])
            y = ng.ngram_forward_staged(ctx, i % 2, res[i], gate)
            if sync:
                torch.cuda.synchronize()
            outs.append((uu, inv, cc, u, c, g, gg, y))
        torch.cuda.synchronize()
        return outs

    ref = run(True)
    got = run(False)
    for a, b in zip(ref, got):
        n_u = int(a[2].item())
        assert int(b[2].item()) == n_u and int(b[4].item()) == n_u
        assert torch.equal(a[0][:n_u], b[0][:n_u]) and torch.equal(a[1], b[1])
        assert torch.equal(a[3][:n_u], b[3][:n_u])
        assert torch.equal(a[5][:n_u].view(torch.int32), b[5][:n_u].view(torch.int32))
        assert torch.equal(a[6].view(torch.int32), b[6].view(torch.int32))
        assert torch.equal(a[7].view(torch.int16), b[7].view(torch.int16))
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


def test_backward_replays_from_a_cuda_graph(cuda_device):
    """The table and gate gradients captured in a CUDA graph (their memsets and programmatic
    dependent launches become graph nodes and edges) and replayed on new inputs copied into
    the captured buffers equal the same calls run eagerly."""
    R, d, V = 65_536, 264, 7000
    w = gen.Workload("bwgraph", R, d, "bf16", V, 2, 150, history=True)
    table, _ = TABLES.get(R, d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V), w.N)
    ins = [gen.make_inputs(w, token_seed=950 + i) for i in range(2)]
    toks = [to_dev_tokens(x["tokens"], cuda_device) for x in ins]
    hsts = [to_dev_tokens(x["history"], cuda_device) for x in ins]
    dys = [to_dev_bf16(_dy(w.N, d, 40 + i), cuda_device).view(w.N, d) for i in range(2)]
    gate = torch.from_numpy(ins[0]["gate"]).to(cuda_device)
    want = []
    for i in range(2):                       # eager; the first call also allocates the scratch
        u, c, g = ng.ngram_backward_rows(ctx, toks[i], dys[i], gate, history=hsts[i])
        gg = ng.ngram_backward_gate(ctx, toks[i], dys[i], history=hsts[i])
        want.append((u.clone(), int(c.item()), g.clone(), gg.clone()))
    tok_b, hst_b, dy_b = toks[0].clone(), hsts[0].clone(), dys[0].clone()
    uniq = torch.empty(w.N * 16, dtype=torch.int32, device=cuda_device)
    count = torch.empty(1, dtype=torch.int32, device=cuda_device)
    grad = torch.empty((w.N * 16, d), dtype=torch.float32, device=cuda_device)
    ggate = torch.empty(d, dtype=torch.float32, device=cuda_device)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cs = torch.cuda.current_stream()
        ng.ngram_backward_rows(ctx, tok_b, dy_b, gate, history=hst_b, uniq_out=uniq, count_out=count,
                               grad_rows=grad, stream=cs)
        ng.ngram_backward_gate(ctx, tok_b, dy_b, history=hst_b, out=ggate, stream=cs)
    for i in (1, 0):
        tok_b.copy_(toks[i])
        hst_b.copy_(hsts[i])
        dy_b.copy_(dys[i])
        graph.replay()
        torch.cuda.synchronize()
        u, n_u, g, gg = want[i]
        assert int(count.item()) == n_u
        assert torch.equal(uniq[:n_u], u[:n_u])
        assert torch.equal(grad[:n_u].view(torch.int32), g[:n_u].view(torch.int32))
        assert torch.equal(ggate.view(torch.int32), gg.view(torch.int32))
    del graph
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


# --------------------------------------------------------------------------- gate gradient
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("tg", [False, True])
def test_backward_gate_every_token(cuda_device, fmt, tg):
    R, d, V = 5003, 272 if fmt != "nvfp4" else 288, 7000
    nb, nt = (8, 8) if fmt in ("bf16", "nvfp4") else (3, 5)
    w = gen.Workload("bwg", R, d, fmt, V, 3, 45, history=True)
    inp = gen.make_inputs(w, token_seed=72)
    N = w.N
    dy = _dy(N, d, 5)
    table, scale = TABLES.get(R, d, ng_dtype(fmt), gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng_dtype(fmt), ng.NGRAM_RES_HBM,
                        _hp(V, nb, nt, flags=ng.NGRAM_FLAG_TOKEN_GATE if tg else 0), N, row_scale=scale)
    tok = to_dev_tokens(inp["tokens"], cuda_device)
    hst = to_dev_tokens(inp["history"], cuda_device)
    got = ng.ngram_backward_gate(ctx, tok, to_dev_bf16(dy, cuda_device).view(N, d), history=hst)
    got = got.cpu().numpy()
    kw = dict(R=R, d=d, dtype=oracle_dtype(fmt), table_seed=gen.TABLE_SEED, per_token=tg,
              n_bigram=nb, n_trigram=nt, vocab_size=V, n_threads=N_CPU)
    want32 = oracle.backward_gate(inp["tokens"], inp["history"], dy, acc=oracle.ACC_F32, **kw)
    want64, mag = oracle.backward_gate(inp["tokens"], inp["history"], dy, acc=oracle.ACC_F64,
                                       want_mag=True, **kw)
    if tg:
        assert np.array_equal(got.view(np.uint32), want32.astype(np.float32).view(np.uint32))
    else:
        # both sum exact products in fp64 (different orders) and round once
        slack = 2.0 * N * 2.0 ** -53 * mag
        assert np.all(np.abs(got - want32) <= _f32_ulp(want32) + slack)
    H = nb + nt
    assert np.all(np.abs(got - want64) <= (H + 2) * 2.0 ** -24 * mag + _f32_ulp(want64))
    again = ng.ngram_backward_gate(ctx, tok, to_dev_bf16(dy, cuda_device).view(N, d), history=hst)
    assert np.array_equal(again.cpu().numpy().view(np.uint32), got.view(np.uint32))


@pytest.mark.parametrize("name", ["full_prefill", "nvfp4_prefill"])
def test_backward_gate_full_size(cuda_device, name):
    """Full tables, 32,768 tokens: per-token values on sampled tokens bit for bit; the
    shared-gate sum equals the fp64 sum of the per-token products within fp32 rounding."""
    w = W[name]
    inp, dv = workload_on_device(w, cuda_device)
    N, d = w.N, w.d
    dy = _dy(N, d, 6)
    dy_d = to_dev_bf16(dy, cuda_device).view(N, d)
    table, scale = TABLES.get(w.R, d, ng_dtype(w.dtype), gen.TABLE_SEED, cuda_device)
    per = ng.ngram_init(table, w.R, d, ng_dtype(w.dtype), ng.NGRAM_RES_HBM,
                        _hp(w.vocab, flags=ng.NGRAM_FLAG_TOKEN_GATE), N, row_scale=scale)
    shared = ng.ngram_init(table, w.R, d, ng_dtype(w.dtype), ng.NGRAM_RES_HBM, _hp(w.vocab), N,
                           row_scale=scale)
    pt = ng.ngram_backward_gate(per, dv["tokens"], dy_d)
    sg = ng.ngram_backward_gate(shared, dv["tokens"], dy_d).cpu().numpy()
    sel = sample_tokens(w, 128)
    want = oracle.backward_gate(inp["tokens"], None, dy, R=w.R, d=d, dtype=oracle_dtype(w.dtype),
                                table_seed=gen.TABLE_SEED, per_token=True, sel=sel,
                                vocab_size=w.vocab, n_threads=N_CPU)
    got = pt[torch.from_numpy(sel).to(cuda_device)].cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.astype(np.float32).view(np.uint32))
    p64 = pt.double()
    total = p64.sum(0).cpu().numpy()
    absum = p64.abs().sum(0).cpu().numpy()
    # per-token values are fp32(dy * e): each off the exact product by <= 2^-24 of itself
    assert np.all(np.abs(sg - total) <= 2.0 ** -24 * absum * 1.01 + _f32_ulp(total))


# --------------------------------------------------------------------------- per-token gate forward
@pytest.mark.parametrize("fmt", FMTS)
def test_forward_token_gate_every_token(cuda_device, fmt):
    R, d, V = 5003, 288, 7000
    w = gen.Workload("tg", R, d, fmt, V, 2, 70, history=True)
    inp = gen.make_inputs(w, token_seed=73)
    N = w.N
    gt = _gate_tok(N, d, 7)
    table, scale = TABLES.get(R, d, ng_dtype(fmt), gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng_dtype(fmt), ng.NGRAM_RES_HBM,
                        _hp(V, flags=ng.NGRAM_FLAG_TOKEN_GATE), N, row_scale=scale)
    tok = to_dev_tokens(inp["tokens"], cuda_device)
    hst = to_dev_tokens(inp["history"], cuda_device)
    res = to_dev_bf16(inp["residual"], cuda_device).view(N, d)
    gate = to_dev_bf16(gt, cuda_device).view(N, d)
    got = from_dev_bf16(ng.ngram_forward(ctx, tok, res, gate, history=hst))
    want = oracle.forward(inp["tokens"], inp["history"], inp["residual"], None, gate_tok=gt, R=R, d=d,
                          dtype=oracle_dtype(fmt), table_seed=gen.TABLE_SEED, acc=oracle.ACC_F32,
                          n_threads=N_CPU, vocab_size=V)
    r = assert_parity(got, want)
    assert r["exact"] == r["n"]
    # grouped order, batch order, dedup staging and prefetch + staged: the same bits
    for flags in (ng.NGRAM_FLAG_SORT, ng.NGRAM_FLAG_BATCH_ORDER, ng.NGRAM_FLAG_DEDUP):
        c = ng.ngram_init(table, R, d, ng_dtype(fmt), ng.NGRAM_RES_HBM,
                          _hp(V, flags=flags | ng.NGRAM_FLAG_TOKEN_GATE), N, row_scale=scale)
        assert np.array_equal(from_dev_bf16(ng.ngram_forward(c, tok, res, gate, history=hst)), got)
    ng.ngram_prefetch(ctx, 0, tok, history=hst)
    assert np.array_equal(from_dev_bf16(ng.ngram_forward_staged(ctx, 0, res, gate)), got)
    with pytest.raises(ng.NgramError) as ei:
        ng.ngram_forward_host(ctx, tok.cpu(), res.cpu(), torch.zeros(d, device=cuda_device),
                              history=hst.cpu())
    assert ei.value.status == ng.NGRAM_EUNSUPPORTED


def test_forward_token_gate_constant_equals_shared_gate(cuda_device):
    R, d, V = 5003, 256, 7000
    w = gen.Workload("tgc", R, d, "bf16", V, 3, 50)
    inp = gen.make_inputs(w, token_seed=74)
    N = w.N
    gb = _bf16_bits(inp["gate"])
    g32 = (gb.astype(np.uint32) << 16).view(np.float32)
    table, _ = TABLES.get(R, d, ng.NGRAM_BF16, gen.TABLE_SEED, cuda_device)
    a = ng.ngram_init(table, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V), N)
    b = ng.ngram_init(table, R, d, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, _hp(V, flags=ng.NGRAM_FLAG_TOKEN_GATE), N)
    tok = to_dev_tokens(inp["tokens"], cuda_device)
    res = to_dev_bf16(inp["residual"], cuda_device).view(N, d)
    ya = ng.ngram_forward(a, tok, res, torch.from_numpy(g32).to(cuda_device))
    yb = ng.ngram_forward(b, tok, res, to_dev_bf16(np.tile(gb, (N, 1)), cuda_device).view(N, d))
    assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))
