"""GPU parity of the low-precision row formats -- FP8 E4M3 with an fp32 row scale, and
NVFP4 (E2M1 codes, an E4M3 scale per 16 columns, an fp32 global scale) -- through the
C ABI against the CPU oracle, which regenerates the same synthetic tables from the seed.

Table bytes and scales must match the oracle bit for bit; outputs must equal the
oracle's fp32-accumulated result bit for bit (the kernels compute acc = fma(q, s, acc)
per head in order, as the oracle does) and lie within the stated tolerance of its exact
fp64 result.  The hardware E4M3 / E2M1 conversions are checked on every code against
torch.float8_e4m3fn and the OCP MX value table.  Every residency mode and flag must give
the default result bit for bit.
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
FP8, NVFP4 = ng.NGRAM_FP8_E4M3_ROWSCALE, ng.NGRAM_NVFP4
E2M1_OCP = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # OCP MX v1.0, FP4 E2M1 magnitudes


def _hp(vocab, nb=8, nt=8, **kw):
    return ng.ngram_default_hash_params(vocab_size=vocab, n_bigram_heads=nb,
                                        n_trigram_heads=nt, **kw)


def _oracle(w, inp, sel=None, acc=oracle.ACC_F32, want_aux=False, **kw):
    return oracle.forward(inp["tokens"], inp["history"], inp["residual"], inp["gate"],
                          R=w.R, d=w.d, dtype=oracle_dtype(w.dtype), table_seed=gen.TABLE_SEED,
                          sel=sel, acc=acc, n_threads=N_CPU, vocab_size=w.vocab,
                          want_aux=want_aux, **kw)


def _dev(w, inp, dev):
    return {"tokens": to_dev_tokens(inp["tokens"], dev),
            "history": to_dev_tokens(inp["history"], dev),
            "residual": to_dev_bf16(inp["residual"], dev).view(w.N, w.d),
            "gate": torch.from_numpy(inp["gate"]).to(dev)}


def _fwd(ctx, dv, out=None):
    return ng.ngram_forward(ctx, dv["tokens"], dv["residual"], dv["gate"], out=out,
                            history=dv["history"])


# --------------------------------------------------------------------------- table bytes
def test_fp8_table_bitexact(cuda_device):
    R, d = 3001, 272
    table, scale = TABLES.get(R, d, FP8, 777, cuda_device)
    wq, ws = oracle.fill_fp8(777, 0, R, d)
    assert np.array_equal(table.cpu().numpy(), wq)
    assert np.array_equal(scale.cpu().numpy().view(np.uint32), ws.view(np.uint32))


@pytest.mark.parametrize("d", [32, 96, 2560])
def test_nvfp4_table_bitexact(cuda_device, d):
    """Codes, block scales and the zero padding (d = 32, 96: 14 and 10 pad bytes)."""
    R = 2001
    table, gs = TABLES.get(R, d, NVFP4, 777, cuda_device)
    assert np.array_equal(table.cpu().numpy(), oracle.fill_fp4(777, 0, R, d))
    assert gs.item() == oracle.FP4_GLOBAL_SCALE


# --------------------------------------------------------------------------- every code
def test_fp8_decode_every_code(cuda_device):
    """One row holding all 256 E4M3 codes, scale 1, R = 1 (all 16 heads read it): every
    output is 16 * e4m3(code) exactly (4 significant bits), NaN for S.1111.111."""
    d = 256
    table = torch.arange(256, dtype=torch.uint8).view(1, d).to(cuda_device)
    scale = torch.ones(1, dtype=torch.float32, device=cuda_device)
    ctx = ng.ngram_init(table, 1, d, FP8, ng.NGRAM_RES_HBM, _hp(100), 8, row_scale=scale)
    tok = torch.tensor([[3, 5]], dtype=torch.int32, device=cuda_device)
    res = torch.zeros((2, d), dtype=torch.bfloat16, device=cuda_device)
    gate = torch.ones(d, dtype=torch.float32, device=cuda_device)
    got = ng.ngram_forward(ctx, tok, res, gate).float().cpu().numpy()
    want = 16.0 * torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for row in got:
        nan = np.isnan(want)
        assert np.array_equal(np.isnan(row), nan) and nan.sum() == 2
        assert np.array_equal(row[~nan], want[~nan])


def test_nvfp4_decode_every_code_and_block_scale(cuda_device):
    """d = 4096: block b has scale code b (all 256 E4M3 codes), its 16 columns the 16 E2M1
    codes in order; global scale 1, R = 1.  Output column 16b + k = 16 * e2m1(k) *
    e4m3(b) exactly; NaN in the blocks whose scale is NaN."""
    d = 4096
    rb = ng.ngram_row_bytes(NVFP4, d)
    row = np.zeros(rb, dtype=np.uint8)
    row[:d // 2] = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], np.uint8), 256)
    row[d // 2:d // 2 + 256] = np.arange(256, dtype=np.uint8)
    table = torch.from_numpy(row).view(1, rb).to(cuda_device)
    gs = torch.ones(1, dtype=torch.float32, device=cuda_device)
    ctx = ng.ngram_init(table, 1, d, NVFP4, ng.NGRAM_RES_HBM, _hp(100), 8, row_scale=gs)
    tok = torch.tensor([[7]], dtype=torch.int32, device=cuda_device)
    res = torch.zeros((1, d), dtype=torch.bfloat16, device=cuda_device)
    gate = torch.ones(d, dtype=torch.float32, device=cuda_device)
    got = ng.ngram_forward(ctx, tok, res, gate).float().cpu().numpy()[0]
    e2m1 = np.array([(-1.0 if k & 8 else 1.0) * E2M1_OCP[k & 7] for k in range(16)])
    e4m3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    want = 16.0 * (e4m3[:, None] * e2m1[None, :]).ravel()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    # the same materialised row through the oracle
    o = oracle.forward(np.array([[7]], np.int32), None, np.zeros(d, np.uint16), np.ones(d, np.float32),
                       R=1, d=d, dtype=oracle.NVFP4, table_i8=row.reshape(1, rb),
                       row_scale=np.ones(1, np.float32), acc=oracle.ACC_F32, vocab_size=100)
    ob = (o.astype(np.uint32) << 16).view(np.float32).ravel()
    assert np.array_equal(np.isnan(ob), nan) and np.array_equal(ob[~nan], got[~nan])


# --------------------------------------------------------------------------- every token
SHAPES = {
    "fp8": [(16, 8, 8, 3, 37, False),      # one 16-column vector per row
            (272, 3, 5, 2, 45, True),      # 17 vectors: ragged strip
            (528, 16, 0, 1, 70, True),     # 33 vectors
            (2560, 8, 8, 2, 60, True),     # the pages' width
            (2576, 0, 16, 3, 11, False),   # 161 vectors: ragged tail
            (272, 3, 4, 2, 45, True)],     # 7 heads
    "nvfp4": [(32, 8, 8, 3, 37, False),    # two scale blocks, 14 pad bytes
              (288, 3, 5, 2, 45, True),    # 18 blocks
              (544, 16, 0, 1, 70, True),   # 34 blocks
              (2560, 8, 8, 2, 60, True),
              (2592, 0, 16, 3, 11, False),   # 162 blocks: ragged tail
              (288, 3, 4, 2, 45, True),    # 7 heads: the last block scale converted alone
              (32, 1, 0, 2, 9, False)],    # a single head
}


@pytest.mark.parametrize("fmt,shape", [(f, s) for f in ("fp8", "nvfp4") for s in SHAPES[f]])
def test_forward_every_token(cuda_device, fmt, shape):
    d, nb, nt, n_seq, T, hist = shape
    R, V = 5003, 7000
    w = gen.Workload(fmt + "_ragged", R, d, fmt, V, n_seq, T, history=hist)
    inp = gen.make_inputs(w, token_seed=61)
    table, scale = TABLES.get(R, d, ng_dtype(fmt), gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, ng_dtype(fmt), ng.NGRAM_RES_HBM, _hp(V, nb, nt), w.N,
                        row_scale=scale)
    got = from_dev_bf16(_fwd(ctx, _dev(w, inp, cuda_device)))
    r = assert_parity(got, _oracle(w, inp, n_bigram=nb, n_trigram=nt))
    assert r["exact"] == r["n"]
    want64, _, mag, _ = _oracle(w, inp, acc=oracle.ACC_F64, want_aux=True, n_bigram=nb,
                                n_trigram=nt)
    assert_parity(got, want64, mag)
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


@pytest.mark.parametrize("name", ["fp8_prefill", "nvfp4_prefill"])
def test_forward_full_size_sampled(cuda_device, name):
    """20M x 2560 tables (FP8 47.8 GiB, NVFP4 26.8 GiB), one 32,768-token Zipf prefill in
    the benchmark's launch configuration; 512 tokens sampled."""
    w = W[name]
    inp, dv = workload_on_device(w, cuda_device)
    table, scale = TABLES.get(w.R, w.d, ng_dtype(w.dtype), gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, w.R, w.d, ng_dtype(w.dtype), ng.NGRAM_RES_HBM, _hp(w.vocab), w.N,
                        row_scale=scale)
    got = from_dev_bf16(_fwd(ctx, dv)).reshape(w.N, w.d)
    sel = sample_tokens(w, 512)
    r = assert_parity(got[sel], _oracle(w, inp, sel=sel))
    assert r["exact"] == r["n"]
    # the stated bar against the exact definition, independent of the fp32 rounding order
    want64, _, mag, _ = _oracle(w, inp, sel=sel, acc=oracle.ACC_F64, want_aux=True)
    assert_parity(got[sel], want64, mag)
    # batch order gives the same bits as the default grouped order
    b = ng.ngram_init(table, w.R, w.d, ng_dtype(w.dtype), ng.NGRAM_RES_HBM,
                      _hp(w.vocab, flags=ng.NGRAM_FLAG_BATCH_ORDER), w.N, row_scale=scale)
    assert np.array_equal(from_dev_bf16(_fwd(b, dv)).reshape(w.N, w.d), got)
    assert ng.ngram_get_device_error(ctx)[0] == ng.NGRAM_OK


def test_nvfp4_global_scale_from_host_memory_and_other_values(cuda_device):
    """The global scale is copied at init from host or device memory; another value gives
    the oracle's result for that value."""
    R, d, V = 5003, 288, 7000
    w = gen.Workload("nvfp4_gs", R, d, "nvfp4", V, 2, 40, history=True)
    inp = gen.make_inputs(w, token_seed=62)
    dv = _dev(w, inp, cuda_device)
    table, gs_dev = TABLES.get(R, d, NVFP4, gen.TABLE_SEED, cuda_device)
    a = ng.ngram_init(table, R, d, NVFP4, ng.NGRAM_RES_HBM, _hp(V), w.N, row_scale=gs_dev)
    ref = from_dev_bf16(_fwd(a, dv))
    host_gs = torch.tensor([oracle.FP4_GLOBAL_SCALE], dtype=torch.float32)   # pageable
    b = ng.ngram_init(table, R, d, NVFP4, ng.NGRAM_RES_HBM, _hp(V), w.N, row_scale=host_gs)
    assert np.array_equal(from_dev_bf16(_fwd(b, dv)), ref)
    other = np.array([0.3125], dtype=np.float32)
    c = ng.ngram_init(table, R, d, NVFP4, ng.NGRAM_RES_HBM, _hp(V), w.N,
                      row_scale=torch.from_numpy(other))
    got = from_dev_bf16(_fwd(c, dv))
    r = assert_parity(got, _oracle(w, inp, row_scale=other))
    assert r["exact"] == r["n"]


# --------------------------------------------------------------------------- modes and flags
@pytest.mark.parametrize("fmt", ["int8", "fp8", "nvfp4"])
@pytest.mark.parametrize("n_seq,T,hist", [(3, 200, True), (1, 20_000, False)])
def test_tma_staged_gather_bitidentical(cuda_device, fmt, n_seq, T, hist):
    """NGRAM_FLAG_TMA_STAGING (whole rows staged in shared memory by cp.async.bulk) gives
    the register gather's bits, in batch order and in grouped order (20,000 tokens)."""
    R, d, V = 400_000, 2560, 151_936
    w = gen.Workload(fmt + "_tma", R, d, fmt, V, n_seq, T, history=hist)
    inp, dv = workload_on_device(w, cuda_device, token_seed=65)
    dt = ng_dtype(fmt)
    table, scale = TABLES.get(R, d, dt, gen.TABLE_SEED, cuda_device)
    ref = from_dev_bf16(_fwd(ng.ngram_init(table, R, d, dt, ng.NGRAM_RES_HBM, _hp(V), w.N, row_scale=scale), dv))
    c = ng.ngram_init(table, R, d, dt, ng.NGRAM_RES_HBM, _hp(V, flags=ng.NGRAM_FLAG_TMA_STAGING), w.N,
                      row_scale=scale)
    for _ in range(2):
        assert np.array_equal(from_dev_bf16(_fwd(c, dv)), ref)
    assert ng.ngram_get_device_error(c)[0] == ng.NGRAM_OK
    sel = sample_tokens(w, 64, seed=4)
    r = assert_parity(ref.reshape(w.N, d)[sel], _oracle(w, inp, sel=sel))
    assert r["exact"] == r["n"]


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_flags_and_staging_bitidentical(cuda_device, fmt):
    """Dedup staging, grouped order, batch order and prefetch + staged gather give the
    default result bit for bit; the default equals the oracle."""
    R, d, V = 400_000, 2560, 151_936
    w = gen.Workload(fmt + "_modes", R, d, fmt, V, 4, 1500, history=True)
    inp, dv = workload_on_device(w, cuda_device, token_seed=63)
    dt = ng_dtype(fmt)
    table, scale = TABLES.get(R, d, dt, gen.TABLE_SEED, cuda_device)
    ctx = ng.ngram_init(table, R, d, dt, ng.NGRAM_RES_HBM, _hp(V), w.N, row_scale=scale)
    ref = from_dev_bf16(_fwd(ctx, dv))
    sel = sample_tokens(w, 96, seed=3)
    r = assert_parity(ref.reshape(w.N, d)[sel], _oracle(w, inp, sel=sel))
    assert r["exact"] == r["n"]
    for flags in (ng.NGRAM_FLAG_DEDUP, ng.NGRAM_FLAG_SORT, ng.NGRAM_FLAG_BATCH_ORDER):
        c = ng.ngram_init(table, R, d, dt, ng.NGRAM_RES_HBM, _hp(V, flags=flags), w.N, row_scale=scale)
        for _ in range(2):
            assert np.array_equal(from_dev_bf16(_fwd(c, dv)), ref), flags
    ng.ngram_prefetch(ctx, 1, dv["tokens"], history=dv["history"])
    got = ng.ngram_forward_staged(ctx, 1, dv["residual"], dv["gate"])
    assert np.array_equal(from_dev_bf16(got), ref)
    host_out = ng.ngram_forward_host(ctx, dv["tokens"].cpu(), dv["residual"].cpu(), dv["gate"],
                                     history=dv["history"].cpu())
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_bf16(host_out), ref)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_host_residency_bitidentical(cuda_device, fmt):
    """The table in pinned host memory (filled through its device alias): UVA, DMA, AUTO,
    UVA grouped and UVA + dedup equal the HBM result bit for bit."""
    R, d, V = 300_000, 2560, 151_936
    dt = ng_dtype(fmt)
    TABLES.drop()
    rb = ng.ngram_row_bytes(dt, d)
    host = ng.HostTable((R, rb), torch.uint8)
    hs = ng.HostTable((R if fmt == "fp8" else 1,), torch.float32)
    try:
        ng.ngram_fill_synthetic(host.tensor, R, d, dt, gen.TABLE_SEED, row_scale=hs.tensor)
        torch.cuda.synchronize()
        table, scale = TABLES.get(R, d, dt, gen.TABLE_SEED, cuda_device)
        rows = torch.tensor([0, 1, 4567, R - 1])
        assert torch.equal(host.tensor[rows], table[rows.to(cuda_device)].cpu())
        for n_seq, T, hist in ((1, 1, True), (64, 1, True), (2, 900, False)):
            w = gen.Workload(fmt + "_host", R, d, fmt, V, n_seq, T, history=hist)
            inp, dv = workload_on_device(w, cuda_device, token_seed=64 + n_seq)
            hbm = ng.ngram_init(table, R, d, dt, ng.NGRAM_RES_HBM, _hp(V), w.N, row_scale=scale)
            ref = from_dev_bf16(_fwd(hbm, dv))
            for where, flags in ((ng.NGRAM_RES_HOST_UVA, 0), (ng.NGRAM_RES_HOST_DMA, 0),
                                 (ng.NGRAM_RES_HOST_AUTO, 0), (ng.NGRAM_RES_HOST_UVA, ng.NGRAM_FLAG_SORT),
                                 (ng.NGRAM_RES_HOST_UVA, ng.NGRAM_FLAG_DEDUP)):
                c = ng.ngram_init(host.tensor, R, d, dt, where, _hp(V, flags=flags), w.N,
                                  row_scale=hs.tensor)
                for _ in range(2):
                    assert np.array_equal(from_dev_bf16(_fwd(c, dv)), ref), (where, flags)
                if where == ng.NGRAM_RES_HOST_UVA and flags == 0:
                    # the gate gradient reads the host rows through UVA: the HBM result
                    dy = dv["residual"]
                    g_hbm = ng.ngram_backward_gate(hbm, dv["tokens"], dy, history=dv["history"])
                    g_uva = ng.ngram_backward_gate(c, dv["tokens"], dy, history=dv["history"])
                    assert torch.equal(g_hbm, g_uva)
                c.close()
    finally:
        TABLES.drop()
        host.close()
        hs.close()
