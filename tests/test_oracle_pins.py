"""Pins for the CPU oracle: each test checks it against something other than itself.

Published known-answer values (tests/golden/), closed forms, library routines
(torch.nn.functional.embedding_bag / embedding, torch's fp32 -> bf16 conversion),
brute force on tiny inputs and invariants of the method.  The method is the one in
"Qwen Brought Back N-Grams. All 51 Billion Parameters of Them." (section "N-grams, of
all things": hash bigram + trigram context, gather 16 rows, sum, add to the residual)
with the gate of "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with Heterogeneous
Memory Prefetch", Key point 1 (h = h + W_g elementwise e_Ngram).
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import ngram_inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GAMMA = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1
PAD = oracle.DEFAULT_PAD_ID
K_BF16 = float.fromhex("0x1.1bc77ap-22")
K_INT8 = float.fromhex("0x1.1bc5f4p-11")


def _kat(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(x, 16) for x in line.split()])
    return rows


def _bits_to_f64(bits):
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def _bf16_ulp(v):
    """Spacing of bf16 values at |v| (8 significant bits; 2^-133 below the normals)."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    return np.where(v > 0, np.exp2(np.maximum(e - 7, -133)), 2.0 ** -133)


# --------------------------------------------------------------------------- generators
def test_splitmix64_known_answers():
    for seed, *outs in _kat("splitmix64_kat.txt"):
        assert oracle.splitmix64_outputs(seed, len(outs)) == outs


def test_head_seeds_are_successive_splitmix64_outputs():
    (seed, *outs), = _kat("splitmix64_kat.txt")
    assert [int(x) for x in oracle.head_seeds(seed, 3)] == outs


def test_philox4x32_10_known_answers():
    for row in _kat("philox4x32_10_kat.txt"):
        ctr, key, want = row[0:4], row[4:6], row[6:10]
        assert [int(x) for x in oracle.philox4x32_10(ctr, key)] == want


# --------------------------------------------------------------------------- the hash
def _unxorshift(y, s):
    x = y
    for _ in range(64 // s + 1):
        x = y ^ (x >> s)
    return x & M64


def _splitmix_state_for_output(z):
    """Invert the splitmix64 output function (xorshifts and odd multipliers are
    bijections mod 2^64): returns the state whose next() output is z."""
    z = _unxorshift(z, 31)
    z = (z * pow(0x94D049BB133111EB, -1, 1 << 64)) & M64
    z = _unxorshift(z, 27)
    z = (z * pow(0xBF58476D1CE4E5B9, -1, 1 << 64)) & M64
    return _unxorshift(z, 30)


@pytest.mark.parametrize("head,R", [(0, 20_000_000), (5, 65_536), (8, 1_000_003),
                                    (15, 4_294_967_291)])
def test_hash_path_reaches_known_answer(head, R):
    """Choose base_seed so that seed_head equals the packed key of one context; then
    key ^ seed = 0 and the row must be splitmix64's first output from 0, mod R."""
    (_, first_out, *_), = _kat("splitmix64_kat.txt")
    w2, w1, w0 = 1_500_001, 678_901, 12_345
    key = ((w1 << 21) | w0) if head < 8 else ((w2 << 42) | (w1 << 21) | w0)
    state = _splitmix_state_for_output(key)
    base = (state - (head + 1) * GAMMA) & M64
    assert int(oracle.head_seeds(base, 16)[head]) == key
    idx = oracle.indices([[w2, w1, w0]], None, R, base_seed=base, vocab_size=PAD)
    assert int(idx[2, head]) == first_out % R


def test_bigram_heads_ignore_w2_and_trigram_heads_do_not():
    toks = np.array([[7, 100, 200], [9, 100, 200]], dtype=np.int32)
    idx = oracle.indices(toks, None, 1 << 30, vocab_size=1000)
    a, b = idx[2], idx[5]
    assert np.array_equal(a[:8], b[:8])
    assert np.all(a[8:] != b[8:])
    assert len(set(a.tolist())) == 16          # 16 distinct heads on this context


def test_power_of_two_R_is_a_mask():
    toks = gen.zipf_tokens(2, 300, 32_000, seed=11)
    big = oracle.indices(toks, None, 1 << 31, vocab_size=32_000)
    for k in (1, 10, 16, 20):
        small = oracle.indices(toks, None, 1 << k, vocab_size=32_000)
        assert np.array_equal(small, big & ((1 << k) - 1))


def test_repeated_context_gives_identical_rows():
    toks = np.array([[3, 4, 5, 6, 3, 4, 5, 9, 4, 5]], dtype=np.int32)
    idx = oracle.indices(toks, None, 65_536, vocab_size=100)
    assert np.array_equal(idx[2], idx[6])      # (3,4,5) at t=2 and t=6
    assert np.array_equal(idx[6, :8], idx[9, :8])   # bigram (4,5) again at t=9
    assert not np.array_equal(idx[6, 8:], idx[9, 8:])


# --------------------------------------------------------------------------- boundaries
def test_pad_history_equivalences():
    V = 32_000
    toks = gen.zipf_tokens(1, 64, V, seed=5)
    full = oracle.indices(toks, None, 65_536, vocab_size=V)
    # no history == explicit PAD history
    assert np.array_equal(full, oracle.indices(toks, [[PAD, PAD]], 65_536, vocab_size=V))
    # writing the pads as tokens reproduces the boundary positions
    padded = np.concatenate([[[PAD, PAD]], toks], axis=1).astype(np.int32)
    assert np.array_equal(oracle.indices(padded, None, 65_536, vocab_size=V)[2:], full)


def test_chunked_prefill_and_decode_equal_full_prefill():
    V = 151_936
    toks = gen.zipf_tokens(1, 40, V, seed=6)
    full = oracle.indices(toks, None, 20_000_000, vocab_size=V)
    c1, c2 = toks[:, :17], toks[:, 17:]
    i1 = oracle.indices(c1, None, 20_000_000, vocab_size=V)
    i2 = oracle.indices(c2, c1[:, -2:], 20_000_000, vocab_size=V)
    assert np.array_equal(np.concatenate([i1, i2]), full)
    ext = np.concatenate([[PAD, PAD], toks[0]])
    for t in range(toks.shape[1]):
        step = oracle.indices([[toks[0, t]]], [[ext[t], ext[t + 1]]], 20_000_000, vocab_size=V)
        assert np.array_equal(step[0], full[t])


def test_contexts_do_not_cross_sequences():
    V = 32_000
    toks = gen.zipf_tokens(3, 20, V, seed=7)
    allidx = oracle.indices(toks, None, 65_536, vocab_size=V)
    for s in range(3):
        alone = oracle.indices(toks[s:s + 1], None, 65_536, vocab_size=V)
        assert np.array_equal(allidx[s * 20:(s + 1) * 20], alone)


def test_out_of_vocab_tokens_read_as_pad():
    V = 1000
    a = oracle.indices([[5, 6, 7]], None, 65_536, vocab_size=V)
    b = oracle.indices([[5, V + 3, 7]], None, 65_536, vocab_size=V)
    c = oracle.indices([[5, PAD, 7]], None, 65_536, vocab_size=V)
    assert np.array_equal(b, c) and not np.array_equal(a, b)


def test_empty_batch():
    assert oracle.indices(np.zeros((0, 5), np.int32), None, 100).shape == (0, 16)
    out = oracle.forward(np.zeros((2, 0), np.int32), None, np.zeros((0, 8), np.uint16),
                         np.ones(8, np.float32), R=100, d=8, table_seed=1)
    assert out.shape == (0, 8)


# --------------------------------------------------------------------------- bf16 rounding
def test_bf16_from_f32_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2**16, size=5000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    bits = np.concatenate([bits, ties, np.array([0, 0x80000000, 0x7F7FFFFF, 0x7F7F8000], np.uint32)])
    bits = bits[(bits & 0x7F800000) != 0x7F800000]             # finite only
    f = bits.view(np.float32)
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_from_f32(x) for x in f[:20000]], dtype=np.uint16)
    assert np.array_equal(got, want[:20000])
    got_t = np.array([oracle.bf16_from_f32(x) for x in f[-5004:]], dtype=np.uint16)
    assert np.array_equal(got_t, want[-5004:])


def test_bf16_from_f64_is_nearest_even():
    rng = np.random.default_rng(1)
    ys = list(rng.standard_normal(3000) * np.exp2(rng.integers(-40, 40, 3000)))
    # exact midpoints between neighbouring bf16 values, both parities
    for m in range(128, 256, 7):
        for e in (-30, -3, 0, 5):
            ys.append((m + 0.5) * 2.0 ** (e - 7))
            ys.append(-(m + 0.5) * 2.0 ** (e - 7))
    for y in ys:
        b = oracle.bf16_from_f64(y)
        v = Fraction(float(_bits_to_f64([b])[0]))
        nb = [Fraction(float(_bits_to_f64([(b + k) & 0xFFFF])[0])) for k in (-1, 1)]
        fy = Fraction(y)
        assert all(abs(fy - v) <= abs(fy - w) for w in nb), y
        for w in nb:
            if abs(fy - v) == abs(fy - w):
                assert b % 2 == 0, y


# --------------------------------------------------------------------------- table values
def test_bf16_table_distribution_closed_form():
    """C = 2S - 262140, S a sum of four iid U{0..65535}: mean 0, std
    4 * sqrt((65536^2 - 1) / 12) = 75674.4, so std(C * K) = 0.02, |C| <= 262140."""
    v = _bits_to_f64(oracle.fill_bf16(gen.TABLE_SEED, 1234, 300, 512)).ravel()
    n = v.size
    assert abs(v.mean()) < 4 * 0.02 / np.sqrt(n)
    assert abs(v.std() / 0.02 - 1) < 0.01
    assert np.abs(v).max() <= 262140 * K_BF16 * (1 + 2 ** -8)
    # Irwin-Hall(4) kurtosis = 3 - 6/(5*4) = 2.7
    kurt = ((v - v.mean()) ** 4).mean() / v.var() ** 2
    assert abs(kurt - 2.7) < 0.03
    # columns and rows are independent streams
    m = v.reshape(300, 512)
    assert abs(np.corrcoef(m[:, 0::2].ravel(), m[:, 1::2].ravel())[0, 1]) < 0.01
    assert abs(np.corrcoef(m[:-1].ravel(), m[1:].ravel())[0, 1]) < 0.01


def test_int8_table_distribution_closed_form():
    """q = floor((B - 510) / 4), B a sum of four iid bytes: std(B) = sqrt(4*(256^2-1)/12),
    mean(q) = -3/8 (floor of quarter steps), range [-128, 127]; row scale in
    [0.75, 1.25) * K8 with mean K8."""
    q, s = oracle.fill_int8(gen.TABLE_SEED, 77, 400, 512)
    qf = q.astype(np.float64).ravel()
    assert q.min() >= -128 and q.max() <= 127
    assert abs(qf.mean() + 0.375) < 4 * 37 / np.sqrt(qf.size)
    var_b = 4 * (256 ** 2 - 1) / 12
    # var(q) = var(B) / 16 + 5/64 (the dropped quarter steps, uniform on {0, 1/4, 1/2, 3/4})
    assert abs(qf.std() / np.sqrt(var_b / 16 + 5 / 64) - 1) < 0.01
    assert np.all(s >= 0.75 * K_INT8) and np.all(s < 1.25 * K_INT8)
    assert abs(s.mean() / K_INT8 - 1) < 0.02


def test_table_is_a_pure_function_of_seed_row_col():
    a = oracle.fill_bf16(99, 10, 4, 64)
    b = oracle.fill_bf16(99, 12, 2, 64)
    assert np.array_equal(a[2:], b)
    assert oracle.table_bf16(99, 11, 5) == a[1, 5]
    assert not np.array_equal(a, oracle.fill_bf16(100, 10, 4, 64))


# --------------------------------------------------------------------------- the sum
def _tiny_case(seed=0, n_seq=3, T=17, V=50, R=97, d=24, nb=8, nt=8):
    rng = np.random.default_rng(seed)
    toks = rng.integers(0, V, (n_seq, T)).astype(np.int32)
    res = gen.residual_bf16_bits(n_seq * T, d, seed + 1)
    g = gen.gate_f32(d, seed + 2)
    return toks, res, g


def _one_hot_sum(idx, E):
    N, H = idx.shape
    A = np.zeros((N, E.shape[0]))
    for t in range(N):
        for h in range(H):
            A[t, idx[t, h]] += 1.0          # colliding heads count twice
    return A @ E


@pytest.mark.parametrize("dtype", [oracle.BF16, oracle.INT8])
def test_brute_force_one_hot_matmul_and_embedding_bag(dtype):
    R, d, V = 97, 24, 50
    toks, res, g = _tiny_case(R=R, d=d, V=V)
    if dtype == oracle.BF16:
        E = _bits_to_f64(oracle.fill_bf16(42, 0, R, d)).reshape(R, d)
    else:
        q, s = oracle.fill_int8(42, 0, R, d)
        E = q.astype(np.float64) * s.astype(np.float64)[:, None]
    out, y, mag, idx = oracle.forward(toks, None, res, g, R=R, d=d, dtype=dtype, table_seed=42,
                                      acc=oracle.ACC_F64, vocab_size=V, want_aux=True)
    assert np.array_equal(idx, oracle.indices(toks, None, R, vocab_size=V))
    e = _one_hot_sum(idx, E)
    bag = torch.nn.functional.embedding_bag(torch.from_numpy(idx.astype(np.int64)),
                                            torch.from_numpy(E), mode="sum").numpy()
    assert np.array_equal(e, bag)
    r = _bits_to_f64(res).reshape(-1, d)
    assert np.array_equal(y, r + g.astype(np.float64)[None, :] * e)
    v = _bits_to_f64(out).reshape(y.shape)
    assert np.all(np.abs(v - y) <= _bf16_ulp(y) / 2)     # rounded to a nearest bf16
    assert np.allclose(mag, np.abs(r) + g[None, :] * (np.abs(E)[idx].sum(axis=1)))


def test_collisions_count_once_per_head():
    """R = 2 forces heads to collide: the sum must count every head's row."""
    toks, res, g = _tiny_case(R=2, d=8, T=5, n_seq=1)
    E = _bits_to_f64(oracle.fill_bf16(3, 0, 2, 8)).reshape(2, 8)
    out, y, _, idx = oracle.forward(toks, None, np.zeros_like(res), np.ones(8, np.float32),
                                    R=2, d=8, table_seed=3, acc=oracle.ACC_F64,
                                    vocab_size=50, want_aux=True)
    counts = np.stack([(idx == 0).sum(1), (idx == 1).sum(1)], 1).astype(np.float64)
    assert np.array_equal(y, counts @ E)


def test_single_head_reduces_to_embedding():
    R, d, V = 1000, 32, 500
    toks, res, g = _tiny_case(R=R, d=d, V=V)
    Eb = oracle.fill_bf16(8, 0, R, d)
    for nb, nt in ((1, 0), (0, 1)):
        out, _, _, idx = oracle.forward(toks, None, np.zeros_like(res), np.ones(d, np.float32),
                                        R=R, d=d, table_seed=8, n_bigram=nb, n_trigram=nt,
                                        vocab_size=V, want_aux=True)
        emb = torch.nn.functional.embedding(torch.from_numpy(idx[:, 0].astype(np.int64)),
                                            torch.from_numpy(Eb.astype(np.int32))).numpy()
        assert np.array_equal(out, emb.astype(np.uint16))


@pytest.mark.parametrize("acc", [oracle.ACC_F32, oracle.ACC_F64])
def test_zero_gate_returns_residual_bitwise(acc):
    toks, res, g = _tiny_case()
    out = oracle.forward(toks, None, res, np.zeros_like(g), R=97, d=24, table_seed=1,
                         acc=acc, vocab_size=50)
    assert np.array_equal(out, res.reshape(out.shape))


def test_unit_gate_zero_residual_is_fp32_head_order_sum():
    """r = 0, g = 1: the fp32 reference is bf16(fp32 sum in head order), computed here
    with torch fp32 adds and torch's bf16 conversion."""
    R, d, V = 300, 40, 60
    toks, res, _ = _tiny_case(R=R, d=d, V=V)
    E32 = torch.from_numpy(_bits_to_f64(oracle.fill_bf16(5, 0, R, d)).reshape(R, d).astype(np.float32))
    out, _, _, idx = oracle.forward(toks, None, np.zeros_like(res), np.ones(d, np.float32), R=R,
                                    d=d, table_seed=5, acc=oracle.ACC_F32, vocab_size=V,
                                    want_aux=True)
    rows = E32[torch.from_numpy(idx.astype(np.int64))]          # [N][H][d]
    acc = torch.zeros(rows.shape[0], d, dtype=torch.float32)
    for h in range(rows.shape[1]):
        acc = acc + rows[:, h]
    want = acc.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out, want)


def test_head_order_invariance_fp64_exact_fp32_within_rounding():
    R, d, V = 500, 32, 80
    toks, res, g = _tiny_case(R=R, d=d, V=V)
    E = _bits_to_f64(oracle.fill_bf16(9, 0, R, d)).reshape(R, d)
    _, y64, mag, idx = oracle.forward(toks, None, np.zeros_like(res), np.ones(d, np.float32),
                                      R=R, d=d, table_seed=9, acc=oracle.ACC_F64, vocab_size=V,
                                      want_aux=True)
    _, y32, _, _ = oracle.forward(toks, None, np.zeros_like(res), np.ones(d, np.float32), R=R,
                                  d=d, table_seed=9, acc=oracle.ACC_F32, vocab_size=V,
                                  want_aux=True)
    rev = E[idx[:, ::-1]].sum(axis=1)        # reverse head order, fp64 (exact)
    assert np.array_equal(y64, rev)
    # fp32 head-order sum: at most 15 roundings of partial sums bounded by sum |E|
    assert np.all(np.abs(y32 - y64) <= 16 * 2.0 ** -24 * mag)


def test_fp32_reference_within_tolerance_of_exact_definition():
    """The two accumulation modes agree to 1 bf16 ulp except where cancellation brings
    y close to zero (absolute slack 2^-20 * (|r| + |g| sum |E|))."""
    w = gen.WORKLOADS["tiny"]
    inp = gen.make_inputs(w)
    o32 = oracle.forward(inp["tokens"], None, inp["residual"], inp["gate"], R=w.R, d=w.d,
                         table_seed=gen.TABLE_SEED, acc=oracle.ACC_F32, vocab_size=w.vocab,
                         n_threads=4)
    o64, y64, mag, _ = oracle.forward(inp["tokens"], None, inp["residual"], inp["gate"], R=w.R,
                                      d=w.d, table_seed=gen.TABLE_SEED, acc=oracle.ACC_F64,
                                      vocab_size=w.vocab, n_threads=4, want_aux=True)
    a, b = _bits_to_f64(o32).reshape(y64.shape), _bits_to_f64(o64).reshape(y64.shape)
    tol = _bf16_ulp(b) + 2.0 ** -20 * mag
    assert np.all(np.abs(a - b) <= tol)
    assert np.mean(a == b) > 0.999


# --------------------------------------------------------------------------- dedup
def test_unique_rows_against_numpy_unique():
    """First-appearance order and inverse map agree with numpy.unique (library) and
    reconstruct every entry."""
    toks = gen.zipf_tokens(4, 300, 2000, seed=61)
    idx = oracle.indices(toks, None, 5000, vocab_size=2000)
    uniq, inv = oracle.unique_rows(idx)
    flat = idx.ravel()
    u_sorted, first, _ = np.unique(flat, return_index=True, return_inverse=True)
    order = np.argsort(first, kind="stable")
    assert np.array_equal(uniq, u_sorted[order])
    assert np.array_equal(uniq[inv], flat)
    assert len(set(uniq.tolist())) == uniq.size == u_sorted.size
    # the inverse of each first occurrence is increasing: 0, 1, 2, ...
    assert np.array_equal(inv[np.sort(first)], np.arange(uniq.size))


def test_unique_rows_keeps_colliding_heads():
    idx = np.array([[3, 3, 3, 7], [7, 3, 9, 9]], dtype=np.uint32)
    uniq, inv = oracle.unique_rows(idx)
    assert uniq.tolist() == [3, 7, 9]
    assert inv.tolist() == [0, 0, 0, 1, 1, 0, 2, 2]


# --------------------------------------------------------------------------- int8 fp32 mode
def test_fmaf_is_correctly_rounded():
    """The oracle's int8 fp32 accumulation is one fmaf per head; check that the C
    library's fmaf returns the float nearest to the exact a * b + c."""
    import ctypes
    import random
    libm = ctypes.CDLL("libm.so.6")
    libm.fmaf.restype = ctypes.c_float
    libm.fmaf.argtypes = [ctypes.c_float] * 3
    rng = random.Random(3)
    for _ in range(5000):
        a, b, c = (float(np.float32(rng.uniform(-1, 1) * 2.0 ** rng.randint(-30, 30)))
                   for _ in range(3))
        exact = Fraction(a) * Fraction(b) + Fraction(c)
        f = np.float32(libm.fmaf(a, b, c))
        for nb in (np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))):
            assert abs(Fraction(float(f)) - exact) <= abs(Fraction(float(nb)) - exact)


def test_int8_fp32_mode_within_tolerance_of_exact():
    R, d, V = 3000, 64, 500
    toks, res, g = _tiny_case(R=R, d=d, V=V, n_seq=4, T=40)
    o32 = oracle.forward(toks, None, res, g, R=R, d=d, dtype=oracle.INT8, table_seed=17,
                         acc=oracle.ACC_F32, vocab_size=V)
    o64, y64, mag, _ = oracle.forward(toks, None, res, g, R=R, d=d, dtype=oracle.INT8,
                                      table_seed=17, acc=oracle.ACC_F64, vocab_size=V,
                                      want_aux=True)
    a, b = _bits_to_f64(o32).reshape(y64.shape), _bits_to_f64(o64).reshape(y64.shape)
    assert np.all(np.abs(a - b) <= _bf16_ulp(b) + 2.0 ** -20 * mag)


def _f32_of_exact_sum(p64, acc32):
    """fp32 nearest (ties to even) to the exact p64 + acc32, where p64 is an exact fp64
    product: the fp64 sum s plus its exact error (Knuth's TwoSum) is the exact value; s
    rounds to the right fp32 unless s sits exactly halfway between two fp32 values, where
    the sign of the error decides.  Written from IEEE 754 round-to-nearest, no fmaf."""
    a = acc32.astype(np.float64)
    s = p64 + a
    bb = s - p64
    err = (p64 - (s - bb)) + (a - bb)
    f = s.astype(np.float32)
    dlt = s - f.astype(np.float64)                          # exact: f is within an ulp of s
    toward = np.where(dlt > 0, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf)))
    mid = (dlt != 0) & (2.0 * dlt == toward.astype(np.float64) - f.astype(np.float64))
    return np.where(mid & (err != 0) & (np.sign(err) == np.sign(dlt)), toward, f)


@pytest.mark.parametrize("fmt", ["int8", "fp8"])
def test_scaled_rows_fp32_mode_is_one_rounding_per_head(fmt):
    """The fp32 reference of the row-scale formats (int8, FP8 E4M3), restated without the
    oracle's arithmetic: per head, the exact product q * s (q: the int8 value, or the E4M3
    code decoded by torch's float8_e4m3fn; s: the fp32 row scale) is added to the fp32
    accumulator with ONE rounding, in head order 0..15; then y = fp32(r + fp32(g * acc))
    with numpy's fp32 multiply and add, and bf16 by torch.  The oracle's fp32 value y and
    its bf16 output must equal this bit for bit.  The same chain with the product rounded
    on its own first (two roundings per head) must differ somewhere, so this pin tells the
    two readings apart (the bf16 output alone rarely can)."""
    R, d, V = 211, 64, 90
    toks, res, g = _tiny_case(seed=5, R=R, d=d, V=V, n_seq=4, T=40)
    N = toks.size
    if fmt == "int8":
        q, s = oracle.fill_int8(23, 0, R, d)
        qv, dt = q.astype(np.float64), oracle.INT8
    else:
        q, s = oracle.fill_fp8(23, 0, R, d)
        qv, dt = _e4m3_torch(q), oracle.FP8
    idx = oracle.indices(toks, None, R=R, vocab_size=V).reshape(N, 16)
    acc1 = np.zeros((N, d), dtype=np.float32)                 # one rounding per head
    acc2 = np.zeros((N, d), dtype=np.float32)                 # product rounded first
    for h in range(16):
        p = qv[idx[:, h]] * s[idx[:, h]].astype(np.float64)[:, None]     # exact in fp64
        acc1 = _f32_of_exact_sum(p, acc1)
        acc2 = (p.astype(np.float32) + acc2).astype(np.float32)
    r32 = _bits_to_f64(res).reshape(N, d).astype(np.float32)
    for rr, gg in ((np.zeros_like(r32), np.ones(d, np.float32)), (r32, g)):
        y1 = (rr + (gg[None, :] * acc1).astype(np.float32)).astype(np.float32)
        y2 = (rr + (gg[None, :] * acc2).astype(np.float32)).astype(np.float32)
        rbits = torch.from_numpy(rr.ravel()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        want = torch.from_numpy(y1.ravel()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        for kw in (dict(table_i8=q, row_scale=s), dict(table_seed=23)):
            out, y, _, _ = oracle.forward(toks, None, rbits, gg, R=R, d=d, dtype=dt,
                                          acc=oracle.ACC_F32, vocab_size=V, want_aux=True, **kw)
            assert np.array_equal(y.astype(np.float32).ravel().view(np.uint32), y1.ravel().view(np.uint32))
            assert np.array_equal(out.ravel(), want)
        assert np.any(y1 != y2)



# --------------------------------------------------------------------------- low-precision rows
def test_e4m3_decode_matches_torch_float8_e4m3fn():
    want = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and got[0x7E] == 448.0


def test_e2m1_decode_matches_the_ocp_value_table():
    """OCP Microscaling Formats (MX) v1.0, FP4 E2M1: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6
    for codes 0..7; bit 3 is the sign."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        v = oracle.e2m1_value(c)
        assert abs(v) == mags[c & 7] and (np.signbit(v) == bool(c & 8))


def test_fp8_table_is_never_nan_and_has_its_closed_form_spread():
    q, s = oracle.fill_fp8(gen.TABLE_SEED, 5, 200, 512)
    assert not np.any(((q & 0x7F) == 0x7F))                 # no NaN codes
    e = (q >> 3) & 15
    assert e.min() >= 4 and e.max() <= 10
    v = np.array([oracle.e4m3_value(int(c)) for c in q.ravel()[:50000]]) * np.repeat(s, 512)[:50000]
    assert abs(v.std() / 0.02 - 1) < 0.03 and abs(v.mean()) < 4 * 0.02 / np.sqrt(v.size)
    K = float.fromhex("0x1.4dp-8")
    assert np.all(s >= 0.75 * K) and np.all(s < 1.25 * K)


def test_fp4_table_layout_and_spread():
    d = 512
    rows = oracle.fill_fp4(gen.TABLE_SEED, 7, 100, d)
    assert rows.shape == (100, d // 2 + d // 16) and oracle.fp4_row_bytes(256) == 144
    sc = rows[:, d // 2:]
    e = (sc >> 3) & 15
    assert e.min() >= 5 and e.max() <= 9 and not np.any(sc & 0x80)
    codes = np.stack([rows[:, :d // 2] & 15, rows[:, :d // 2] >> 4], axis=2).reshape(100, d)
    counts = np.bincount(codes.ravel(), minlength=16)
    assert counts.min() > 0.8 * codes.size / 16                    # uniform over the 16 codes
    e2 = np.array([oracle.e2m1_value(c) for c in range(16)])
    bs = np.array([[oracle.e4m3_value(int(b)) for b in r] for r in sc])
    v = e2[codes] * np.repeat(bs, 16, axis=1) * oracle.FP4_GLOBAL_SCALE
    assert abs(v.std() / 0.02 - 1) < 0.05


@pytest.mark.parametrize("dtype", [oracle.FP8, oracle.NVFP4])
def test_low_precision_brute_force_and_fp32_mode(dtype):
    R, d, V = 257, 64, 300
    toks, res, g = _tiny_case(R=R, d=d, V=V, n_seq=3, T=30)
    if dtype == oracle.FP8:
        q, s = oracle.fill_fp8(21, 0, R, d)
        E = np.array([[oracle.e4m3_value(int(c)) for c in r] for r in q]) * s[:, None].astype(np.float64)
        tab, sc = q, s
    else:
        rows = oracle.fill_fp4(21, 0, R, d)
        codes = np.stack([rows[:, :d // 2] & 15, rows[:, :d // 2] >> 4], axis=2).reshape(R, d)
        e2 = np.array([oracle.e2m1_value(c) for c in range(16)])
        # value = e2m1 * e4m3(block scale) * global scale, exactly (the sum is scaled once)
        cs = np.array([[oracle.e4m3_value(int(b)) * float(oracle.FP4_GLOBAL_SCALE)
                        for b in r[d // 2:d // 2 + d // 16]] for r in rows], dtype=np.float64)
        E = e2[codes] * np.repeat(cs, 16, axis=1)
        tab, sc = rows, np.array([oracle.FP4_GLOBAL_SCALE], dtype=np.float32)
    out, y, mag, idx = oracle.forward(toks, None, res, g, R=R, d=d, dtype=dtype, table_seed=21,
                                      acc=oracle.ACC_F64, vocab_size=V, want_aux=True)
    e = _one_hot_sum(idx, E)
    r = _bits_to_f64(res).reshape(-1, d)
    assert np.array_equal(y, r + g.astype(np.float64)[None, :] * e)
    # the materialised table gives the same result as regenerating rows
    out_m = oracle.forward(toks, None, res, g, R=R, d=d, dtype=dtype, table_i8=tab, row_scale=sc,
                           acc=oracle.ACC_F64, vocab_size=V)
    assert np.array_equal(out, out_m)
    o32 = oracle.forward(toks, None, res, g, R=R, d=d, dtype=dtype, table_seed=21,
                         acc=oracle.ACC_F32, vocab_size=V)
    a, b = _bits_to_f64(o32).reshape(y.shape), _bits_to_f64(out).reshape(y.shape)
    assert np.all(np.abs(a - b) <= _bf16_ulp(b) + 2.0 ** -20 * mag)


# --------------------------------------------------------------------------- per-token gate, backward
def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _autograd_case(seed, gate_tok, R=61, d=16, V=40, n_seq=2, T=13, nb=5, nt=3):
    """Small batch with a bf16 table: fp64 autograd of L = sum(dy * out) with
    out = r + g * (A E) (A the occurrence counts of the hashed rows)."""
    toks, res, g = _tiny_case(seed=seed, n_seq=n_seq, T=T, V=V, R=R, d=d, nb=nb, nt=nt)
    N = n_seq * T
    rng = np.random.default_rng(seed + 9)
    dy = _bf16_bits(rng.normal(0, 1.0, (N, d)))
    gt = _bf16_bits(rng.normal(0, 1.0, (N, d))) if gate_tok else None
    Eb = oracle.fill_bf16(77, 0, R, d)
    idx = oracle.indices(toks, None, R=R, n_bigram=nb, n_trigram=nt, vocab_size=V).reshape(N, nb + nt)
    E = torch.tensor(_bits_to_f64(Eb).reshape(R, d), requires_grad=True)
    G = torch.tensor(_bits_to_f64(gt).reshape(N, d) if gate_tok else g.astype(np.float64),
                     requires_grad=True)
    e = torch.nn.functional.embedding_bag(torch.from_numpy(idx.astype(np.int64)), E, mode="sum")
    out = torch.tensor(_bits_to_f64(res).reshape(N, d)) + G * e
    (torch.tensor(_bits_to_f64(dy).reshape(N, d)) * out).sum().backward()
    return dict(toks=toks, res=res, g=g, dy=dy, gt=gt, Eb=Eb, idx=idx, R=R, d=d, V=V, nb=nb, nt=nt,
                dE=E.grad.numpy(), dG=G.grad.numpy())


@pytest.mark.parametrize("gate_tok", [False, True])
def test_backward_rows_matches_autograd(gate_tok):
    c = _autograd_case(11, gate_tok)
    kw = dict(R=c["R"], d=c["d"], gate_tok=c["gt"], n_bigram=c["nb"], n_trigram=c["nt"], vocab_size=c["V"])
    uniq, grad = oracle.backward_rows(c["toks"], None, c["dy"], c["g"], acc=oracle.ACC_F64, **kw)
    # the distinct rows in order of first occurrence (flat token-major, head-minor order)
    first = {}
    for r in c["idx"].ravel():
        first.setdefault(int(r), len(first))
    assert list(uniq) == list(first)
    assert np.allclose(grad, c["dE"][uniq], rtol=1e-12, atol=1e-12)
    others = np.setdiff1d(np.arange(c["R"]), uniq)
    assert np.all(c["dE"][others] == 0.0)
    # fp32 mode: within the sequential-sum bound of the exact one
    u32, g32, mag = oracle.backward_rows(c["toks"], None, c["dy"], c["g"], acc=oracle.ACC_F32,
                                         want_mag=True, **kw)
    count = np.bincount(np.searchsorted(np.sort(uniq), c["idx"].ravel()), minlength=len(uniq))
    n_terms = count[np.argsort(np.argsort(uniq))][:, None]
    assert np.array_equal(u32, uniq)
    assert np.all(np.abs(g32 - grad) <= (n_terms + 1) * 2.0 ** -24 * mag + 1e-300)
    # a selection of rows gives those rows
    sel = np.array([len(uniq) - 1, 0, 3])
    _, gs = oracle.backward_rows(c["toks"], None, c["dy"], c["g"], acc=oracle.ACC_F32, sel_u=sel, **kw)
    assert np.array_equal(gs, g32[sel])


def test_backward_rows_closed_form_single_row():
    """R = 1: every occurrence hits row 0, so grad = g * H * sum_t dy[t]; with dy small
    multiples of 2^-4 every fp32 sum is exact and the fp32 mode equals it exactly."""
    n_seq, T, d, V = 2, 9, 8, 30
    rng = np.random.default_rng(5)
    toks = rng.integers(0, V, (n_seq, T)).astype(np.int32)
    dyv = rng.integers(-8, 9, (n_seq * T, d)) / 16.0
    g = np.array([0.5, -1.0, 3.0, 0.25, 1.0, -2.0, 0.125, 7.0], dtype=np.float32)
    uniq, grad = oracle.backward_rows(toks, None, _bf16_bits(dyv), g, R=1, d=d, vocab_size=V)
    assert list(uniq) == [0]
    assert np.array_equal(grad[0], g.astype(np.float64) * 16 * dyv.sum(0))


@pytest.mark.parametrize("gate_tok", [False, True])
def test_backward_gate_matches_autograd(gate_tok):
    c = _autograd_case(12, gate_tok)
    kw = dict(R=c["R"], d=c["d"], dtype=oracle.BF16, table=c["Eb"].reshape(c["R"], c["d"]),
              per_token=gate_tok, n_bigram=c["nb"], n_trigram=c["nt"], vocab_size=c["V"])
    dg = oracle.backward_gate(c["toks"], None, c["dy"], acc=oracle.ACC_F64, **kw)
    assert np.allclose(dg, c["dG"], rtol=1e-12, atol=1e-15)
    dg32, mag = oracle.backward_gate(c["toks"], None, c["dy"], acc=oracle.ACC_F32, want_mag=True, **kw)
    # fp32 head sum (16 roundings) and one rounding of the product / of the fp64 sum
    H = c["nb"] + c["nt"]
    assert np.all(np.abs(dg32 - dg) <= (H + 2) * 2.0 ** -24 * mag + 2.0 ** -24 * np.abs(dg))
    if gate_tok:
        sel = np.array([5, 0, 20])
        part = oracle.backward_gate(c["toks"], None, c["dy"], acc=oracle.ACC_F32, sel=sel, **kw)
        assert np.array_equal(part, dg32[sel])


_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,            # OCP MX v1.0 FP4 E2M1
                  -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def _e4m3_torch(codes):
    """E4M3 codes -> fp64 through torch's float8_e4m3fn (independent of the oracle)."""
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
@pytest.mark.parametrize("gate_tok", [False, True])
def test_backward_gate_low_precision_matches_autograd(fmt, gate_tok):
    """The gate gradient over FP8 and NVFP4 tables: fp64 autograd of sum(dy * out), with
    out = r + G * (A E) and E the table decoded by torch's E4M3 and the OCP E2M1 table."""
    R, d, V, n_seq, T, nb, nt = 61, 32, 40, 2, 13, 5, 3
    toks, res, g = _tiny_case(seed=14, n_seq=n_seq, T=T, V=V, R=R, d=d, nb=nb, nt=nt)
    N = n_seq * T
    rng = np.random.default_rng(23)
    dy = _bf16_bits(rng.normal(0, 1.0, (N, d)))
    gt = _bf16_bits(rng.normal(0, 1.0, (N, d))) if gate_tok else None
    if fmt == "fp8":
        q, sc = oracle.fill_fp8(31, 0, R, d)
        E = _e4m3_torch(q) * sc.astype(np.float64)[:, None]
        dtype, tab = oracle.FP8, q
    else:
        rows = oracle.fill_fp4(31, 0, R, d)
        codes = np.stack([rows[:, :d // 2] & 15, rows[:, :d // 2] >> 4], axis=2).reshape(R, d)
        bs = _e4m3_torch(rows[:, d // 2:d // 2 + d // 16])
        gs = float.fromhex("0x1.4fp-9")
        E = _E2M1[codes] * np.repeat(bs, 16, axis=1) * gs
        sc = np.array([gs], dtype=np.float32)
        dtype, tab = oracle.NVFP4, rows
    idx = oracle.indices(toks, None, R=R, n_bigram=nb, n_trigram=nt, vocab_size=V).reshape(N, nb + nt)
    Et = torch.tensor(E)
    G = torch.tensor(_bits_to_f64(gt).reshape(N, d) if gate_tok else g.astype(np.float64),
                     requires_grad=True)
    e = torch.nn.functional.embedding_bag(torch.from_numpy(idx.astype(np.int64)), Et, mode="sum")
    out = torch.tensor(_bits_to_f64(res).reshape(N, d)) + G * e
    (torch.tensor(_bits_to_f64(dy).reshape(N, d)) * out).sum().backward()
    dg = oracle.backward_gate(toks, None, dy, R=R, d=d, dtype=dtype, table_i8=tab, row_scale=sc,
                              per_token=gate_tok, acc=oracle.ACC_F64, n_bigram=nb, n_trigram=nt,
                              vocab_size=V)
    assert np.allclose(dg, G.grad.numpy(), rtol=1e-12, atol=1e-15)


def test_backward_gate_shared_is_the_sum_of_per_token():
    c = _autograd_case(13, False)
    kw = dict(R=c["R"], d=c["d"], dtype=oracle.BF16, table=c["Eb"].reshape(c["R"], c["d"]),
              n_bigram=c["nb"], n_trigram=c["nt"], vocab_size=c["V"], acc=oracle.ACC_F64)
    shared = oracle.backward_gate(c["toks"], None, c["dy"], per_token=False, **kw)
    per_tok = oracle.backward_gate(c["toks"], None, c["dy"], per_token=True, **kw)
    assert np.allclose(shared, per_tok.sum(0), rtol=1e-13, atol=1e-15)


def test_forward_per_token_gate():
    """A per-token gate whose rows all equal bf16(g) gives the shared-gate result with
    that gate bit for bit; a general one matches r + G * (A E) in fp64."""
    R, d, V = 97, 24, 50
    toks, res, g = _tiny_case(R=R, d=d, V=V)
    N = toks.size
    gb = _bf16_bits(g)
    kw = dict(R=R, d=d, table_seed=3, vocab_size=V)
    a = oracle.forward(toks, None, res, _bits_to_f64(gb).astype(np.float32), **kw)
    b = oracle.forward(toks, None, res, None, gate_tok=np.tile(gb, (N, 1)), **kw)
    assert np.array_equal(a, b)
    G = _bf16_bits(np.random.default_rng(3).normal(0, 1, (N, d)))
    _, y, _, idx = oracle.forward(toks, None, res, None, gate_tok=G, acc=oracle.ACC_F64,
                                  want_aux=True, **kw)
    E = _bits_to_f64(oracle.fill_bf16(3, 0, R, d)).reshape(R, d)
    want = _bits_to_f64(res).reshape(N, d) + _bits_to_f64(G).reshape(N, d) * _one_hot_sum(idx, E)
    assert np.array_equal(y, want)


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_forward_per_token_gate_low_precision(fmt):
    """FP8 / NVFP4 tables: a per-token gate whose rows all equal bf16(g) gives the shared-
    gate result bit for bit (fp32 mode), and a general one matches r + G * (A E) in fp64
    with E decoded by torch's float8_e4m3fn and the OCP E2M1 table."""
    R, d, V = 97, 32, 50
    toks, res, g = _tiny_case(R=R, d=d, V=V)
    N = toks.size
    gb = _bf16_bits(g)
    if fmt == "fp8":
        q, sc = oracle.fill_fp8(5, 0, R, d)
        E = _e4m3_torch(q) * sc.astype(np.float64)[:, None]
        kw = dict(R=R, d=d, dtype=oracle.FP8, table_i8=q, row_scale=sc, vocab_size=V)
    else:
        rows = oracle.fill_fp4(5, 0, R, d)
        codes = np.stack([rows[:, :d // 2] & 15, rows[:, :d // 2] >> 4], axis=2).reshape(R, d)
        gs = float.fromhex("0x1.4fp-9")
        E = _E2M1[codes] * np.repeat(_e4m3_torch(rows[:, d // 2:d // 2 + d // 16]), 16, axis=1) * gs
        kw = dict(R=R, d=d, dtype=oracle.NVFP4, table_i8=rows, row_scale=np.array([gs], np.float32),
                  vocab_size=V)
    a = oracle.forward(toks, None, res, _bits_to_f64(gb).astype(np.float32), **kw)
    b = oracle.forward(toks, None, res, None, gate_tok=np.tile(gb, (N, 1)), **kw)
    assert np.array_equal(a, b)
    G = _bf16_bits(np.random.default_rng(4).normal(0, 1, (N, d)))
    _, y, _, idx = oracle.forward(toks, None, res, None, gate_tok=G, acc=oracle.ACC_F64,
                                  want_aux=True, **kw)
    want = _bits_to_f64(res).reshape(N, d) + _bits_to_f64(G).reshape(N, d) * _one_hot_sum(idx, E)
    assert np.allclose(y, want, rtol=1e-15, atol=0)


def test_hash_rows_are_uniform():
    """Sanity, not parity: 100,000 random contexts x 16 heads land in R = 1009 rows
    uniformly (chi-square with 1008 degrees of freedom, p > 1e-4), and the heads of one
    context are independent of one another (pairwise equal rows at the 1/R rate)."""
    from scipy import stats
    R, V = 1009, 151_936
    rng = np.random.default_rng(123)
    toks = rng.integers(0, V, (1000, 100)).astype(np.int32)
    hist = rng.integers(0, V, (1000, 2)).astype(np.int32)
    idx = oracle.indices(toks, hist, R=R, vocab_size=V).reshape(-1, 16)
    counts = np.bincount(idx.ravel(), minlength=R)
    chi2, p = stats.chisquare(counts)
    assert p > 1e-4, (chi2, p)
    same = np.mean(idx[:, 0] == idx[:, 8])                 # a bigram and a trigram head
    assert abs(same - 1.0 / R) < 5 * np.sqrt(1.0 / R / idx.shape[0])



def test_nvfp4_fp32_mode_scales_the_head_sum_once():
    """NVFP4 in fp32 mode: each head adds q * block scale (exact) with one rounding, and the
    global scale multiplies the sum once.  With gs = 1, r = 0, g = 1 the output is the
    bf16 of the fp32 fma chain over exact products; with gs = 2^k it is that times 2^k."""
    R, d, V = 61, 32, 40
    toks, res, g = _tiny_case(R=R, d=d, V=V)
    N = toks.size
    rows = oracle.fill_fp4(9, 0, R, d)
    idx = oracle.indices(toks, None, R=R, vocab_size=V).reshape(N, 16)
    codes = np.stack([rows[:, :d // 2] & 15, rows[:, :d // 2] >> 4], axis=2).reshape(R, d)
    e2 = np.array([oracle.e2m1_value(c) for c in range(16)], dtype=np.float32)
    bsv = np.array([[oracle.e4m3_value(int(b)) for b in r[d // 2:d // 2 + d // 16]] for r in rows],
                   dtype=np.float32)
    zero = np.zeros(N * d, dtype=np.uint16)
    one = np.ones(d, dtype=np.float32)
    for gs in (1.0, 0.25):
        acc = np.zeros((N, d), dtype=np.float32)
        for h in range(16):                  # fp32 fma chain: q * s exact, one rounding each
            q = e2[codes[idx[:, h]]].astype(np.float64)
            sc = np.repeat(bsv[idx[:, h]], 16, axis=1).astype(np.float64)
            acc = (q * sc + acc.astype(np.float64)).astype(np.float32)
        y = torch.from_numpy((np.float32(gs) * acc).ravel())           # fp32 multiply, rounded once
        want = y.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        got = oracle.forward(toks, None, zero, one, R=R, d=d, dtype=oracle.NVFP4, table_i8=rows,
                             row_scale=np.array([gs], np.float32), acc=oracle.ACC_F32, vocab_size=V)
        assert np.array_equal(got.ravel(), want)
