"""The seeded synthetic inputs follow the recipe the benchmarks state: Zipf(1.1) token ids
over the vocabulary (rank == id), or uniform ones; bf16 residuals of N(0, 1); an fp32 gate
of U(0, 1).  Checked against the closed forms on large samples (CPU only)."""
import numpy as np
import torch
from scipy import stats

import ngram_inputs as gen


def test_zipf_tokens_follow_the_power_law():
    V, s = 151_936, gen.ZIPF_S
    assert s == 1.1
    toks = gen.zipf_tokens(64, 16_384, V, seed=3).ravel()          # 1,048,576 draws
    assert toks.min() >= 0 and toks.max() < V
    p = np.arange(1, V + 1, dtype=np.float64) ** -s
    p /= p.sum()
    counts = np.bincount(toks, minlength=V)
    # the 200 most frequent ranks against their probabilities, the rest pooled
    top = 200
    obs = np.append(counts[:top], counts[top:].sum())
    exp = np.append(p[:top], p[top:].sum()) * toks.size
    chi2, pval = stats.chisquare(obs, exp)
    assert pval > 1e-4, (chi2, pval)
    # the slope of log frequency against log rank over ranks 1..100 is -s
    k = np.arange(1, 101)
    slope = np.polyfit(np.log(k), np.log(counts[:100]), 1)[0]
    assert abs(slope + s) < 0.03, slope


def test_uniform_tokens_are_uniform():
    V = 151_936
    toks = gen.uniform_tokens(16, 4096, V, seed=8).ravel()
    counts = np.bincount(toks // 1187, minlength=128)               # 128 equal bins
    assert stats.chisquare(counts).pvalue > 1e-4


def test_residual_is_bf16_of_standard_normal():
    bits = gen.residual_bf16_bits(4096, 256)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy().ravel()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert stats.kstest(x[:200_000], "norm").pvalue > 1e-4
    # every value is a bf16 (the low 16 bits of its fp32 form are zero)
    assert np.all((x.view(np.uint32) & 0xFFFF) == 0)


def test_gate_is_uniform_on_the_unit_interval():
    g = gen.gate_f32(100_000)
    assert g.dtype == np.float32 and g.min() >= 0.0 and g.max() < 1.0
    assert stats.kstest(g, "uniform").pvalue > 1e-4


def test_inputs_are_seeded():
    w = gen.WORKLOADS["mid"]
    a, b = gen.make_inputs(w), gen.make_inputs(w)
    for k in ("tokens", "residual", "gate"):
        assert np.array_equal(a[k], b[k])
    c = gen.make_inputs(w, token_seed=gen.TOKEN_SEED + 1)
    assert not np.array_equal(a["tokens"], c["tokens"])
