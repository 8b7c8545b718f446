"""Seeded synthetic inputs for the hashed n-gram embedding lookup.

This module is shared by the tests, the benchmark and the oracle checks.  It holds
no step of the method (no hashing, gathering, summing, gating or rounding of
results): only random inputs and the workload sizes.

Workloads follow the sizes the pages give for the table -- "Qwen Brought Back
N-Grams. All 51 Billion Parameters of Them.", "Key Takeaways": 20,000,000 rows of
2560 dims, 16 rows read per token, BF16 -- and the INT8 footprint named in
"Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with Heterogeneous Memory
Prefetch", Key point 3.  The pages print no token stream, so tokens are iid
Zipf(1.1) over a 151,936-id vocabulary (rank == id), a stand-in for natural text.
The table values themselves are not made here: they are a counter-based function of
(seed, row, col) that the CUDA library and the oracle each implement on their own.
"""
from __future__ import annotations

import dataclasses

import numpy as np

TABLE_SEED = 0x5EED0001
TOKEN_SEED = 1
RESIDUAL_SEED = 2
GATE_SEED = 3
HISTORY_SEED = 4
ZIPF_S = 1.1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    R: int                 # table rows
    d: int                 # row width
    dtype: str             # "bf16", "int8", "fp8" (E4M3 + row scale) or "nvfp4"
    vocab: int
    n_seq: int
    T: int
    tokens: str = "zipf"   # "zipf" or "uniform"
    history: bool = False  # decode / chunked prefill pass the two preceding tokens
    residency: str = "hbm" # "hbm" or "host" (table in pinned host memory)

    @property
    def N(self) -> int:
        return self.n_seq * self.T


WORKLOADS = {
    # 65,536 x 256 bf16 table, 4 x 128 Zipf tokens, no history (PAD at t < 2)
    "tiny": Workload("tiny", 65_536, 256, "bf16", 32_000, 4, 128),
    # 2M x 2560 bf16 (9.5 GiB), 8 x 1024 Zipf tokens
    "mid": Workload("mid", 2_000_000, 2560, "bf16", 151_936, 8, 1024),
    # 20M x 2560 bf16 (95.4 GiB), one 32,768-token prefill
    "full_prefill": Workload("full_prefill", 20_000_000, 2560, "bf16", 151_936, 1, 32_768),
    # same table, decode steps: n_seq sequences of one token with two tokens of history
    "full_decode_1": Workload("full_decode_1", 20_000_000, 2560, "bf16", 151_936, 1, 1, history=True),
    "full_decode_16": Workload("full_decode_16", 20_000_000, 2560, "bf16", 151_936, 16, 1, history=True),
    "full_decode_64": Workload("full_decode_64", 20_000_000, 2560, "bf16", 151_936, 64, 1, history=True),
    "full_decode_256": Workload("full_decode_256", 20_000_000, 2560, "bf16", 151_936, 256, 1, history=True),
    # same table in pinned host memory: decode steps and an 8192-token prefill
    "host_decode_1": Workload("host_decode_1", 20_000_000, 2560, "bf16", 151_936, 1, 1, history=True, residency="host"),
    "host_decode_16": Workload("host_decode_16", 20_000_000, 2560, "bf16", 151_936, 16, 1, history=True, residency="host"),
    "host_decode_64": Workload("host_decode_64", 20_000_000, 2560, "bf16", 151_936, 64, 1, history=True, residency="host"),
    "host_decode_256": Workload("host_decode_256", 20_000_000, 2560, "bf16", 151_936, 256, 1, history=True, residency="host"),
    "host_prefill": Workload("host_prefill", 20_000_000, 2560, "bf16", 151_936, 1, 8192, residency="host"),
    # profiling case for full ncu captures: 400k x 2560 bf16 (2 GB), 4 x 2048 Zipf tokens
    "profile_small": Workload("profile_small", 400_000, 2560, "bf16", 151_936, 4, 2048),
    # profiling case for the int8 gather: 1M x 2560 int8 (2.4 GiB), 16 x 1024 uniform tokens
    "profile_int8": Workload("profile_int8", 1_000_000, 2560, "int8", 151_936, 16, 1024, tokens="uniform"),
    # 20M x 2560 int8 + fp32 row scale (47.8 GiB), 65,536 uniform tokens (little reuse)
    "int8_uniform": Workload("int8_uniform", 20_000_000, 2560, "int8", 151_936, 16, 4096, tokens="uniform"),
    # 20M x 2560 FP8 E4M3 + fp32 row scale (47.8 GiB), one 32,768-token Zipf prefill
    "fp8_prefill": Workload("fp8_prefill", 20_000_000, 2560, "fp8", 151_936, 1, 32_768),
    # 20M x 2560 NVFP4, 1,440-byte rows (26.8 GiB), one 32,768-token Zipf prefill
    "nvfp4_prefill": Workload("nvfp4_prefill", 20_000_000, 2560, "nvfp4", 151_936, 1, 32_768),
    # the same tables, 65,536 uniform tokens (little reuse)
    "fp8_uniform": Workload("fp8_uniform", 20_000_000, 2560, "fp8", 151_936, 16, 4096, tokens="uniform"),
    "nvfp4_uniform": Workload("nvfp4_uniform", 20_000_000, 2560, "nvfp4", 151_936, 16, 4096, tokens="uniform"),
    # profiling cases: 1M x 2560 fp8 (2.4 GiB) and 2M x 2560 nvfp4 (2.7 GiB), 16 x 1024 uniform
    "profile_fp8": Workload("profile_fp8", 1_000_000, 2560, "fp8", 151_936, 16, 1024, tokens="uniform"),
    "profile_nvfp4": Workload("profile_nvfp4", 2_000_000, 2560, "nvfp4", 151_936, 16, 1024, tokens="uniform"),
    # small cases of the prefill launch configuration (one 32,768-token Zipf(1.1) batch,
    # grouped order) for ncu counter captures: 400k x 2560 bf16 (2.0 GB), 1M x 2560 FP8
    # (2.6 GB), 2M x 2560 NVFP4 (2.9 GB)
    "profile_prefill": Workload("profile_prefill", 400_000, 2560, "bf16", 151_936, 1, 32_768),
    "profile_fp8_prefill": Workload("profile_fp8_prefill", 1_000_000, 2560, "fp8", 151_936, 1, 32_768),
    "profile_nvfp4_prefill": Workload("profile_nvfp4_prefill", 2_000_000, 2560, "nvfp4", 151_936, 1, 32_768),
}


def zipf_cdf(vocab: int, s: float = ZIPF_S) -> np.ndarray:
    """Cumulative distribution of p(k) ~ k^-s over ranks k = 1..vocab (fp64)."""
    k = np.arange(1, vocab + 1, dtype=np.float64)
    w = k ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def zipf_tokens(n_seq: int, T: int, vocab: int, seed: int, s: float = ZIPF_S) -> np.ndarray:
    """int32 [n_seq][T]; token id = rank - 1, drawn by inverse CDF."""
    u = np.random.default_rng(seed).random(n_seq * T)
    ids = np.searchsorted(zipf_cdf(vocab, s), u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32).reshape(n_seq, T)


def uniform_tokens(n_seq: int, T: int, vocab: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.integers(0, vocab, size=(n_seq, T), dtype=np.int64).astype(np.int32)


def residual_bf16_bits(N: int, d: int, seed: int = RESIDUAL_SEED) -> np.ndarray:
    """N(0,1) residual rows converted to bf16 by torch (CPU), as uint16 bit patterns."""
    import torch
    x = np.random.default_rng(seed).standard_normal((N, d), dtype=np.float32)
    b = torch.from_numpy(x).to(torch.bfloat16)
    return b.view(torch.int16).numpy().view(np.uint16)


def gate_f32(d: int, seed: int = GATE_SEED) -> np.ndarray:
    """Static gate W_g, U(0,1) fp32 [d]."""
    return np.random.default_rng(seed).random(d, dtype=np.float32)


def tokens_for(w: Workload, seed: int = TOKEN_SEED) -> np.ndarray:
    if w.tokens == "uniform":
        return uniform_tokens(w.n_seq, w.T, w.vocab, seed)
    return zipf_tokens(w.n_seq, w.T, w.vocab, seed)


def history_for(w: Workload, seed: int = HISTORY_SEED):
    """int32 [n_seq][2] = (w_-2, w_-1) per sequence, or None when the workload has none."""
    if not w.history:
        return None
    if w.tokens == "uniform":
        return uniform_tokens(w.n_seq, 2, w.vocab, seed)
    return zipf_tokens(w.n_seq, 2, w.vocab, seed)


def make_inputs(w: Workload, token_seed: int = TOKEN_SEED, residual_seed: int = RESIDUAL_SEED,
                gate_seed: int = GATE_SEED, history_seed: int = HISTORY_SEED) -> dict:
    """All host inputs of one workload: tokens, history, residual bits, gate."""
    return {
        "tokens": tokens_for(w, token_seed),
        "history": history_for(w, history_seed),
        "residual": residual_bf16_bits(w.N, w.d, residual_seed),
        "gate": gate_f32(w.d, gate_seed),
    }
