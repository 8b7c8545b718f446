"""Helpers for the GPU parity tests: moving seeded inputs to the device, the parity
tolerance, and a cache that keeps one synthetic table on the device at a time.

Tolerance (the stated bar for outputs): |gpu - ref| <= 1 bf16 ulp of ref, where ref
is the oracle's fp32-accumulated result.  Against the oracle's exact (fp64) mode an
absolute slack of 2^-20 * (|r| + |g| * sum_h |E_h|) is added: that is where
cancellation brings y near zero and the fp32 rounding error of the sum (at most
~16 * 2^-24 of that magnitude) can move the bf16 result by more than one ulp.
"""
from __future__ import annotations

import gc
import os

import numpy as np
import torch

import ngram_inputs as gen

N_CPU = os.cpu_count() or 1


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    v = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    return np.where(v > 0, np.exp2(np.maximum(e - 7, -133)), 2.0 ** -133)


def parity_report(got_bits, want_bits, mag=None) -> dict:
    g = bits_to_f64(got_bits).ravel()
    w = bits_to_f64(want_bits).ravel()
    tol = bf16_ulp(w)
    slack = 0.0 if mag is None else (2.0 ** -20) * np.asarray(mag, dtype=np.float64).ravel()
    diff = np.abs(g - w)
    within_ulp = diff <= tol
    ok = diff <= tol + slack
    return {
        "n": int(g.size),
        "exact": int((np.asarray(got_bits).ravel() == np.asarray(want_bits).ravel()).sum()),
        "bad": int((~ok).sum()),
        "needed_slack": int((ok & ~within_ulp).sum()),
        "max_ulps": float(np.max(diff / tol)) if g.size else 0.0,
    }


def assert_parity(got_bits, want_bits, mag=None):
    r = parity_report(got_bits, want_bits, mag)
    assert r["bad"] == 0, r
    return r


def to_dev_tokens(a, dev):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)


def to_dev_bf16(bits, dev):
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(dev)


def from_dev_bf16(t) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class TableCache:
    """Keeps at most one large synthetic table on the device (the full one is 102 GB)."""

    def __init__(self):
        self.key = None
        self.table = None
        self.scale = None

    def get(self, R, d, dtype, seed, dev):
        import hashed_gram_embedding_ngram_b200 as ng
        key = (R, d, dtype, seed)
        if self.key == key:
            return self.table, self.scale
        self.drop()
        if dtype == ng.NGRAM_BF16:
            table = torch.empty((R, d), dtype=torch.bfloat16, device=dev)
            scale = None
        elif dtype == ng.NGRAM_INT8_ROWSCALE:
            table = torch.empty((R, d), dtype=torch.int8, device=dev)
            scale = torch.empty((R,), dtype=torch.float32, device=dev)
        elif dtype == ng.NGRAM_FP8_E4M3_ROWSCALE:
            table = torch.empty((R, d), dtype=torch.uint8, device=dev)
            scale = torch.empty((R,), dtype=torch.float32, device=dev)
        else:                                   # NVFP4: row bytes, one global scale
            table = torch.empty((R, ng.ngram_row_bytes(dtype, d)), dtype=torch.uint8, device=dev)
            scale = torch.empty((1,), dtype=torch.float32, device=dev)
        ng.ngram_fill_synthetic(table, R, d, dtype, seed, row_scale=scale)
        torch.cuda.synchronize()
        self.key, self.table, self.scale = key, table, scale
        return table, scale

    def drop(self):
        self.key = self.table = self.scale = None
        gc.collect()
        torch.cuda.empty_cache()


TABLES = TableCache()


def ng_dtype(name: str) -> int:
    import hashed_gram_embedding_ngram_b200 as ng
    return {"bf16": ng.NGRAM_BF16, "int8": ng.NGRAM_INT8_ROWSCALE,
            "fp8": ng.NGRAM_FP8_E4M3_ROWSCALE, "nvfp4": ng.NGRAM_NVFP4}[name]


def oracle_dtype(name: str) -> int:
    import oracle
    return {"bf16": oracle.BF16, "int8": oracle.INT8, "fp8": oracle.FP8, "nvfp4": oracle.NVFP4}[name]


def workload_on_device(w, dev, token_seed=gen.TOKEN_SEED):
    inp = gen.make_inputs(w, token_seed=token_seed)
    return inp, {
        "tokens": to_dev_tokens(inp["tokens"], dev),
        "history": to_dev_tokens(inp["history"], dev),
        "residual": to_dev_bf16(inp["residual"], dev).view(w.N, w.d),
        "gate": torch.from_numpy(inp["gate"]).to(dev),
    }


def sample_tokens(w, n, seed=0) -> np.ndarray:
    """Flat token ids to check at full size: the first two and last positions of every
    sequence (pad / history boundaries and the ragged tail) plus a seeded sample."""
    N = w.N
    if N <= n:
        return np.arange(N, dtype=np.int64)
    must = []
    for s in range(min(w.n_seq, 64)):
        must += [s * w.T, s * w.T + min(1, w.T - 1), s * w.T + w.T - 1]
    rng = np.random.default_rng(seed)
    extra = rng.choice(N, size=max(0, n - len(must)), replace=False)
    return np.unique(np.concatenate([np.array(must, dtype=np.int64), extra]))
