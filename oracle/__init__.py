"""CPU oracle for the hashed n-gram embedding lookup.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The product library
(``hashed_gram_embedding_ngram_b200``) never imports it, and it never imports the
product: the two share no source.  The arithmetic lives in ``ngram_oracle.c`` (plain
scalar C, built with ``-ffp-contract=off``); this module only builds it with gcc and
marshals numpy arrays through ctypes.

Definitions followed (see the header of ``ngram_oracle.c`` for the full text):

* "Qwen Brought Back N-Grams. All 51 Billion Parameters of Them.", section "N-grams,
  of all things": hash the bigram and trigram context, gather 16 rows of one table,
  sum them, add the sum to the residual stream.
* "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with Heterogeneous Memory
  Prefetch", Key point 1: the n-gram vector enters through an elementwise gate W_g.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ngram_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ACC_F64 = 0
ACC_F32 = 1
BF16 = 0
INT8 = 1
FP8 = 2      # FP8 E4M3 codes + fp32 row scale
NVFP4 = 3    # E2M1 codes + E4M3 scale per 16 columns + fp32 global scale
FP4_GLOBAL_SCALE = float.fromhex("0x1.4fp-9")

DEFAULT_BASE_SEED = 0x6E6772616D5F7631   # ASCII "ngram_v1"
DEFAULT_PAD_ID = 0x1FFFFF                # 2^21 - 1, outside any vocabulary below 2^21 - 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ngram_oracle.c into liboracle.so (gcc, OpenMP, no FP contraction)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


class _HashParams(ctypes.Structure):
    _fields_ = [("base_seed", ctypes.c_uint64),
                ("n_bigram_heads", ctypes.c_uint32),
                ("n_trigram_heads", ctypes.c_uint32),
                ("pad_id", ctypes.c_uint32),
                ("vocab_size", ctypes.c_uint32)]


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        u32, u64, i32, i64 = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int32, ctypes.c_int64
        lib.oracle_splitmix64_next.argtypes = [ctypes.POINTER(u64)]
        lib.oracle_splitmix64_next.restype = u64
        lib.oracle_head_seeds.argtypes = [u64, u32, P]
        lib.oracle_philox4x32_10.argtypes = [P, P, P]
        lib.oracle_bf16_from_f32.argtypes = [ctypes.c_float]
        lib.oracle_bf16_from_f32.restype = ctypes.c_uint16
        lib.oracle_bf16_from_f64.argtypes = [ctypes.c_double]
        lib.oracle_bf16_from_f64.restype = ctypes.c_uint16
        lib.oracle_table_bf16.argtypes = [u64, u64, u32]
        lib.oracle_table_bf16.restype = ctypes.c_uint16
        lib.oracle_table_int8.argtypes = [u64, u64, u32]
        lib.oracle_table_int8.restype = ctypes.c_int8
        lib.oracle_row_scale.argtypes = [u64, u64]
        lib.oracle_row_scale.restype = ctypes.c_float
        lib.oracle_fill_bf16.argtypes = [u64, u64, u64, u32, P]
        lib.oracle_fill_int8.argtypes = [u64, u64, u64, u32, P, P]
        lib.oracle_indices.argtypes = [P, P, u32, u32, u64, ctypes.POINTER(_HashParams), P]
        lib.oracle_indices.restype = ctypes.c_int
        lib.oracle_forward.argtypes = [ctypes.c_int, P, P, P, u64, u64, u32,
                                       ctypes.POINTER(_HashParams), P, P, u32, u32, P, P, P,
                                       P, u64, ctypes.c_int, ctypes.c_int, P, P, P, P]
        lib.oracle_forward.restype = ctypes.c_int
        lib.oracle_backward_rows.argtypes = [u64, u32, ctypes.POINTER(_HashParams), P, P, u32, u32,
                                             P, P, P, P, u64, ctypes.c_int, ctypes.c_int, P, P, P]
        lib.oracle_backward_rows.restype = ctypes.c_int64
        lib.oracle_backward_gate.argtypes = [ctypes.c_int, P, P, P, u64, u64, u32,
                                             ctypes.POINTER(_HashParams), P, P, u32, u32, P,
                                             ctypes.c_int, P, u64, ctypes.c_int, ctypes.c_int, P, P]
        lib.oracle_backward_gate.restype = ctypes.c_int
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_fill_fp8.argtypes = [u64, u64, u64, u32, P, P]
        lib.oracle_fill_fp4.argtypes = [u64, u64, u64, u32, P]
        lib.oracle_fp4_row_bytes.argtypes = [u32]
        lib.oracle_fp4_row_bytes.restype = u32
        del i32, i64
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _hp(base_seed=DEFAULT_BASE_SEED, n_bigram=8, n_trigram=8, pad_id=DEFAULT_PAD_ID,
        vocab_size=DEFAULT_PAD_ID):
    return _HashParams(base_seed & (2**64 - 1), n_bigram, n_trigram, pad_id, vocab_size)


# --------------------------------------------------------------------------- generators
def splitmix64_outputs(seed: int, n: int) -> list[int]:
    lib = _load()
    st = ctypes.c_uint64(seed & (2**64 - 1))
    return [int(lib.oracle_splitmix64_next(ctypes.byref(st))) for _ in range(n)]


def head_seeds(base_seed: int, n_heads: int) -> np.ndarray:
    out = np.zeros(n_heads, dtype=np.uint64)
    _load().oracle_head_seeds(base_seed & (2**64 - 1), n_heads, _ptr(out))
    return out


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    o = np.zeros(4, dtype=np.uint32)
    _load().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(o))
    return o


def bf16_from_f32(x: float) -> int:
    return int(_load().oracle_bf16_from_f32(float(x)))


def bf16_from_f64(x: float) -> int:
    return int(_load().oracle_bf16_from_f64(float(x)))


def table_bf16(seed: int, row: int, col: int) -> int:
    return int(_load().oracle_table_bf16(seed, row, col))


def fill_bf16(seed: int, row0: int, n_rows: int, d: int) -> np.ndarray:
    """Rows [row0, row0+n_rows) of the synthetic bf16 table, as uint16 bit patterns."""
    out = np.zeros((n_rows, d), dtype=np.uint16)
    _load().oracle_fill_bf16(seed, row0, n_rows, d, _ptr(out))
    return out


def fill_int8(seed: int, row0: int, n_rows: int, d: int):
    """Rows of the synthetic int8 table and their fp32 row scales."""
    q = np.zeros((n_rows, d), dtype=np.int8)
    s = np.zeros(n_rows, dtype=np.float32)
    _load().oracle_fill_int8(seed, row0, n_rows, d, _ptr(q), _ptr(s))
    return q, s


def e4m3_value(code: int) -> float:
    return float(_load().oracle_e4m3_value(code))


def e2m1_value(nibble: int) -> float:
    return float(_load().oracle_e2m1_value(nibble))


def fp4_row_bytes(d: int) -> int:
    return int(_load().oracle_fp4_row_bytes(d))


def fill_fp8(seed: int, row0: int, n_rows: int, d: int):
    """Rows of the synthetic FP8 E4M3 table (uint8 codes) and their fp32 row scales."""
    q = np.zeros((n_rows, d), dtype=np.uint8)
    s = np.zeros(n_rows, dtype=np.float32)
    _load().oracle_fill_fp8(seed, row0, n_rows, d, _ptr(q), _ptr(s))
    return q, s


def fill_fp4(seed: int, row0: int, n_rows: int, d: int) -> np.ndarray:
    """Rows of the synthetic NVFP4 table as bytes: d/2 code bytes then the block scales."""
    out = np.zeros((n_rows, fp4_row_bytes(d)), dtype=np.uint8)
    _load().oracle_fill_fp4(seed, row0, n_rows, d, _ptr(out))
    return out


def rows_bf16(seed: int, rows, d: int) -> np.ndarray:
    """Selected rows (any order, repeats allowed) of the synthetic bf16 table."""
    rows = np.asarray(rows, dtype=np.uint64).ravel()
    out = np.zeros((rows.size, d), dtype=np.uint16)
    for i, r in enumerate(rows):
        out[i] = fill_bf16(seed, int(r), 1, d)[0]
    return out


# --------------------------------------------------------------------------- the method
def indices(tokens, history, R, *, base_seed=DEFAULT_BASE_SEED, n_bigram=8, n_trigram=8,
            pad_id=DEFAULT_PAD_ID, vocab_size=DEFAULT_PAD_ID) -> np.ndarray:
    """Row indices [N][H] uint32 for tokens [n_seq][T] (history [n_seq][2] or None)."""
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    if tok.ndim == 1:
        tok = tok[None, :]
    n_seq, T = tok.shape
    hist = None if history is None else np.ascontiguousarray(history, dtype=np.int32)
    H = n_bigram + n_trigram
    out = np.zeros((n_seq * T, H), dtype=np.uint32)
    hp = _hp(base_seed, n_bigram, n_trigram, pad_id, vocab_size)
    rc = _load().oracle_indices(_ptr(tok), _ptr(hist), n_seq, T, R, ctypes.byref(hp), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_indices: bad arguments")
    return out


def unique_rows(idx):
    """Per-batch dedup of the gathered rows (the optional dedup step of the lookup):
    the distinct row ids of the flattened [N][H] index array in order of first
    appearance, and for every entry the position of its row in that list.  Every entry
    keeps its own inverse slot, so colliding heads still contribute once each."""
    flat = np.asarray(idx, dtype=np.uint32).ravel()
    where = {}
    uniq = []
    inv = np.empty(flat.size, dtype=np.uint32)
    for i, r in enumerate(flat.tolist()):
        u = where.get(r)
        if u is None:
            u = len(uniq)
            where[r] = u
            uniq.append(r)
        inv[i] = u
    return np.array(uniq, dtype=np.uint32), inv


def forward(tokens, history, residual_bits, gate, *, R, d, dtype=BF16, table_seed=None,
            table=None, table_i8=None, row_scale=None, sel=None, acc=ACC_F32, n_threads=1,
            base_seed=DEFAULT_BASE_SEED, n_bigram=8, n_trigram=8, pad_id=DEFAULT_PAD_ID,
            vocab_size=DEFAULT_PAD_ID, want_aux=False, gate_tok=None):
    """Gated gather-sum for the selected tokens.

    residual_bits: [N][d] uint16 (bf16 bit patterns); gate: [d] float32, or (gate_tok)
    a per-token gate [N][d] uint16 (bf16 bit patterns), in which case gate is unused.
    Rows come from ``table`` (uint16 [R][d]) / ``table_i8`` + ``row_scale`` if given,
    otherwise they are regenerated from ``table_seed``.
    Returns out bits [n_sel][d] uint16, and with want_aux also (y, mag, idx).
    """
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    if tok.ndim == 1:
        tok = tok[None, :]
    n_seq, T = tok.shape
    N = n_seq * T
    hist = None if history is None else np.ascontiguousarray(history, dtype=np.int32)
    res = np.ascontiguousarray(residual_bits, dtype=np.uint16).reshape(N, d)
    g = None if gate is None else np.ascontiguousarray(gate, dtype=np.float32).reshape(d)
    if g is None and gate_tok is None:
        raise ValueError("need gate or gate_tok")
    sel_a = None if sel is None else np.ascontiguousarray(sel, dtype=np.int64).ravel()
    n_sel = N if sel_a is None else sel_a.size
    if table is None and table_i8 is None and table_seed is None:
        raise ValueError("need a table or a table_seed")
    tb = None if table is None else np.ascontiguousarray(table, dtype=np.uint16)
    ti = None if table_i8 is None else np.ascontiguousarray(table_i8).view(np.int8)
    sc = None if row_scale is None else np.ascontiguousarray(row_scale, dtype=np.float32)
    gt = None if gate_tok is None else np.ascontiguousarray(gate_tok, dtype=np.uint16).reshape(N, d)
    H = n_bigram + n_trigram
    out = np.zeros((n_sel, d), dtype=np.uint16)
    y = np.zeros((n_sel, d), dtype=np.float64) if want_aux else None
    mag = np.zeros((n_sel, d), dtype=np.float64) if want_aux else None
    idx = np.zeros((n_sel, H), dtype=np.uint32) if want_aux else None
    hp = _hp(base_seed, n_bigram, n_trigram, pad_id, vocab_size)
    rc = _load().oracle_forward(dtype, _ptr(tb), _ptr(ti), _ptr(sc),
                                (table_seed or 0) & (2**64 - 1), R, d, ctypes.byref(hp),
                                _ptr(tok), _ptr(hist), n_seq, T, _ptr(res), _ptr(g), _ptr(gt),
                                _ptr(sel_a), n_sel, acc, n_threads,
                                _ptr(out), _ptr(y), _ptr(mag), _ptr(idx))
    if rc != 0:
        raise ValueError("oracle_forward: bad arguments")
    if want_aux:
        return out, y, mag, idx
    return out


def backward_rows(tokens, history, dy_bits, gate, *, R, d, gate_tok=None, sel_u=None,
                  acc=ACC_F32, n_threads=1, base_seed=DEFAULT_BASE_SEED, n_bigram=8,
                  n_trigram=8, pad_id=DEFAULT_PAD_ID, vocab_size=DEFAULT_PAD_ID, want_mag=False):
    """Gradient with respect to the table rows the batch read.

    dy_bits: [N][d] uint16 (bf16 bits of dL/dout); gate: [d] float32, or gate_tok [N][d]
    uint16.  Returns (uniq [U] uint32 in order of first occurrence, grad [n_sel][d] fp64
    for the positions sel_u of that list (all U if None)[, mag])."""
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    if tok.ndim == 1:
        tok = tok[None, :]
    n_seq, T = tok.shape
    N = n_seq * T
    H = n_bigram + n_trigram
    hist = None if history is None else np.ascontiguousarray(history, dtype=np.int32)
    dyb = np.ascontiguousarray(dy_bits, dtype=np.uint16).reshape(N, d)
    g = None if gate is None else np.ascontiguousarray(gate, dtype=np.float32).reshape(d)
    gt = None if gate_tok is None else np.ascontiguousarray(gate_tok, dtype=np.uint16).reshape(N, d)
    if g is None and gt is None:
        raise ValueError("need gate or gate_tok")
    uniq = np.zeros(max(1, N * H), dtype=np.uint32)
    if sel_u is None:
        # U is not known before the call: size for the largest possible U
        n_sel, sel_a = N * H, None
    else:
        sel_a = np.ascontiguousarray(sel_u, dtype=np.int64).ravel()
        n_sel = sel_a.size
    grad = np.zeros((n_sel, d), dtype=np.float64)
    mag = np.zeros((n_sel, d), dtype=np.float64) if want_mag else None
    hp = _hp(base_seed, n_bigram, n_trigram, pad_id, vocab_size)
    U = _load().oracle_backward_rows(R, d, ctypes.byref(hp), _ptr(tok), _ptr(hist), n_seq, T,
                                     _ptr(dyb), _ptr(g), _ptr(gt), _ptr(sel_a), n_sel, acc,
                                     n_threads, _ptr(uniq), _ptr(grad), _ptr(mag))
    if U < 0:
        raise ValueError("oracle_backward_rows: bad arguments")
    if sel_u is None:
        grad = grad[:U]
        mag = None if mag is None else mag[:U]
    uniq = uniq[:U]
    return (uniq, grad, mag) if want_mag else (uniq, grad)


def backward_gate(tokens, history, dy_bits, *, R, d, dtype=BF16, table_seed=None, table=None,
                  table_i8=None, row_scale=None, per_token=False, sel=None, acc=ACC_F32,
                  n_threads=1, base_seed=DEFAULT_BASE_SEED, n_bigram=8, n_trigram=8,
                  pad_id=DEFAULT_PAD_ID, vocab_size=DEFAULT_PAD_ID, want_mag=False):
    """Gradient with respect to the gate: [d] (shared gate, every token summed) or
    [n_sel][d] (per-token gate, the tokens in sel, all if None); fp64 values."""
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    if tok.ndim == 1:
        tok = tok[None, :]
    n_seq, T = tok.shape
    N = n_seq * T
    hist = None if history is None else np.ascontiguousarray(history, dtype=np.int32)
    dyb = np.ascontiguousarray(dy_bits, dtype=np.uint16).reshape(N, d)
    if table is None and table_i8 is None and table_seed is None:
        raise ValueError("need a table or a table_seed")
    tb = None if table is None else np.ascontiguousarray(table, dtype=np.uint16)
    ti = None if table_i8 is None else np.ascontiguousarray(table_i8).view(np.int8)
    sc = None if row_scale is None else np.ascontiguousarray(row_scale, dtype=np.float32)
    sel_a = None if (sel is None or not per_token) else np.ascontiguousarray(sel, dtype=np.int64).ravel()
    rows = (N if sel_a is None else sel_a.size) if per_token else 1
    out = np.zeros((rows, d), dtype=np.float64)
    mag = np.zeros((rows, d), dtype=np.float64) if want_mag else None
    hp = _hp(base_seed, n_bigram, n_trigram, pad_id, vocab_size)
    rc = _load().oracle_backward_gate(dtype, _ptr(tb), _ptr(ti), _ptr(sc),
                                      (table_seed or 0) & (2**64 - 1), R, d, ctypes.byref(hp),
                                      _ptr(tok), _ptr(hist), n_seq, T, _ptr(dyb), int(per_token),
                                      _ptr(sel_a), 0 if sel_a is None else sel_a.size, acc,
                                      n_threads, _ptr(out), _ptr(mag))
    if rc != 0:
        raise ValueError("oracle_backward_gate: bad arguments")
    if not per_token:
        out = out[0]
        mag = None if mag is None else mag[0]
    return (out, mag) if want_mag else out
