"""ctypes binding of libngram.so: argument marshalling only.

Each function has the name of the C entry point it calls (include/ngram.h) and does
nothing but check tensor shapes, dtypes, devices and contiguity, take raw pointers
and the CUDA stream handle, and turn a non-OK status into an exception.  Every step
of the lookup runs in the library's kernels; there is no Python or CPU fallback: if
libngram.so is missing, importing this package fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libngram.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libngram.so is not built (expected at %s); build it with "
        "`python hashed_gram_embedding_ngram_b200/build.py`" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

# ngram_status
NGRAM_OK, NGRAM_EINVAL, NGRAM_ENOMEM, NGRAM_ECUDA = 0, 1, 2, 3
NGRAM_EUNSUPPORTED, NGRAM_ETIMEOUT, NGRAM_EDEVICE = 4, 5, 6
# ngram_dtype
NGRAM_BF16, NGRAM_INT8_ROWSCALE, NGRAM_FP8_E4M3_ROWSCALE, NGRAM_NVFP4 = 0, 1, 2, 3
# ngram_residency
NGRAM_RES_HBM, NGRAM_RES_HOST_UVA, NGRAM_RES_HOST_DMA, NGRAM_RES_HOST_AUTO = 0, 1, 2, 3
NGRAM_AUTO_UVA_DEDUP = 4      # ngram_auto_choice: HOST_UVA with NGRAM_FLAG_DEDUP

NGRAM_FLAG_DEDUP = 0x1
NGRAM_FLAG_TMA_STAGING = 0x2
NGRAM_FLAG_SORT = 0x4
NGRAM_FLAG_BATCH_ORDER = 0x8
NGRAM_FLAG_TOKEN_GATE = 0x10
NGRAM_SORT_MIN_TOKENS = 16384
NGRAM_STAGE_SLOTS = 2

MAX_HEADS = 16
DEFAULT_BASE_SEED = 0x6E6772616D5F7631
DEFAULT_PAD_ID = 0x1FFFFF


class NgramError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (ngram_status_string(status), message))
        self.status = status


class HashParams(ctypes.Structure):
    _fields_ = [("base_seed", ctypes.c_uint64),
                ("n_bigram_heads", ctypes.c_uint32),
                ("n_trigram_heads", ctypes.c_uint32),
                ("pad_id", ctypes.c_uint32),
                ("vocab_size", ctypes.c_uint32),
                ("flags", ctypes.c_uint32),
                ("reserved", ctypes.c_uint32)]


_P = ctypes.c_void_p
_u32, _u64, _i32 = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int

_lib.ngram_default_hash_params.argtypes = [ctypes.POINTER(HashParams)]
_lib.ngram_default_hash_params.restype = _i32
_lib.ngram_init.argtypes = [ctypes.POINTER(_P), _P, _P, _u64, _u32, _i32, _i32,
                            ctypes.POINTER(HashParams), _u32]
_lib.ngram_init.restype = _i32
_lib.ngram_forward.argtypes = [_P, _P, _P, _u32, _u32, _P, _P, _P, _P]
_lib.ngram_forward.restype = _i32
_lib.ngram_hash_indices.argtypes = [_P, _P, _P, _u32, _u32, _P, _P]
_lib.ngram_hash_indices.restype = _i32
_lib.ngram_fill_synthetic.argtypes = [_P, _P, _u64, _u32, _i32, _u64, _P]
_lib.ngram_fill_synthetic.restype = _i32
_lib.ngram_get_device_error.argtypes = [_P, _P, _i32]
_lib.ngram_get_device_error.restype = _i32
_lib.ngram_last_error.argtypes = []
_lib.ngram_last_error.restype = ctypes.c_char_p
_lib.ngram_status_string.argtypes = [_i32]
_lib.ngram_status_string.restype = ctypes.c_char_p
_lib.ngram_destroy.argtypes = [_P]
_lib.ngram_destroy.restype = None
_lib.ngram_forward_host.argtypes = [_P, _P, _P, _u32, _u32, _P, _P, _P, _P]
_lib.ngram_forward_host.restype = _i32
_lib.ngram_prefetch.argtypes = [_P, _u32, _P, _P, _u32, _u32, _P]
_lib.ngram_prefetch.restype = _i32
_lib.ngram_forward_staged.argtypes = [_P, _u32, _P, _P, _P, _P]
_lib.ngram_forward_staged.restype = _i32
_lib.ngram_host_alloc.argtypes = [ctypes.POINTER(_P), _u64]
_lib.ngram_host_alloc.restype = _i32
_lib.ngram_host_free.argtypes = [_P]
_lib.ngram_host_free.restype = _i32
_lib.ngram_set_wait_timeout.argtypes = [_P, _u32]
_lib.ngram_set_wait_timeout.restype = _i32
_lib.ngram_auto_choice.argtypes = [_P, _u32, ctypes.POINTER(ctypes.c_int)]
_lib.ngram_auto_choice.restype = _i32
_lib.ngram_dedup_rows.argtypes = [_P, _P, _P, _u32, _u32, _P, _P, _P, _P]
_lib.ngram_dedup_rows.restype = _i32
_lib.ngram_row_bytes.argtypes = [_i32, _u32, ctypes.POINTER(_u32)]
_lib.ngram_row_bytes.restype = _i32
_lib.ngram_backward_rows.argtypes = [_P, _P, _P, _u32, _u32, _P, _P, _P, _P, _P, _P]
_lib.ngram_backward_rows.restype = _i32
_lib.ngram_backward_gate.argtypes = [_P, _P, _P, _u32, _u32, _P, _P, _P]
_lib.ngram_backward_gate.restype = _i32
_lib.ngram_fill_synthetic_cols.argtypes = [_P, _P, _u64, _u32, _u32, _i32, _u64, _P]
_lib.ngram_fill_synthetic_cols.restype = _i32
_lib.ngram_forward_shard.argtypes = [_P, _P, _P, _u32, _u32, _u32, _u32, _P, _P, _P, _u32, _P]
_lib.ngram_forward_shard.restype = _i32
_lib.ngram_device_alloc.argtypes = [ctypes.POINTER(_P), _u64]
_lib.ngram_device_alloc.restype = _i32
_lib.ngram_device_free.argtypes = [_P]
_lib.ngram_device_free.restype = _i32
_lib.ngram_ipc_get_handle.argtypes = [_P, ctypes.c_char_p]
_lib.ngram_ipc_get_handle.restype = _i32
_lib.ngram_ipc_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(_P)]
_lib.ngram_ipc_open.restype = _i32
_lib.ngram_ipc_close.argtypes = [_P]
_lib.ngram_ipc_close.restype = _i32
_lib.ngram_selftest_wait_timeout.argtypes = [_P, _u32, _P]
_lib.ngram_selftest_wait_timeout.restype = _i32


def lib() -> ctypes.CDLL:
    """The loaded libngram.so handle."""
    return _lib


def ngram_status_string(status: int) -> str:
    return _lib.ngram_status_string(status).decode()


def ngram_last_error() -> str:
    return _lib.ngram_last_error().decode()


def _check(status: int) -> None:
    if status != NGRAM_OK:
        raise NgramError(status, ngram_last_error())


def ngram_default_hash_params(**overrides) -> HashParams:
    hp = HashParams()
    _check(_lib.ngram_default_hash_params(ctypes.byref(hp)))
    for k, v in overrides.items():
        setattr(hp, k, v)
    return hp


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _need(t, name, dtype, device=None, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if device is not None and t.device != device:
        raise ValueError("%s must be on %s, got %s" % (name, device, t.device))
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims, got %d" % (name, ndim, t.dim()))


class Context:
    """An ngram_ctx handle; keeps the table tensors alive while it lives."""

    def __init__(self, handle, table, row_scale, R, d, dtype, residency, hp, max_tokens):
        self.handle = handle
        self.table, self.row_scale = table, row_scale
        self.R, self.d, self.dtype, self.residency = R, d, dtype, residency
        self.hp, self.max_tokens = hp, max_tokens
        self.n_heads = hp.n_bigram_heads + hp.n_trigram_heads

    def close(self):
        if self.handle:
            ngram_destroy(self)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def ngram_row_bytes(dtype: int, d: int) -> int:
    out = ctypes.c_uint32()
    _check(_lib.ngram_row_bytes(dtype, d, ctypes.byref(out)))
    return out.value


def ngram_init(table: torch.Tensor, R: int, d: int, dtype: int = NGRAM_BF16,
               where: int = NGRAM_RES_HBM, hp: HashParams | None = None,
               max_tokens: int = 65536, row_scale: torch.Tensor | None = None) -> Context:
    if hp is None:
        hp = ngram_default_hash_params()
    handle = ctypes.c_void_p()
    _check(_lib.ngram_init(ctypes.byref(handle), _ptr(table), _ptr(row_scale), R, d, dtype,
                           where, ctypes.byref(hp), max_tokens))
    return Context(handle.value, table, row_scale, R, d, dtype, where, hp, max_tokens)


def _token_gate(ctx: Context) -> bool:
    return bool(ctx.hp.flags & NGRAM_FLAG_TOKEN_GATE)


def _check_gate(ctx: Context, gate: torch.Tensor, N: int, dev) -> None:
    """fp32 [d], or bf16 [N][d] for a context made with NGRAM_FLAG_TOKEN_GATE."""
    if _token_gate(ctx):
        _need(gate, "gate", torch.bfloat16, dev)
        if gate.numel() != N * ctx.d:
            raise ValueError("a per-token gate must hold N * d = %d elements" % (N * ctx.d))
    else:
        _need(gate, "gate", torch.float32, dev)
        if gate.numel() != ctx.d:
            raise ValueError("gate must hold d = %d elements" % ctx.d)


def ngram_forward(ctx: Context, tokens: torch.Tensor, residual: torch.Tensor,
                  gate: torch.Tensor, out: torch.Tensor | None = None,
                  history: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out = residual + gate * sum of the 16 hashed rows (bf16).  tokens int32
    [n_seq][T]; residual bf16 [N][d]; gate fp32 [d]; history int32 [n_seq][2] or None;
    out bf16 [N][d] (allocated if None; may be residual itself)."""
    dev = tokens.device
    _need(tokens, "tokens", torch.int32, ndim=2)
    n_seq, T = tokens.shape
    N = n_seq * T
    _need(residual, "residual", torch.bfloat16, dev)
    if residual.numel() != N * ctx.d:
        raise ValueError("residual must hold N * d = %d elements" % (N * ctx.d))
    _check_gate(ctx, gate, N, dev)
    if history is not None:
        _need(history, "history", torch.int32, dev, ndim=2)
        if tuple(history.shape) != (n_seq, 2):
            raise ValueError("history must be [n_seq][2]")
    if out is None:
        out = torch.empty_like(residual)
    _need(out, "out", torch.bfloat16, dev)
    if out.numel() != N * ctx.d:
        raise ValueError("out must hold N * d elements")
    _check(_lib.ngram_forward(ctx.handle, _ptr(tokens), _ptr(history), n_seq, T,
                              _ptr(residual), _ptr(gate), _ptr(out), _stream(stream)))
    return out


def ngram_forward_host(ctx: Context, tokens: torch.Tensor, residual: torch.Tensor,
                       gate: torch.Tensor, out: torch.Tensor | None = None,
                       history: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """ngram_forward with tokens, history, residual and out in host (CPU, ideally pinned)
    memory and the gate on the device.  Returns out; it is complete once `stream` (the
    current stream by default) is synchronised."""
    cpu = torch.device("cpu")
    _need(tokens, "tokens", torch.int32, cpu, ndim=2)
    n_seq, T = tokens.shape
    N = n_seq * T
    _need(residual, "residual", torch.bfloat16, cpu)
    if residual.numel() != N * ctx.d:
        raise ValueError("residual must hold N * d = %d elements" % (N * ctx.d))
    _need(gate, "gate", torch.float32)
    if gate.device.type != "cuda" or gate.numel() != ctx.d:
        raise ValueError("gate must be a CUDA tensor of d = %d elements" % ctx.d)
    if history is not None:
        _need(history, "history", torch.int32, cpu, ndim=2)
        if tuple(history.shape) != (n_seq, 2):
            raise ValueError("history must be [n_seq][2]")
    if out is None:
        out = torch.empty_like(residual, pin_memory=True)
    _need(out, "out", torch.bfloat16, cpu)
    if out.numel() != N * ctx.d:
        raise ValueError("out must hold N * d elements")
    _check(_lib.ngram_forward_host(ctx.handle, _ptr(tokens), _ptr(history), n_seq, T,
                                   _ptr(residual), _ptr(gate), _ptr(out), _stream(stream)))
    return out


def ngram_hash_indices(ctx: Context, tokens: torch.Tensor, history: torch.Tensor | None = None,
                       idx_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Row indices [N][H] (int32 tensor holding uint32 values) of every token and head."""
    _need(tokens, "tokens", torch.int32, ndim=2)
    n_seq, T = tokens.shape
    if history is not None:
        _need(history, "history", torch.int32, tokens.device, ndim=2)
    if idx_out is None:
        idx_out = torch.empty((n_seq * T, ctx.n_heads), dtype=torch.int32, device=tokens.device)
    _need(idx_out, "idx_out", torch.int32, tokens.device)
    _check(_lib.ngram_hash_indices(ctx.handle, _ptr(tokens), _ptr(history), n_seq, T,
                                   _ptr(idx_out), _stream(stream)))
    return idx_out


def ngram_fill_synthetic(table: torch.Tensor, R: int, d: int, dtype: int = NGRAM_BF16,
                         seed: int = 0, row_scale: torch.Tensor | None = None,
                         stream=None) -> None:
    _check(_lib.ngram_fill_synthetic(_ptr(table), _ptr(row_scale), R, d, dtype,
                                     seed & (2**64 - 1), _stream(stream)))


def ngram_get_device_error(ctx: Context, clear: bool = True):
    """(status, [flag, position, bad id, 0]); synchronises the device."""
    info = (ctypes.c_uint32 * 4)()
    st = _lib.ngram_get_device_error(ctx.handle, info, 1 if clear else 0)
    if st not in (NGRAM_OK, NGRAM_EDEVICE):
        _check(st)
    return st, list(info)


def ngram_destroy(ctx: Context) -> None:
    if ctx.handle:
        _lib.ngram_destroy(ctx.handle)
        ctx.handle = None


class HostTable:
    """Pinned, device-mapped host memory from ngram_host_alloc, viewed as a torch CPU
    tensor (no copy).  The view must not outlive close()."""

    def __init__(self, shape, dtype: torch.dtype):
        n = 1
        for x in shape:
            n *= int(x)
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.ptr = ngram_host_alloc(self.nbytes)
        buf = (ctypes.c_uint8 * self.nbytes).from_address(self.ptr)
        self.tensor = torch.frombuffer(buf, dtype=torch.uint8).view(dtype).view(*shape)

    def close(self):
        if self.ptr:
            self.tensor = None
            ngram_host_free(self.ptr)
            self.ptr = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def ngram_host_alloc(nbytes: int) -> int:
    """Address of nbytes of pinned, device-mapped host memory."""
    p = ctypes.c_void_p()
    _check(_lib.ngram_host_alloc(ctypes.byref(p), nbytes))
    return p.value


def ngram_host_free(ptr: int) -> None:
    _check(_lib.ngram_host_free(ctypes.c_void_p(ptr)))


def ngram_set_wait_timeout(ctx: Context, ms: int) -> None:
    _check(_lib.ngram_set_wait_timeout(ctx.handle, ms))


def ngram_auto_choice(ctx: Context, n_tokens: int) -> int:
    w = ctypes.c_int()
    _check(_lib.ngram_auto_choice(ctx.handle, n_tokens, ctypes.byref(w)))
    return w.value


def ngram_dedup_rows(ctx: Context, tokens: torch.Tensor, history: torch.Tensor | None = None,
                     uniq_out=None, inv_out=None, count_out=None, stream=None):
    """(uniq [N*H], inv [N*H], count [1]) int32 tensors holding uint32 values: the
    batch's distinct rows in order of first appearance (entries [0, count)) and the
    inverse map."""
    _need(tokens, "tokens", torch.int32, ndim=2)
    n_seq, T = tokens.shape
    M = n_seq * T * ctx.n_heads
    dev = tokens.device
    if history is not None:
        _need(history, "history", torch.int32, dev, ndim=2)
    if uniq_out is None:
        uniq_out = torch.empty(M, dtype=torch.int32, device=dev)
    if inv_out is None:
        inv_out = torch.empty(M, dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty(1, dtype=torch.int32, device=dev)
    _check(_lib.ngram_dedup_rows(ctx.handle, _ptr(tokens), _ptr(history), n_seq, T,
                                 _ptr(uniq_out), _ptr(inv_out), _ptr(count_out),
                                 _stream(stream)))
    return uniq_out, inv_out, count_out


def ngram_prefetch(ctx: Context, slot: int, tokens: torch.Tensor, history: torch.Tensor | None = None,
                   stream=None) -> None:
    """Stage the distinct rows of this batch in HBM slot `slot` (asynchronous)."""
    _need(tokens, "tokens", torch.int32, ndim=2)
    n_seq, T = tokens.shape
    if history is not None:
        _need(history, "history", torch.int32, tokens.device, ndim=2)
    _check(_lib.ngram_prefetch(ctx.handle, slot, _ptr(tokens), _ptr(history), n_seq, T,
                               _stream(stream)))


def ngram_forward_staged(ctx: Context, slot: int, residual: torch.Tensor, gate: torch.Tensor,
                         out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """ngram_forward for the batch staged in `slot`, gathering from HBM staging."""
    _need(residual, "residual", torch.bfloat16)
    _check_gate(ctx, gate, residual.numel() // ctx.d, residual.device)
    if out is None:
        out = torch.empty_like(residual)
    _need(out, "out", torch.bfloat16, residual.device)
    _check(_lib.ngram_forward_staged(ctx.handle, slot, _ptr(residual), _ptr(gate), _ptr(out),
                                     _stream(stream)))
    return out


def ngram_backward_rows(ctx: Context, tokens: torch.Tensor, grad_out: torch.Tensor,
                        gate: torch.Tensor, history: torch.Tensor | None = None,
                        uniq_out: torch.Tensor | None = None, count_out: torch.Tensor | None = None,
                        grad_rows: torch.Tensor | None = None, stream=None):
    """Gradient with respect to the table rows the batch read.  Returns (uniq int32 [N*H],
    count int32 [1], grad_rows fp32 [N*H][d]); the first count entries / rows are valid."""
    _need(tokens, "tokens", torch.int32, ndim=2)
    dev = tokens.device
    n_seq, T = tokens.shape
    N = n_seq * T
    M = N * ctx.n_heads
    _need(grad_out, "grad_out", torch.bfloat16, dev)
    if grad_out.numel() != N * ctx.d:
        raise ValueError("grad_out must hold N * d elements")
    _check_gate(ctx, gate, N, dev)
    if history is not None:
        _need(history, "history", torch.int32, dev, ndim=2)
    if uniq_out is None:
        uniq_out = torch.empty(max(1, M), dtype=torch.int32, device=dev)
    if count_out is None:
        count_out = torch.empty(1, dtype=torch.int32, device=dev)
    if grad_rows is None:
        grad_rows = torch.empty((max(1, M), ctx.d), dtype=torch.float32, device=dev)
    _need(grad_rows, "grad_rows", torch.float32, dev)
    if grad_rows.numel() < M * ctx.d:
        raise ValueError("grad_rows must hold N * H * d elements")
    _check(_lib.ngram_backward_rows(ctx.handle, _ptr(tokens), _ptr(history), n_seq, T,
                                    _ptr(grad_out), _ptr(gate), _ptr(uniq_out), _ptr(count_out),
                                    _ptr(grad_rows), _stream(stream)))
    return uniq_out, count_out, grad_rows


def ngram_backward_gate(ctx: Context, tokens: torch.Tensor, grad_out: torch.Tensor,
                        history: torch.Tensor | None = None, out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """Gradient with respect to the gate: fp32 [d], or fp32 [N][d] for a per-token gate."""
    _need(tokens, "tokens", torch.int32, ndim=2)
    dev = tokens.device
    n_seq, T = tokens.shape
    N = n_seq * T
    _need(grad_out, "grad_out", torch.bfloat16, dev)
    if grad_out.numel() != N * ctx.d:
        raise ValueError("grad_out must hold N * d elements")
    if history is not None:
        _need(history, "history", torch.int32, dev, ndim=2)
    shape = (N, ctx.d) if _token_gate(ctx) else (ctx.d,)
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=dev)
    _need(out, "out", torch.float32, dev)
    if out.numel() != (N * ctx.d if _token_gate(ctx) else ctx.d):
        raise ValueError("out must hold %s elements" % (shape,))
    _check(_lib.ngram_backward_gate(ctx.handle, _ptr(tokens), _ptr(history), n_seq, T,
                                    _ptr(grad_out), _ptr(out), _stream(stream)))
    return out


def ngram_fill_synthetic_cols(table: torch.Tensor, R: int, d: int, col0: int, dtype: int = NGRAM_BF16,
                              seed: int = 0, row_scale: torch.Tensor | None = None, stream=None) -> None:
    """Columns [col0, col0 + d) of the synthetic table (a column shard)."""
    _check(_lib.ngram_fill_synthetic_cols(_ptr(table), _ptr(row_scale), R, d, col0, dtype,
                                          seed & (2**64 - 1), _stream(stream)))


def _addr(x) -> int:
    return x.data_ptr() if isinstance(x, torch.Tensor) else int(x)


def ngram_forward_shard(ctx: Context, tokens: torch.Tensor, residual: torch.Tensor, gate: torch.Tensor,
                        outs, d_full: int, col0: int, history: torch.Tensor | None = None,
                        stream=None) -> None:
    """This rank's columns [col0, col0 + ctx.d) of the lookup, stored into every buffer of
    `outs` (tensors or device addresses of bf16 [N][d_full]: this rank's output and the
    peers' mapped ones).  residual bf16 [N][d_full]; gate fp32 [d_full] (or bf16
    [N][d_full] with NGRAM_FLAG_TOKEN_GATE)."""
    _need(tokens, "tokens", torch.int32, ndim=2)
    dev = tokens.device
    n_seq, T = tokens.shape
    N = n_seq * T
    _need(residual, "residual", torch.bfloat16, dev)
    if residual.numel() != N * d_full:
        raise ValueError("residual must hold N * d_full elements")
    if _token_gate(ctx):
        _need(gate, "gate", torch.bfloat16, dev)
        if gate.numel() != N * d_full:
            raise ValueError("a per-token gate must hold N * d_full elements")
    else:
        _need(gate, "gate", torch.float32, dev)
        if gate.numel() != d_full:
            raise ValueError("gate must hold d_full elements")
    if history is not None:
        _need(history, "history", torch.int32, dev, ndim=2)
    ptrs = (_P * 8)()
    outs = list(outs)
    if not 1 <= len(outs) <= 8:
        raise ValueError("1 to 8 output buffers")
    for i, o in enumerate(outs):
        if isinstance(o, torch.Tensor):
            _need(o, "outs[%d]" % i, torch.bfloat16)
            if o.numel() < N * d_full:
                raise ValueError("outs[%d] must hold N * d_full elements" % i)
        ptrs[i] = _addr(o)
    _check(_lib.ngram_forward_shard(ctx.handle, _ptr(tokens), _ptr(history), n_seq, T, d_full, col0,
                                    _ptr(residual), _ptr(gate), ptrs, len(outs), _stream(stream)))


def ngram_device_alloc(nbytes: int) -> int:
    p = _P()
    _check(_lib.ngram_device_alloc(ctypes.byref(p), nbytes))
    return p.value


def ngram_device_free(ptr: int) -> None:
    _check(_lib.ngram_device_free(ptr))


def ngram_ipc_get_handle(ptr: int) -> bytes:
    buf = ctypes.create_string_buffer(64)
    _check(_lib.ngram_ipc_get_handle(ptr, buf))
    return buf.raw


def ngram_ipc_open(handle: bytes) -> int:
    if len(handle) != 64:
        raise ValueError("an IPC handle is 64 bytes")
    p = _P()
    _check(_lib.ngram_ipc_open(handle, ctypes.byref(p)))
    return p.value


def ngram_ipc_close(ptr: int) -> None:
    _check(_lib.ngram_ipc_close(ptr))


def ngram_selftest_wait_timeout(ctx: Context, limit_ms: int = 100, stream=None) -> None:
    """Run one bounded wait that nothing ends; it must give up and set error code 2."""
    _check(_lib.ngram_selftest_wait_timeout(ctx.handle, limit_ms, _stream(stream)))
