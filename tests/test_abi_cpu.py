"""Host-side checks of libngram.so that need no GPU: the library loads, exports every
entry point include/ngram.h declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import pytest
import torch

import hashed_gram_embedding_ngram_b200 as ng

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ngram.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NGRAM_API\s+[\w\s\*]*?\b(ngram_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("ngram_init", "ngram_forward", "ngram_hash_indices", "ngram_fill_synthetic",
              "ngram_get_device_error", "ngram_last_error", "ngram_status_string",
              "ngram_destroy", "ngram_default_hash_params"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(ng.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else():
    out = os.popen("nm -D --defined-only %s" % ng.LIB_PATH).read().split("\n")
    exported = sorted(l.split()[-1] for l in out if " T " in l)
    assert exported == _declared()


def _header_constants():
    """Integer constants of the header: #define NGRAM_X <literal> and enum entries."""
    text = open(HEADER).read()
    out = {}
    for name, val in re.findall(r"#define\s+(NGRAM_\w+)\s+(0x[0-9A-Fa-f]+|\d+)[uUlL]*\b", text):
        out[name] = int(val, 0)
    for name, val in re.findall(r"^\s+(NGRAM_\w+)\s*=\s*(\d+)", text, flags=re.M):
        out[name] = int(val)
    return out


def test_binding_constants_match_the_header():
    consts = _header_constants()
    assert {"NGRAM_FLAG_DEDUP", "NGRAM_AUTO_UVA_DEDUP", "NGRAM_NVFP4", "NGRAM_RES_HOST_AUTO",
            "NGRAM_EDEVICE", "NGRAM_SORT_MIN_TOKENS", "NGRAM_STAGE_SLOTS"} <= set(consts)
    aliases = {"NGRAM_MAX_HEADS": "MAX_HEADS", "NGRAM_DEFAULT_BASE_SEED": "DEFAULT_BASE_SEED",
               "NGRAM_DEFAULT_PAD_ID": "DEFAULT_PAD_ID"}
    checked = 0
    for name, val in consts.items():
        attr = aliases.get(name, name)
        if hasattr(ng, attr):
            assert getattr(ng, attr) == val, name
            checked += 1
    assert checked >= 20


def _prototypes():
    """(name, parameter count) of every NGRAM_API prototype of the header."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for name, params in re.findall(r"NGRAM_API\s+[\w\s\*]*?\b(ngram_\w+)\s*\(([^;]*?)\)\s*;", text,
                                   flags=re.S):
        p = params.strip()
        out[name] = 0 if p in ("", "void") else len(p.split(","))
    return out


def test_binding_argument_counts_match_the_header():
    """Every entry point the binding declares argtypes for takes as many arguments as its
    prototype (an ABI drift would otherwise only show as a crash on the GPU)."""
    protos = _prototypes()
    assert set(protos) == set(_declared())
    lib = ng.lib()
    checked = 0
    for name, n in protos.items():
        at = getattr(lib, name).argtypes
        if at is not None:
            assert len(at) == n, (name, len(at), n)
            checked += 1
    assert checked >= len(protos) - 1          # ngram_dedup_rows_noalloc is bound by its test


def test_status_strings():
    assert ng.ngram_status_string(ng.NGRAM_OK) == "NGRAM_OK"
    assert ng.ngram_status_string(ng.NGRAM_EDEVICE) == "NGRAM_EDEVICE"
    assert ng.ngram_status_string(99) == "NGRAM_UNKNOWN"


def test_default_hash_params():
    hp = ng.ngram_default_hash_params()
    assert (hp.base_seed, hp.n_bigram_heads, hp.n_trigram_heads, hp.pad_id, hp.vocab_size) == (
        0x6E6772616D5F7631, 8, 8, 0x1FFFFF, 0x1FFFFF)


_T = torch.zeros(64, dtype=torch.bfloat16)      # any 16-byte aligned host address


@pytest.mark.parametrize("kw,msg", [
    (dict(R=0), "R must"),
    (dict(R=2**32), "R must"),
    (dict(d=12), "d % 8"),
    (dict(d=0), "d % 8"),
    (dict(max_tokens=0), "max_tokens"),
    (dict(hp=dict(n_bigram_heads=9, n_trigram_heads=8)), "heads"),
    (dict(hp=dict(n_bigram_heads=0, n_trigram_heads=0)), "heads"),
    (dict(hp=dict(pad_id=1 << 21)), "pad_id"),
    (dict(hp=dict(vocab_size=1 << 21)), "vocab_size"),
    (dict(hp=dict(vocab_size=0)), "vocab_size"),
    (dict(hp=dict(flags=0x100)), "flags"),
    (dict(dtype=7), "dtype"),
    (dict(where=9), "residency"),
    (dict(dtype=ng.NGRAM_INT8_ROWSCALE, d=32), "row_scale"),
    (dict(dtype=ng.NGRAM_FP8_E4M3_ROWSCALE, d=32), "row_scale"),
    (dict(dtype=ng.NGRAM_FP8_E4M3_ROWSCALE, d=24), "d % 16"),
    (dict(dtype=ng.NGRAM_NVFP4, d=48), "d % 32"),
    (dict(dtype=ng.NGRAM_NVFP4, d=64), "global scale"),
    (dict(hp=dict(flags=0x12)), "TOKEN_GATE"),
    (dict(d=264, max_tokens=2**31), "too large"),
])
def test_init_rejects_bad_arguments_before_cuda(kw, msg):
    args = dict(R=1000, d=256, dtype=ng.NGRAM_BF16, where=ng.NGRAM_RES_HBM, max_tokens=16)
    hpo = kw.pop("hp", None)
    args.update(kw)
    hp = ng.ngram_default_hash_params(**(hpo or {}))
    with pytest.raises(ng.NgramError) as ei:
        ng.ngram_init(_T, args["R"], args["d"], args["dtype"], args["where"], hp,
                      args["max_tokens"])
    assert ei.value.status == ng.NGRAM_EINVAL
    assert msg in str(ei.value)


def test_row_bytes_of_every_format():
    assert ng.ngram_row_bytes(ng.NGRAM_BF16, 2560) == 5120
    assert ng.ngram_row_bytes(ng.NGRAM_INT8_ROWSCALE, 2560) == 2560
    assert ng.ngram_row_bytes(ng.NGRAM_FP8_E4M3_ROWSCALE, 2560) == 2560
    # nvfp4: d/2 code bytes + d/16 scale bytes padded to 16 (always a multiple of 16)
    for d in (32, 96, 256, 2560, 2592, 4096):
        rb = ng.ngram_row_bytes(ng.NGRAM_NVFP4, d)
        assert rb == d // 2 + -(-(d // 16) // 16) * 16 and rb % 16 == 0
    assert ng.ngram_row_bytes(ng.NGRAM_NVFP4, 2560) == 1440
    for dt, d in ((ng.NGRAM_NVFP4, 16), (ng.NGRAM_FP8_E4M3_ROWSCALE, 8), (ng.NGRAM_BF16, 4), (9, 64)):
        with pytest.raises(ng.NgramError):
            ng.ngram_row_bytes(dt, d)


def test_bf16_init_rejects_a_row_scale():
    s = torch.zeros(4, dtype=torch.float32)
    with pytest.raises(ng.NgramError) as ei:
        ng.ngram_init(_T, 1000, 256, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, None, 16, row_scale=s)
    assert "no row_scale" in str(ei.value)


def test_init_rejects_null_and_misaligned_table():
    lib = ng.lib()
    h = ctypes.c_void_p(123)
    assert lib.ngram_init(ctypes.byref(h), None, None, 10, 8, 0, 0, None, 4) == ng.NGRAM_EINVAL
    assert h.value is None                                  # *out reset on failure
    addr = ctypes.c_void_p(_T.data_ptr() + 2)
    assert lib.ngram_init(ctypes.byref(h), addr, None, 10, 8, 0, 0, None, 4) == ng.NGRAM_EINVAL
    assert "aligned" in ng.ngram_last_error()


def test_valid_init_without_a_gpu_reports_a_cuda_error():
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(ng.NgramError) as ei:
        ng.ngram_init(_T, 1000, 256, ng.NGRAM_BF16, ng.NGRAM_RES_HBM, None, 16)
    assert ei.value.status in (ng.NGRAM_ECUDA, ng.NGRAM_ENOMEM)


def test_fill_rejects_bad_arguments():
    with pytest.raises(ng.NgramError):
        ng.ngram_fill_synthetic(_T, 0, 8, stream=0)
    with pytest.raises(ng.NgramError):
        ng.ngram_fill_synthetic(_T, 10, 12, stream=0)
    with pytest.raises(ng.NgramError):
        ng.ngram_fill_synthetic(_T, 10, 32, ng.NGRAM_INT8_ROWSCALE, stream=0)   # no row_scale
    with pytest.raises(ng.NgramError):
        ng.ngram_fill_synthetic(_T, 10, 32, ng.NGRAM_NVFP4, stream=0)           # no global scale
    with pytest.raises(ng.NgramError):
        ng.ngram_fill_synthetic(_T, 10, 48, ng.NGRAM_NVFP4, row_scale=_T, stream=0)


def test_selftest_rejects_bad_arguments():
    lib = ng.lib()
    assert lib.ngram_selftest_wait_timeout(None, 100, None) == ng.NGRAM_EINVAL


def test_backward_entry_points_reject_a_null_context():
    lib = ng.lib()
    assert lib.ngram_backward_rows(None, None, None, 1, 1, None, None, None, None, None, None) == ng.NGRAM_EINVAL
    assert lib.ngram_backward_gate(None, None, None, 1, 1, None, None, None) == ng.NGRAM_EINVAL


def test_null_context_is_rejected():
    lib = ng.lib()
    assert lib.ngram_forward(None, None, None, 1, 1, None, None, None, None) == ng.NGRAM_EINVAL
    assert lib.ngram_hash_indices(None, None, None, 1, 1, None, None) == ng.NGRAM_EINVAL
    assert lib.ngram_get_device_error(None, None, 0) == ng.NGRAM_EINVAL
    lib.ngram_destroy(None)                                 # no-op


def test_new_entry_points_reject_bad_arguments():
    lib = ng.lib()
    assert lib.ngram_set_wait_timeout(None, 10) == ng.NGRAM_EINVAL
    w = ctypes.c_int()
    assert lib.ngram_auto_choice(None, 1, ctypes.byref(w)) == ng.NGRAM_EINVAL
    assert lib.ngram_dedup_rows(None, None, None, 1, 1, None, None, None, None) == ng.NGRAM_EINVAL
    p = ctypes.c_void_p(5)
    assert lib.ngram_host_alloc(ctypes.byref(p), 0) == ng.NGRAM_EINVAL and p.value is None
    assert lib.ngram_host_alloc(None, 16) == ng.NGRAM_EINVAL
    assert lib.ngram_host_free(None) == ng.NGRAM_OK


def test_dedup_flag_is_for_hbm_and_uva_only():
    hp = ng.ngram_default_hash_params(flags=ng.NGRAM_FLAG_DEDUP)
    for where in (ng.NGRAM_RES_HOST_DMA, ng.NGRAM_RES_HOST_AUTO):
        with pytest.raises(ng.NgramError) as ei:
            ng.ngram_init(_T, 1000, 256, ng.NGRAM_BF16, where, hp, 16)
        assert ei.value.status == ng.NGRAM_EINVAL and "HOST_UVA" in str(ei.value)


def test_sort_flag_combinations_rejected():
    for where, flags in ((ng.NGRAM_RES_HOST_DMA, ng.NGRAM_FLAG_SORT),
                         (ng.NGRAM_RES_HBM, ng.NGRAM_FLAG_SORT | ng.NGRAM_FLAG_DEDUP),
                         (ng.NGRAM_RES_HBM, ng.NGRAM_FLAG_SORT | ng.NGRAM_FLAG_TMA_STAGING),
                         (ng.NGRAM_RES_HBM, ng.NGRAM_FLAG_SORT | ng.NGRAM_FLAG_BATCH_ORDER)):
        with pytest.raises(ng.NgramError) as ei:
            ng.ngram_init(_T, 1000, 256, ng.NGRAM_BF16, where,
                          ng.ngram_default_hash_params(flags=flags), 16)
        assert ei.value.status == ng.NGRAM_EINVAL


def test_prefetch_entry_points_reject_null_context():
    lib = ng.lib()
    assert lib.ngram_prefetch(None, 0, None, None, 1, 1, None) == ng.NGRAM_EINVAL
    assert lib.ngram_forward_staged(None, 0, None, None, None, None) == ng.NGRAM_EINVAL


def test_noalloc_dedup_refuses_over_limit_batches_before_cuda():
    """The limit check of ngram_dedup_rows_noalloc runs before any CUDA call, and a batch
    whose n_seq * T * heads wraps in 64 bits (2^31 x 2^31 x 16 = 2^66) is refused too."""
    lib = ng.lib()
    P, u32, u64 = ctypes.c_void_p, ctypes.c_uint32, ctypes.c_uint64
    f = lib.ngram_dedup_rows_noalloc
    f.argtypes = [P, u64, P, P, u32, u32, P, P, P, P]
    f.restype = ctypes.c_int
    hp = ng.ngram_default_hash_params(vocab_size=1000)
    x = P(16)                                  # never dereferenced: refused first
    for n_seq, T in ((1, 4097), (1 << 31, 1 << 31), (4096, 1 << 20)):
        assert f(ctypes.byref(hp), 1000, x, None, n_seq, T, x, x, x, None) == ng.NGRAM_EINVAL
        assert "65536" in ng.ngram_last_error()
    assert f(ctypes.byref(hp), 0, x, None, 1, 1, x, x, x, None) == ng.NGRAM_EINVAL
