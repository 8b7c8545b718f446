"""B200 (sm_100a) hashed n-gram embedding lookup.

For every token the bigram and trigram context is hashed into one large row table,
16 rows are gathered and summed in fp32, and the sum is added to the residual stream
through an elementwise gate -- the "storage expert" of "Qwen Brought Back N-Grams.
All 51 Billion Parameters of Them." (section "N-grams, of all things") with the gate
of "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with Heterogeneous Memory
Prefetch", Key point 1.

The compute lives in libngram.so (C ABI in include/ngram.h, CUDA kernels in csrc/);
this package is its thin ctypes binding.  Importing it fails if the library is not
built: there is no fallback path.
"""
from ._binding import (  # noqa: F401
    LIB_PATH, Context, HashParams, NgramError, lib,
    NGRAM_OK, NGRAM_EINVAL, NGRAM_ENOMEM, NGRAM_ECUDA, NGRAM_EUNSUPPORTED, NGRAM_ETIMEOUT,
    NGRAM_EDEVICE, NGRAM_BF16, NGRAM_INT8_ROWSCALE, NGRAM_FP8_E4M3_ROWSCALE, NGRAM_NVFP4, NGRAM_RES_HBM, NGRAM_RES_HOST_UVA,
    NGRAM_RES_HOST_DMA, NGRAM_RES_HOST_AUTO, NGRAM_AUTO_UVA_DEDUP, NGRAM_FLAG_DEDUP, NGRAM_FLAG_TMA_STAGING, NGRAM_FLAG_SORT, NGRAM_FLAG_BATCH_ORDER, NGRAM_FLAG_TOKEN_GATE, NGRAM_SORT_MIN_TOKENS,
    NGRAM_STAGE_SLOTS, MAX_HEADS, DEFAULT_BASE_SEED, DEFAULT_PAD_ID,
    ngram_default_hash_params, ngram_init, ngram_forward, ngram_forward_host, ngram_hash_indices,
    ngram_fill_synthetic, ngram_get_device_error, ngram_last_error, ngram_status_string,
    ngram_destroy, HostTable, ngram_host_alloc, ngram_host_free, ngram_set_wait_timeout,
    ngram_auto_choice, ngram_dedup_rows, ngram_prefetch, ngram_forward_staged, ngram_row_bytes,
    ngram_backward_rows, ngram_backward_gate, ngram_fill_synthetic_cols, ngram_forward_shard,
    ngram_device_alloc, ngram_device_free, ngram_ipc_get_handle, ngram_ipc_open, ngram_ipc_close,
    ngram_selftest_wait_timeout,
)
