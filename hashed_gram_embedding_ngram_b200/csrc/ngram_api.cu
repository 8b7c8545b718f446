// ngram_api.cu -- host side of libngram.so: argument checks, context, launches.
//
// Every entry point validates its arguments before touching CUDA and reports through
// an ngram_status; nothing here aborts the process.  Compute is asynchronous on the
// caller's stream, except where a residency mode needs the host in the loop (DMA
// staging, the first AUTO call of a batch-size bucket); those waits are bounded and
// return NGRAM_ETIMEOUT.  The operation and its definitions are stated in
// include/ngram.h.
#include <algorithm>
#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <thread>
#include <utility>
#include <vector>

#if defined(__x86_64__)
#include <cpuid.h>
#include <immintrin.h>
#endif

#include <cuda.h>            // CUcontext / CUresult types for the driver entry points
#include <cuda_runtime.h>

#include "ngram.h"
#include "device_common.cuh"
#include "fill.cuh"
#include "gather.cuh"
#include "gather_int8.cuh"
#include "gather_nvfp4.cuh"
#include "gather_c8.cuh"
#include "gather_staged.cuh"
#include "gather_bulk.cuh"
#include "dedup.cuh"
#include "order.cuh"
#include "sort.cuh"
#include "backward.cuh"

using namespace ngram;


// Build-time tuning of the gathers (measured on B200, 20M x 2560 bf16, 32,768 tokens):
//   NGRAM_SPI_ONE_FORMATS: bit t set = row format t always gives a warp one 32-vector strip
//     per work item, so the strips of a token run on several warps at once and each
//     recomputes the 16 hashes: bf16 (10 strips, 455 us against 470 us with one warp walking
//     them) and NVFP4 (132.5 against 124.7 M tokens/s).  The row-scale formats (int8, FP8)
//     walk a token's strips in one warp once the batch fills the GPU, so the hashes and the
//     dependent row-scale loads run once per token: FP8 114.1 against 107.3 M tokens/s,
//     int8 (uniform tokens) 110.4 against 104.8.
//   The TMA-staged kernel (NGRAM_FLAG_TMA_STAGING) measured 522-895 us depending on
//     chunk and ring depth; its tunables are below.
#ifndef NGRAM_SPI_ONE_FORMATS
#define NGRAM_SPI_ONE_FORMATS ((1u << NGRAM_BF16) | (1u << NGRAM_NVFP4))
#endif
#ifndef NGRAM_PDL                        // 1: gathers and order kernels launch as programmatic dependents
#define NGRAM_PDL 1
#endif
#ifndef NGRAM_THREE_CTA_DECODE           // 1: bf16 batches that fit one wave of 3 CTAs/SM use them
#define NGRAM_THREE_CTA_DECODE 1
#endif
#ifndef NGRAM_BULK_CHUNK_COLS           // columns per work item of the bulk kernel
#define NGRAM_BULK_CHUNK_COLS 1280
#endif
#ifndef NGRAM_BULK_SMEM_BYTES           // shared memory per CTA for the stage ring
#define NGRAM_BULK_SMEM_BYTES (100 * 1024)
#endif
#ifndef NGRAM_STAGED_SMEM_BYTES         // shared memory per CTA of the staged 8- and 4-bit gathers
#define NGRAM_STAGED_SMEM_BYTES (200 * 1024)
#endif
#ifndef NGRAM_STAGED_CTAS_PER_SM
#define NGRAM_STAGED_CTAS_PER_SM 1
#endif
#ifndef NGRAM_BULK_CTAS_PER_SM
#define NGRAM_BULK_CTAS_PER_SM 2
#endif
// NGRAM_UVA_CTAS: CTAs of the host-resident (UVA) gather.  4 CTAs (256 KB of row loads in
//   flight) keep PCIe as busy as 8 or 296 (decode-256 0.416 against 0.414 ms at 8; prefill
//   8192 13.05 ms at both, 0.92 of measured H2D) and leave the most SMs to the work beside
//   the lookup: a bf16 4096x2560x2560 GEMM on another stream keeps 1222-1236 TFLOP/s beside
//   the decode-256 lookup at 4 CTAs, 1061-1063 at 8, 667 at 296; at 2 CTAs the lookup slows
//   to 0.49 ms.
// NGRAM_UVA_COPY_CTAS: CTAs of the copy kernel that moves each distinct host row once into
//   HBM staging (UVA + dedup, prefetch).  Its flat copy needs 8: at 4 the 8192-token copy
//   took 14.1 against 11.4 ms.
#ifndef NGRAM_UVA_CTAS
#define NGRAM_UVA_CTAS 4
#endif
#ifndef NGRAM_UVA_COPY_CTAS
#define NGRAM_UVA_COPY_CTAS 8
#endif
#ifndef NGRAM_DMA_CHUNK_BYTES           // host gather -> H2D pipelining granularity
#define NGRAM_DMA_CHUNK_BYTES (8u << 20)
#endif

// ngram_forward_host pipeline (measured, 32,768-token prefill, pinned host buffers): 16 MB
// chunks on 3 streams 4.20 ms; 8 MB on 2 streams 4.27-4.48 ms; 4 MB 4.6-5.2 ms; a thinner
// gather grid does not help.  The copies alone, both directions, take 3.50 ms.
#ifndef NGRAM_STAGE_SLOTS               // staged batches ngram_prefetch keeps in HBM
#define NGRAM_STAGE_SLOTS 2
#endif
#ifndef NGRAM_HOST_BUFFERS              // pipeline streams of ngram_forward_host
#define NGRAM_HOST_BUFFERS 3
#endif

struct ngram_ctx {
    const void *table;          // caller's pointer (device, or host for host residency)
    const void *table_dev;      // device-visible alias used by kernels (UVA), or table
    const float *row_scale;     // per-row scales (int8, fp8) as passed, else NULL
    const float *row_scale_dev; // what the gather reads: per-row scales, or the NVFP4
                                // global scale (d_gscale)
    uint64_t R;
    uint32_t d;
    uint32_t row_bytes;         // 2d (bf16), d (int8, fp8), d/2 + ceil16(d/16) (nvfp4)
    ngram_dtype dtype;
    ngram_residency where;
    ngram_hash_params hp;
    uint32_t H;
    uint32_t max_tokens;
    uint64_t barrett_m;
    int device;
    int num_sms;
    int gather_blocks_per_sm;
    int bulk_smem_set;
    int staged_smem_set;
    uint32_t wait_ms;           // bound of every host-side wait
    uint32_t *d_err;            // 4 words
    float *d_gscale;            // NVFP4: device copy of the global scale
    // dedup scratch, sized for max_tokens (allocated on first use)
    uint32_t dd_cap;            // entries (max_tokens * H)
    uint32_t dd_pcap;           // hash-table slots (power of two >= 2 * dd_cap)
    uint32_t *d_idx, *d_slot, *d_pos, *d_inv, *d_uniq, *d_keys, *d_first, *d_uid, *d_bsum, *d_count;
    uint32_t *d_rowid;          // [max_tokens][H] row ids of the forward's hash-once step (its
                                // own buffer: ngram_prefetch may use d_idx on another stream)
    // staging of unique rows (HBM dedup, DMA), sized for dd_cap rows
    uint8_t *d_stage;
    float *d_stage_scale;
    uint8_t *h_stage;           // pinned (DMA)
    float *h_stage_scale;
    uint32_t *h_uniq;           // pinned (DMA)
    uint32_t *h_count;          // pinned (DMA)
    cudaEvent_t ev_sync;        // D2H of the unique-row list
    cudaEvent_t ev_stage_free;  // last H2D of the previous DMA call
    int stage_in_use;
    cudaEvent_t ev_t0, ev_t1;   // AUTO timing
    int auto_choice[33];        // per ceil(log2 N): 0 undecided, else HOST_UVA, HOST_DMA or
                                // NGRAM_AUTO_UVA_DEDUP
    // ngram_forward_host: device copies of the host inputs, double-buffered chunks
    int32_t *hp_tok, *hp_hist;
    uint16_t *hp_res[NGRAM_HOST_BUFFERS], *hp_out[NGRAM_HOST_BUFFERS];
    uint32_t hp_chunk;          // tokens per full chunk
    cudaStream_t hp_s[NGRAM_HOST_BUFFERS];   // pipeline streams, one chunk buffer pair each
    cudaEvent_t hp_entry;
    cudaEvent_t hp_h2d[NGRAM_HOST_BUFFERS];   // [0]: tokens uploaded
    cudaEvent_t hp_d2h[NGRAM_HOST_BUFFERS];   // end of each stream's part of the last call
    // NGRAM_FLAG_SORT: bucket of each token, bucket counts / cursors, processing order
    uint32_t *so_bucket, *so_hist, *so_perm;
    // backward: radix-sort buffers (keys, values, twice), digit counts, scan totals,
    // segment starts; the shared-gate gradient's fp64 partials
    uint32_t *bw_k[2], *bw_v[2], *bw_hist, *bw_tot, *bw_seg, *bw_word;
    int bw_rows_per_sm[2];      // resident k_rows_grad CTAs per SM (shared gate, per-token gate)
    double *bw_part;
    // ngram_prefetch / ngram_forward_staged: a ring of staged batches in HBM
    struct Slot {
        uint32_t *inv;          // [max_tokens * H] row ids into `stage`
        uint8_t *stage;         // [max_tokens * H][row_bytes] distinct rows
        float *stage_scale;     // [max_tokens * H] (int8)
        uint32_t n_seq, T;      // the staged batch (0 tokens: empty slot)
        uint64_t epoch;         // prefetch call that filled the slot
    } slot[NGRAM_STAGE_SLOTS];
    uint64_t prefetch_epoch;
};

namespace {

thread_local std::string g_last_error;

ngram_status fail(ngram_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

ngram_status cuda_fail(cudaError_t e, const char *what) {
    return fail(e == cudaErrorMemoryAllocation ? NGRAM_ENOMEM : NGRAM_ECUDA, "%s: %s (%s)", what,
                cudaGetErrorString(e), cudaGetErrorName(e));
}

#define NG_CUDA(call, what)                                  \
    do {                                                     \
        cudaError_t e_ = (call);                             \
        if (e_ != cudaSuccess) return cuda_fail(e_, what);   \
    } while (0)

#define NG_CHECK(expr)                                       \
    do {                                                     \
        ngram_status s_ = (expr);                            \
        if (s_ != NGRAM_OK) return s_;                       \
    } while (0)

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Lazily made scratch: each buffer, event or stream is made only while its handle is still
// NULL, so a call that failed part-way (ENOMEM) leaves the context consistent, and a later
// call makes what is missing instead of running with a NULL buffer.
template <class T>
ngram_status dev_alloc(T **p, size_t bytes, const char *what) {
    if (*p != nullptr) return NGRAM_OK;
    void *q = nullptr;
    NG_CUDA(cudaMalloc(&q, bytes), what);
    *p = static_cast<T *>(q);
    return NGRAM_OK;
}
template <class T>
ngram_status pinned_alloc(T **p, size_t bytes, const char *what) {
    if (*p != nullptr) return NGRAM_OK;
    void *q = nullptr;
    NG_CUDA(cudaHostAlloc(&q, bytes, cudaHostAllocPortable), what);
    *p = static_cast<T *>(q);
    return NGRAM_OK;
}
ngram_status event_once(cudaEvent_t *ev, unsigned flags) {
    if (*ev != nullptr) return NGRAM_OK;
    NG_CUDA(cudaEventCreateWithFlags(ev, flags), "cudaEventCreate");
    return NGRAM_OK;
}

// Row formats.  Per-row scales (int8, fp8) travel with the rows through every staging
// path; the NVFP4 block scales sit inside the row bytes and its global scale stays put.
bool scale_per_row(ngram_dtype t) { return t == NGRAM_INT8_ROWSCALE || t == NGRAM_FP8_E4M3_ROWSCALE; }

uint32_t row_bytes_of(ngram_dtype t, uint32_t d) {
    switch (t) {
        case NGRAM_BF16: return 2u * d;
        case NGRAM_NVFP4: return d / 2u + 16u * ((d / 16u + 15u) / 16u);
        default: return d;
    }
}

// d and row_scale rules of each format (ngram_init and ngram_fill_synthetic).
ngram_status check_format(ngram_dtype t, uint32_t d, const float *row_scale) {
    static const char *const names[] = {"bf16", "int8", "fp8", "nvfp4"};
    static const uint32_t multiple[] = {8u, 16u, 16u, 32u};
    if (t < NGRAM_BF16 || t > NGRAM_NVFP4) return fail(NGRAM_EINVAL, "unknown dtype %d", static_cast<int>(t));
    if (d == 0 || d % multiple[t] != 0)
        return fail(NGRAM_EINVAL, "%s rows need d %% %u == 0 and d > 0, got %u", names[t], multiple[t], d);
    if (t == NGRAM_BF16 && row_scale != nullptr) return fail(NGRAM_EINVAL, "bf16 rows take no row_scale");
    if (t != NGRAM_BF16 && row_scale == nullptr)
        return fail(NGRAM_EINVAL, "%s rows need row_scale (%s)", names[t],
                    t == NGRAM_NVFP4 ? "the fp32 global scale" : "one fp32 per row");
    return NGRAM_OK;
}

uint32_t ceil_log2(uint64_t x) {
    uint32_t k = 0;
    while ((1ull << k) < x) ++k;
    return k;
}

ngram_status check_hash_params(const ngram_hash_params &hp) {
    const uint32_t H = hp.n_bigram_heads + hp.n_trigram_heads;
    if (hp.n_bigram_heads > NGRAM_MAX_HEADS || hp.n_trigram_heads > NGRAM_MAX_HEADS || H == 0 ||
        H > NGRAM_MAX_HEADS)
        return fail(NGRAM_EINVAL, "heads: n_bigram + n_trigram must be in [1, %u], got %u + %u",
                    NGRAM_MAX_HEADS, hp.n_bigram_heads, hp.n_trigram_heads);
    if (hp.pad_id > kTokenMask)
        return fail(NGRAM_EINVAL, "pad_id %u does not fit in %u bits", hp.pad_id, NGRAM_TOKEN_BITS);
    if (hp.vocab_size == 0 || hp.vocab_size > kTokenMask)
        return fail(NGRAM_EINVAL, "vocab_size must be in [1, 2^21 - 1], got %u", hp.vocab_size);
    if ((hp.flags & ~NGRAM_FLAGS_KNOWN) != 0 || hp.reserved != 0)
        return fail(NGRAM_EINVAL, "unknown flags 0x%x / reserved must be 0", hp.flags);
    return NGRAM_OK;
}

HashArgs hash_args(const ngram_ctx *c) {
    HashArgs a;
    a.base_seed = c->hp.base_seed;
    a.R = c->R;
    a.barrett_m = c->barrett_m;
    a.n_bigram = c->hp.n_bigram_heads;
    a.n_heads = c->H;
    a.pad_id = c->hp.pad_id;
    a.vocab = c->hp.vocab_size;
    return a;
}

ngram_status check_batch(const ngram_ctx *c, const int32_t *tokens, uint32_t n_seq, uint32_t T,
                         uint64_t *N_out) {
    if (c == nullptr) return fail(NGRAM_EINVAL, "ctx is NULL");
    const uint64_t N = static_cast<uint64_t>(n_seq) * T;
    *N_out = N;
    if (N == 0) return NGRAM_OK;
    if (N > c->max_tokens)
        return fail(NGRAM_EINVAL, "n_seq * T = %llu exceeds max_tokens %u",
                    static_cast<unsigned long long>(N), c->max_tokens);
    if (tokens == nullptr) return fail(NGRAM_EINVAL, "tokens is NULL");
    int cur = -1;
    NG_CUDA(cudaGetDevice(&cur), "cudaGetDevice");
    if (cur != c->device)
        return fail(NGRAM_EINVAL, "current device %d is not the context's device %d", cur, c->device);
    return NGRAM_OK;
}

// Wait for an event with the context's bound; the GPU is never waited on without one.
ngram_status wait_event(const ngram_ctx *c, cudaEvent_t ev, const char *what) {
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t e = cudaEventQuery(ev);
        if (e == cudaSuccess) return NGRAM_OK;
        if (e != cudaErrorNotReady) return cuda_fail(e, what);
        const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(
                            std::chrono::steady_clock::now() - t0).count();
        if (ms > static_cast<long long>(c->wait_ms))
            return fail(NGRAM_ETIMEOUT, "%s: no completion within %u ms", what, c->wait_ms);
        std::this_thread::yield();
    }
}

void free_all(ngram_ctx *c) {
    if (c->d_gscale) cudaFree(c->d_gscale);
    uint32_t *dev32[] = {c->d_err, c->d_rowid, c->d_idx, c->d_slot, c->d_pos, c->d_inv, c->d_uniq,
                         c->d_keys, c->d_first, c->d_uid, c->d_bsum, c->d_count};
    for (uint32_t *p : dev32)
        if (p) cudaFree(p);
    if (c->d_stage) cudaFree(c->d_stage);
    if (c->d_stage_scale) cudaFree(c->d_stage_scale);
    if (c->h_stage) cudaFreeHost(c->h_stage);
    if (c->h_stage_scale) cudaFreeHost(c->h_stage_scale);
    if (c->h_uniq) cudaFreeHost(c->h_uniq);
    if (c->h_count) cudaFreeHost(c->h_count);
    cudaEvent_t evs[] = {c->ev_sync, c->ev_stage_free, c->ev_t0, c->ev_t1, c->hp_entry};
    for (cudaEvent_t e : evs)
        if (e) cudaEventDestroy(e);
    for (int b = 0; b < NGRAM_HOST_BUFFERS; ++b) {
        cudaEvent_t pe[] = {c->hp_h2d[b], c->hp_d2h[b]};
        for (cudaEvent_t e : pe)
            if (e) cudaEventDestroy(e);
        if (c->hp_res[b]) cudaFree(c->hp_res[b]);
        if (c->hp_out[b]) cudaFree(c->hp_out[b]);
    }
    for (auto &sl : c->slot) {
        if (sl.inv) cudaFree(sl.inv);
        if (sl.stage) cudaFree(sl.stage);
        if (sl.stage_scale) cudaFree(sl.stage_scale);
    }
    void *bufs[] = {c->hp_tok, c->hp_hist, c->so_bucket, c->so_hist, c->so_perm, c->bw_k[0],
                    c->bw_k[1], c->bw_v[0], c->bw_v[1], c->bw_hist, c->bw_tot, c->bw_seg,
                    c->bw_word, c->bw_part};
    for (void *p : bufs)
        if (p) cudaFree(p);
    for (cudaStream_t s : c->hp_s)
        if (s) cudaStreamDestroy(s);
}

// ---------------------------------------------------------------- scratch on first use
ngram_status ensure_dedup_scratch(ngram_ctx *c) {
    const uint32_t M = c->dd_cap, P = c->dd_pcap, NB = (M + kScanBlock - 1) / kScanBlock;
    NG_CHECK(dev_alloc(&c->d_idx, M * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_slot, M * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_pos, M * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_inv, M * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_uniq, M * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_keys, P * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_first, P * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_uid, P * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_bsum, NB * 4ull, "dedup scratch"));
    NG_CHECK(dev_alloc(&c->d_count, 4, "dedup scratch"));
    return NGRAM_OK;
}

ngram_status ensure_device_stage(ngram_ctx *c) {
    NG_CHECK(dev_alloc(&c->d_stage, static_cast<size_t>(c->dd_cap) * c->row_bytes, "staging"));
    if (scale_per_row(c->dtype)) NG_CHECK(dev_alloc(&c->d_stage_scale, c->dd_cap * 4ull, "staging"));
    return NGRAM_OK;
}

ngram_status ensure_host_stage(ngram_ctx *c) {
    NG_CHECK(ensure_device_stage(c));
    NG_CHECK(pinned_alloc(&c->h_stage, static_cast<size_t>(c->dd_cap) * c->row_bytes, "pinned staging"));
    if (scale_per_row(c->dtype)) NG_CHECK(pinned_alloc(&c->h_stage_scale, c->dd_cap * 4ull, "pinned staging"));
    NG_CHECK(pinned_alloc(&c->h_uniq, c->dd_cap * 4ull, "pinned staging"));
    NG_CHECK(pinned_alloc(&c->h_count, 4, "pinned staging"));
    NG_CHECK(event_once(&c->ev_sync, cudaEventDisableTiming));
    NG_CHECK(event_once(&c->ev_stage_free, cudaEventDisableTiming));
    return NGRAM_OK;
}

#ifndef NGRAM_HOST_CHUNK_BYTES          // residual bytes per pipelined chunk (host buffers)
#define NGRAM_HOST_CHUNK_BYTES (16u << 20)
#endif

// NGRAM_HOST_RAMP = 1: the chunks of ngram_forward_host grow from 1/16 of the full chunk
// at the start and shrink back at the end (1/16, 1/8, 1/4, 1/2, full, ..., full, 1/2, ...,
// 1/16), so the output copies start after a small first chunk and the last output copy is
// small.  Measured on the 32,768-token prefill: 7.71-7.75 against 7.58-7.66 M tokens/s end
// to end (+1.6%); a call still waits for the previous call's outputs (the caller's stream
// order), which is most of the remaining gap to the copies alone.
#ifndef NGRAM_HOST_RAMP
#define NGRAM_HOST_RAMP 1
#endif

// Token counts of the chunks of an N-token call with full chunks of C tokens.
void host_chunks(uint64_t N, uint64_t C, std::vector<uint32_t> &out) {
    out.clear();
    std::vector<uint32_t> tail;
    uint64_t lo = 0, hi = N;
    if (NGRAM_HOST_RAMP) {
        for (uint64_t s = std::max<uint64_t>(1, C >> 4); s < C && lo + 2 * s <= hi; s *= 2) {
            out.push_back(static_cast<uint32_t>(s));
            tail.push_back(static_cast<uint32_t>(s));
            lo += s;
            hi -= s;
        }
    }
    for (; lo < hi; lo += C) out.push_back(static_cast<uint32_t>(std::min(C, hi - lo)));
    out.insert(out.end(), tail.rbegin(), tail.rend());
}

ngram_status ensure_host_path(ngram_ctx *c) {
    const uint64_t row = 2ull * c->d;
    uint64_t chunk = NGRAM_HOST_CHUNK_BYTES / row;
    if (chunk < 1) chunk = 1;
    if (chunk > c->max_tokens) chunk = c->max_tokens;
    c->hp_chunk = static_cast<uint32_t>(chunk);
    NG_CHECK(dev_alloc(&c->hp_tok, c->max_tokens * 4ull, "host-path buffers"));
    NG_CHECK(dev_alloc(&c->hp_hist, c->max_tokens * 8ull, "host-path buffers"));
    for (int b = 0; b < NGRAM_HOST_BUFFERS; ++b) {
        NG_CHECK(dev_alloc(&c->hp_res[b], chunk * row, "host-path buffers"));
        NG_CHECK(dev_alloc(&c->hp_out[b], chunk * row, "host-path buffers"));
        NG_CHECK(event_once(&c->hp_h2d[b], cudaEventDisableTiming));
        NG_CHECK(event_once(&c->hp_d2h[b], cudaEventDisableTiming));
    }
    NG_CHECK(event_once(&c->hp_entry, cudaEventDisableTiming));
    for (int i = 0; i < NGRAM_HOST_BUFFERS; ++i)
        if (c->hp_s[i] == nullptr)
            NG_CUDA(cudaStreamCreateWithFlags(&c->hp_s[i], cudaStreamNonBlocking), "cudaStreamCreate");
    return NGRAM_OK;
}

// ---------------------------------------------------------------- launch helpers
// Scales of staged rows: per-row scales are compacted beside the rows; the NVFP4 global
// scale is read where it is.
const float *staged_scale_src(const ngram_ctx *c) { return scale_per_row(c->dtype) ? c->row_scale_dev : nullptr; }
const float *staged_scale(const ngram_ctx *c, const float *stage_scale) {
    return scale_per_row(c->dtype) ? stage_scale : c->row_scale_dev;
}

GatherArgs gather_args(const ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                       uint32_t T, uint32_t N, const uint16_t *residual, const void *gate,
                       uint16_t *out) {
    GatherArgs g;
    g.h = hash_args(c);
    g.table = c->table_dev;
    g.row_scale = c->row_scale_dev;
    g.tokens = tokens;
    g.history = history;
    g.residual = residual;
    const bool tok_gate = (c->hp.flags & NGRAM_FLAG_TOKEN_GATE) != 0;
    g.gate = tok_gate ? nullptr : static_cast<const float *>(gate);
    g.gate_tok = tok_gate ? static_cast<const uint16_t *>(gate) : nullptr;
    g.out = out;
    g.row_ids = nullptr;
    g.perm = nullptr;
    g.err = c->d_err;
    g.T = T;
    g.N = N;
    g.tok_begin = 0;
    g.d = c->d;
    const uint32_t cols_per_lane = (c->dtype == NGRAM_BF16) ? 8u : 16u;   // 16: 8- and 4-bit rows
    g.n_strips = (c->d / cols_per_lane + 31) / 32;
    g.strips_per_item = g.n_strips;
    g.groups_per_token = 1;
    g.ld = c->d;
    g.n_outs = 0;
    for (uint16_t *&o : g.outs) o = nullptr;
    g.trigger_early = 1;
    return g;
}

// The TMA-staged bf16 gather: work items are (token, column chunk); S stages of
// (H + 1) row chunks each fill the shared-memory budget.
ngram_status launch_bulk(ngram_ctx *c, GatherArgs &g, cudaStream_t s) {
    BulkPlan p;
    uint32_t chunk = NGRAM_BULK_CHUNK_COLS < c->d ? NGRAM_BULK_CHUNK_COLS : c->d;
    chunk = (chunk + 7u) & ~7u;
    p.chunk_cols = chunk;
    p.n_chunks = (c->d + chunk - 1) / chunk;
    const uint32_t H = g.h.n_heads;
    p.stage_bytes = ((H + 1u) * chunk * 2u + 127u) & ~127u;
    uint32_t stages = (NGRAM_BULK_SMEM_BYTES - 128u) / p.stage_bytes;
    if (stages > kBulkMaxStages) stages = kBulkMaxStages;
    if (stages < 2) return fail(NGRAM_EUNSUPPORTED, "bulk gather: stage of %u bytes too large", p.stage_bytes);
    p.stages = stages;
    const uint32_t smem = stages * p.stage_bytes + 128u;      // + alignment slack
    uint32_t threads = ((chunk / 8u) + 31u) & ~31u;
    if (threads > 512u) threads = 512u;
    const uint64_t items = static_cast<uint64_t>(g.N) * p.n_chunks;
    uint64_t grid = static_cast<uint64_t>(c->num_sms) * NGRAM_BULK_CTAS_PER_SM;
    if (grid > items) grid = items;
    if (!c->bulk_smem_set) {
        NG_CUDA(cudaFuncSetAttribute(k_gather_bf16_bulk<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     NGRAM_BULK_SMEM_BYTES), "cudaFuncSetAttribute (bulk gather)");
        NG_CUDA(cudaFuncSetAttribute(k_gather_bf16_bulk<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     NGRAM_BULK_SMEM_BYTES), "cudaFuncSetAttribute (bulk gather)");
        c->bulk_smem_set = 1;
    }
    if (H == 16) k_gather_bf16_bulk<16><<<static_cast<unsigned>(grid), threads, smem, s>>>(g, p);
    else k_gather_bf16_bulk<0><<<static_cast<unsigned>(grid), threads, smem, s>>>(g, p);
    NG_CUDA(cudaGetLastError(), "k_gather_bf16_bulk launch");
    return NGRAM_OK;
}

template <class Rows, bool kTok>
void launch_c8_shard(const GatherArgs &g, unsigned nb, cudaStream_t s, uint32_t rb) {
    if (g.h.n_heads == 16) k_gather_c8<16, Rows, kTok, true><<<nb, 256, 0, s>>>(g, rb);
    else k_gather_c8<0, Rows, kTok, true><<<nb, 256, 0, s>>>(g, rb);
}

template <bool kTok>
void launch_shard(ngram_dtype t, const GatherArgs &g, unsigned nb, cudaStream_t s, uint32_t rb) {
    switch (t) {
        case NGRAM_BF16: launch_c8_shard<RowsBf16, kTok>(g, nb, s, rb); break;
        case NGRAM_INT8_ROWSCALE: launch_c8_shard<Rows8bit<Int8Codes>, kTok>(g, nb, s, rb); break;
        case NGRAM_FP8_E4M3_ROWSCALE: launch_c8_shard<Rows8bit<E4m3Codes>, kTok>(g, nb, s, rb); break;
        case NGRAM_NVFP4: launch_c8_shard<RowsNvfp4, kTok>(g, nb, s, rb); break;
    }
}

// Launch with programmatic stream serialization: the kernel may be scheduled while the
// previous kernel of the stream is still running, and waits for it (griddepcontrol.wait)
// before its first global memory access -- the launch latency overlaps the previous
// kernel's tail, the results are those of plain stream order.  Only kernels that call
// grid_dependency_wait() first are launched this way.  dependent = false launches plainly
// (grid_dependency_wait() then returns at once): the bounded-grid lookups that run beside
// other work on the GPU, whose early resident-but-waiting CTAs would hold SM slots that work
// could use.
template <typename... KArgs, typename... Args>
cudaError_t launch_maybe_dependent(bool dependent, void (*kernel)(KArgs...), dim3 grid, unsigned block,
                                   cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (NGRAM_PDL && dependent) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, unsigned block, cudaStream_t s,
                             Args &&...args) {
    return launch_maybe_dependent(true, kernel, grid, block, s, std::forward<Args>(args)...);
}

// kThree: the bf16 gather compiled for 3 resident CTAs per SM (see k_gather_bf16).
template <bool kTok, bool kThree = false>
cudaError_t launch_gather_kernel(ngram_dtype t, const GatherArgs &g, unsigned nb, cudaStream_t s, bool dep) {
    const bool h16 = g.h.n_heads == 16;
    switch (t) {
        case NGRAM_BF16:
            if (kThree) return h16 ? launch_maybe_dependent(dep, k_gather_bf16<16, kTok, 3>, nb, 256, s, g)
                                   : launch_maybe_dependent(dep, k_gather_bf16<0, kTok, 3>, nb, 256, s, g);
            return h16 ? launch_maybe_dependent(dep, k_gather_bf16<16, kTok>, nb, 256, s, g)
                       : launch_maybe_dependent(dep, k_gather_bf16<0, kTok>, nb, 256, s, g);
        case NGRAM_INT8_ROWSCALE:
            return h16 ? launch_maybe_dependent(dep, k_gather_int8<16, kTok>, nb, 256, s, g)
                       : launch_maybe_dependent(dep, k_gather_int8<0, kTok>, nb, 256, s, g);
        case NGRAM_FP8_E4M3_ROWSCALE:
            return h16 ? launch_maybe_dependent(dep, k_gather_fp8<16, kTok>, nb, 256, s, g)
                       : launch_maybe_dependent(dep, k_gather_fp8<0, kTok>, nb, 256, s, g);
        case NGRAM_NVFP4:
            return h16 ? launch_maybe_dependent(dep, k_gather_nvfp4<16, kTok>, nb, 256, s, g)
                       : launch_maybe_dependent(dep, k_gather_nvfp4<0, kTok>, nb, 256, s, g);
    }
    return cudaErrorInvalidValue;
}

// The TMA-staged gather of the 8- and 4-bit formats: whole rows through a shared-memory
// ring, one token per item (gather_staged.cuh).
template <class Rows>
ngram_status launch_staged_fmt(ngram_ctx *c, const GatherArgs &g, const StagedPlan &p, unsigned grid,
                               uint32_t smem, cudaStream_t s) {
    if (!c->staged_smem_set) {
        NG_CUDA(cudaFuncSetAttribute(k_gather_staged<16, Rows>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     NGRAM_STAGED_SMEM_BYTES), "cudaFuncSetAttribute (staged gather)");
        NG_CUDA(cudaFuncSetAttribute(k_gather_staged<0, Rows>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     NGRAM_STAGED_SMEM_BYTES), "cudaFuncSetAttribute (staged gather)");
        c->staged_smem_set = 1;
    }
    if (g.h.n_heads == 16) k_gather_staged<16, Rows><<<grid, 352, smem, s>>>(g, p);
    else k_gather_staged<0, Rows><<<grid, 352, smem, s>>>(g, p);
    NG_CUDA(cudaGetLastError(), "k_gather_staged launch");
    return NGRAM_OK;
}

ngram_status launch_staged(ngram_ctx *c, const GatherArgs &g, cudaStream_t s) {
    StagedPlan p;
    p.row_bytes = c->row_bytes;
    p.res_off = 16u * c->row_bytes;
    p.scale_off = p.res_off + 2u * c->d;
    p.stage_bytes = (p.scale_off + 64u + 127u) & ~127u;
    uint32_t stages = (NGRAM_STAGED_SMEM_BYTES - 128u) / p.stage_bytes;
    if (stages > kBulkMaxStages) stages = kBulkMaxStages;
    if (stages < 2) return fail(NGRAM_EUNSUPPORTED, "staged gather: stage of %u bytes too large", p.stage_bytes);
    p.stages = stages;
    const uint32_t smem = stages * p.stage_bytes + 128u;
    uint64_t grid = static_cast<uint64_t>(c->num_sms) * NGRAM_STAGED_CTAS_PER_SM;
    if (grid > g.N) grid = g.N;
    const unsigned nb = static_cast<unsigned>(grid);
    switch (c->dtype) {
        case NGRAM_INT8_ROWSCALE: return launch_staged_fmt<Rows8bit<Int8Codes>>(c, g, p, nb, smem, s);
        case NGRAM_FP8_E4M3_ROWSCALE: return launch_staged_fmt<Rows8bit<E4m3Codes>>(c, g, p, nb, smem, s);
        case NGRAM_NVFP4: return launch_staged_fmt<RowsNvfp4>(c, g, p, nb, smem, s);
        default: return fail(NGRAM_EUNSUPPORTED, "staged gather: bf16 uses the chunked TMA gather");
    }
}

uint64_t full_grid(const ngram_ctx *c);

// The register gather (every row format); max_blocks bounds the persistent grid.
ngram_status launch_gather(ngram_ctx *c, GatherArgs &g, cudaStream_t s, uint64_t max_blocks) {
    if ((c->hp.flags & NGRAM_FLAG_TMA_STAGING) && c->dtype != NGRAM_BF16 && c->where == NGRAM_RES_HBM &&
        g.row_ids == nullptr && g.gate_tok == nullptr && g.tok_begin == 0)
        return launch_staged(c, g, s);
    const uint64_t resident_warps = max_blocks * 8u;
    g.strips_per_item = (((NGRAM_SPI_ONE_FORMATS >> c->dtype) & 1u) ||
                         static_cast<uint64_t>(g.N) * g.n_strips <= 2ull * resident_warps) ? 1u : g.n_strips;
    g.groups_per_token = (g.n_strips + g.strips_per_item - 1) / g.strips_per_item;
    const uint64_t items = static_cast<uint64_t>(g.N) * g.groups_per_token;
    // a bf16 batch whose items overflow one wave of the full grid but fit one wave at 3
    // CTAs per SM (decode batches of ~240..350 tokens at d = 2560) runs the 3-CTA build:
    // otherwise the items beyond the first wave pay a second round of load latency
    const uint64_t three = static_cast<uint64_t>(c->num_sms) * 3u;
    const bool use_three = NGRAM_THREE_CTA_DECODE && c->dtype == NGRAM_BF16 &&
                           max_blocks == full_grid(c) && c->gather_blocks_per_sm < 3 &&
                           items > max_blocks * 8u && items <= three * 8u;
    uint64_t blocks = (items + 7) / 8;
    if (blocks > (use_three ? three : max_blocks)) blocks = use_three ? three : max_blocks;
    const unsigned nb = static_cast<unsigned>(blocks);
    // a full-grid gather launches as a programmatic dependent; a bounded grid (the
    // host-resident lookup that runs beside other work) launches plainly
    const bool dep = max_blocks == full_grid(c);
    g.trigger_early = dep ? 1u : 0u;
    cudaError_t e;
    if (g.gate_tok != nullptr) e = use_three ? launch_gather_kernel<true, true>(c->dtype, g, nb, s, dep)
                                             : launch_gather_kernel<true>(c->dtype, g, nb, s, dep);
    else e = use_three ? launch_gather_kernel<false, true>(c->dtype, g, nb, s, dep)
                       : launch_gather_kernel<false>(c->dtype, g, nb, s, dep);
    NG_CUDA(e, "gather kernel launch");
    return NGRAM_OK;
}

unsigned grid_for(const ngram_ctx *c, uint64_t work, uint32_t per_block) {
    uint64_t b = (work + per_block - 1) / per_block;
    const uint64_t cap = static_cast<uint64_t>(c->num_sms) * 8;
    if (b > cap) b = cap;
    if (b == 0) b = 1;
    return static_cast<unsigned>(b);
}

ngram_status launch_hash(ngram_ctx *c, const int32_t *tokens, const int32_t *history, uint32_t T,
                         uint32_t N, uint32_t *idx_out, cudaStream_t s) {
    const HashArgs a = hash_args(c);
    NG_CUDA(launch_dependent(k_hash_indices, grid_for(c, static_cast<uint64_t>(N) * a.n_heads, 256), 256, s,
                             a, tokens, history, T, N, c->d_err, idx_out),
            "k_hash_indices launch");
    return NGRAM_OK;
}

// Dedup idx[M] (device) into uniq/inv/count (device) with the context's scratch.
ngram_status launch_dedup(ngram_ctx *c, const uint32_t *idx, uint32_t M, uint32_t *uniq,
                          uint32_t *inv, uint32_t *count, cudaStream_t s) {
    const uint32_t log2p = std::max<uint32_t>(10u, ceil_log2(2ull * M));
    const uint32_t NB = (M + kScanBlock - 1) / kScanBlock;
    const unsigned gm = grid_for(c, M, 256);
    NG_CUDA(launch_dependent(k_dedup_insert, gm, 256, s, idx, M, c->d_keys, c->d_first, c->d_slot, log2p),
            "dedup launch");
    NG_CUDA(launch_dependent(k_dedup_scan_local, NB, 256, s, c->d_slot, c->d_first, M, c->d_pos, c->d_bsum),
            "dedup launch");
    NG_CUDA(launch_dependent(k_dedup_scan_blocks, 1, 1024, s, c->d_bsum, NB, count), "dedup launch");
    NG_CUDA(launch_dependent(k_dedup_emit, gm, 256, s, idx, c->d_slot, c->d_first, c->d_pos, c->d_bsum, M,
                             uniq, c->d_uid),
            "dedup launch");
    NG_CUDA(launch_dependent(k_dedup_inverse, gm, 256, s, c->d_slot, c->d_uid, M, inv), "dedup launch");
    return NGRAM_OK;
}

// The two tables the dedup of M indices starts from, cleared (every slot empty).  Issued
// before the hash kernel, so that the hash and dedup kernels follow one another directly
// and each may be launched as a programmatic dependent of the one before.
ngram_status dedup_clear(ngram_ctx *c, uint32_t M, cudaStream_t s) {
    const uint32_t log2p = std::max<uint32_t>(10u, ceil_log2(2ull * M));
    const uint64_t P = 1ull << log2p;
    NG_CUDA(cudaMemsetAsync(c->d_keys, 0xFF, P * 4ull, s), "dedup clear");
    NG_CUDA(cudaMemsetAsync(c->d_first, 0xFF, P * 4ull, s), "dedup clear");
    return NGRAM_OK;
}

// Hash the N tokens' M = N * H row indices into c->d_idx, then dedup them.
ngram_status launch_hash_dedup(ngram_ctx *c, const int32_t *tokens, const int32_t *history, uint32_t T,
                               uint32_t N, uint32_t *uniq, uint32_t *inv, uint32_t *count, cudaStream_t s) {
    const uint32_t M = N * c->H;
    NG_CHECK(dedup_clear(c, M, s));
    NG_CHECK(launch_hash(c, tokens, history, T, N, c->d_idx, s));
    return launch_dedup(c, c->d_idx, M, uniq, inv, count, s);
}

// ---------------------------------------------------------------- forward paths
struct Call {
    const int32_t *tokens, *history;
    uint32_t T, N;
    const uint16_t *residual;
    const void *gate;
    uint16_t *out;
    cudaStream_t s;
};

// All SMs, every resident CTA: the grid of the HBM-resident gathers.
uint64_t full_grid(const ngram_ctx *c) {
    return static_cast<uint64_t>(c->num_sms) * static_cast<uint64_t>(c->gather_blocks_per_sm);
}

ngram_status forward_direct(ngram_ctx *c, const Call &k, uint64_t max_blocks) {
    GatherArgs g = gather_args(c, k.tokens, k.history, k.T, k.N, k.residual, k.gate, k.out);
    if ((c->hp.flags & NGRAM_FLAG_TMA_STAGING) && c->dtype == NGRAM_BF16 && c->where == NGRAM_RES_HBM)
        return launch_bulk(c, g, k.s);
    return launch_gather(c, g, k.s, max_blocks);
}

// hash -> dedup -> compact the unique rows into HBM staging -> gather from staging.
// compact_grid: CTAs of the copy kernel (a full grid from HBM; NGRAM_UVA_COPY_CTAS from host
// memory, where each distinct row then crosses PCIe once).
ngram_status forward_dedup(ngram_ctx *c, const Call &k, unsigned compact_grid) {
    NG_CHECK(ensure_dedup_scratch(c));
    NG_CHECK(ensure_device_stage(c));
    NG_CHECK(launch_hash_dedup(c, k.tokens, k.history, k.T, k.N, c->d_uniq, c->d_inv, c->d_count, k.s));
    k_compact_rows<<<compact_grid, 256, 0, k.s>>>(
        static_cast<const uint8_t *>(c->table_dev), staged_scale_src(c), c->d_uniq, c->d_count,
        c->row_bytes, c->d_stage, c->d_stage_scale);
    NG_CUDA(cudaGetLastError(), "k_compact_rows launch");
    GatherArgs g = gather_args(c, k.tokens, k.history, k.T, k.N, k.residual, k.gate, k.out);
    g.table = c->d_stage;
    g.row_scale = staged_scale(c, c->d_stage_scale);
    g.row_ids = c->d_inv;
    return launch_gather(c, g, k.s, full_grid(c));
}

// One table row into pinned staging by a host thread.  NGRAM_DMA_NONTEMPORAL (x86-64):
//   0  memcpy;
//   1  the source lines are read after a non-temporal prefetch and the staging lines are
//      written with streaming stores;
//   2  as 1, and every source line is then flushed from the caches (clflushopt, where the
//      CPU has it), so no table row stays in the private caches of the copying cores.
// Rows left in those caches (worker threads that then go idle) made every later GPU read of
// them over PCIe (UVA, or UVA + dedup) 2.4x slower until the cores slept deeper.  bytes and
// both addresses are multiples of 16.
#ifndef NGRAM_DMA_NONTEMPORAL
#define NGRAM_DMA_NONTEMPORAL 2
#endif
#if defined(__x86_64__)
bool cpu_has_clflushopt() {
    unsigned a = 0, b = 0, c = 0, d = 0;
    if (!__get_cpuid_count(7, 0, &a, &b, &c, &d)) return false;
    return (b >> 23) & 1u;                     // CPUID.(EAX=7, ECX=0):EBX[23]
}
const bool g_clflushopt = cpu_has_clflushopt();

// Every 64-byte line that [p, p + bytes) touches, the partial lines at both ends included.
__attribute__((target("clflushopt"))) void flush_lines(const uint8_t *p, uint32_t bytes) {
    const uintptr_t end = reinterpret_cast<uintptr_t>(p) + bytes;
    for (uintptr_t a = reinterpret_cast<uintptr_t>(p) & ~uintptr_t(63); a < end; a += 64)
        _mm_clflushopt(reinterpret_cast<void *>(a));
}
#endif
inline void copy_row_to_staging(uint8_t *dst, const uint8_t *src, uint32_t bytes) {
#if defined(__x86_64__) && NGRAM_DMA_NONTEMPORAL
    for (uint32_t o = 0; o < bytes; o += 64)
        _mm_prefetch(reinterpret_cast<const char *>(src + o), _MM_HINT_NTA);
    for (uint32_t o = 0; o < bytes; o += 16)
        _mm_stream_si128(reinterpret_cast<__m128i *>(dst + o),
                         _mm_load_si128(reinterpret_cast<const __m128i *>(src + o)));
    if (NGRAM_DMA_NONTEMPORAL >= 2 && g_clflushopt) flush_lines(src, bytes);
#else
    memcpy(dst, src, bytes);
#endif
}

// Host-resident, copy-engine path: the unique rows are compacted by host threads
// into pinned staging and moved to HBM by cudaMemcpyAsync in chunks (the copy of
// chunk i overlaps the host gather of chunk i+1), then gathered from HBM.
ngram_status forward_dma(ngram_ctx *c, const Call &k) {
    NG_CHECK(ensure_dedup_scratch(c));
    NG_CHECK(ensure_host_stage(c));
    const uint32_t M = k.N * c->H;
    NG_CHECK(launch_hash_dedup(c, k.tokens, k.history, k.T, k.N, c->d_uniq, c->d_inv, c->d_count, k.s));
    if (c->stage_in_use) NG_CHECK(wait_event(c, c->ev_stage_free, "DMA: previous staging copy"));
    NG_CUDA(cudaMemcpyAsync(c->h_count, c->d_count, 4, cudaMemcpyDeviceToHost, k.s), "D2H count");
    NG_CUDA(cudaMemcpyAsync(c->h_uniq, c->d_uniq, M * 4ull, cudaMemcpyDeviceToHost, k.s), "D2H rows");
    NG_CUDA(cudaEventRecord(c->ev_sync, k.s), "cudaEventRecord");
    NG_CHECK(wait_event(c, c->ev_sync, "DMA: unique-row list"));
    const uint32_t U = *c->h_count;
    if (U > M) return fail(NGRAM_ECUDA, "DMA: unique count %u exceeds %u entries", U, M);
    for (uint32_t u = 0; u < U; ++u)        // host threads read the table: check every row id
        if (c->h_uniq[u] >= c->R)
            return fail(NGRAM_ECUDA, "DMA: row id %u out of range %llu", c->h_uniq[u],
                        static_cast<unsigned long long>(c->R));
    const uint8_t *table = static_cast<const uint8_t *>(c->table);
    const uint32_t rb = c->row_bytes;
    const uint32_t chunk_rows = std::max<uint32_t>(1u, NGRAM_DMA_CHUNK_BYTES / rb);
    for (uint32_t r0 = 0; r0 < U; r0 += chunk_rows) {
        const uint32_t r1 = std::min(U, r0 + chunk_rows);
#pragma omp parallel if (r1 - r0 >= 256)
        {
#pragma omp for schedule(static)
            for (int64_t u = r0; u < static_cast<int64_t>(r1); ++u) {
                copy_row_to_staging(c->h_stage + static_cast<size_t>(u) * rb,
                                    table + static_cast<size_t>(c->h_uniq[u]) * rb, rb);
                if (c->h_stage_scale) c->h_stage_scale[u] = c->row_scale[c->h_uniq[u]];
            }
#if defined(__x86_64__) && NGRAM_DMA_NONTEMPORAL
            _mm_sfence();                     // this thread's streaming stores are visible
#endif
        }
        NG_CUDA(cudaMemcpyAsync(c->d_stage + static_cast<size_t>(r0) * rb,
                                c->h_stage + static_cast<size_t>(r0) * rb,
                                static_cast<size_t>(r1 - r0) * rb, cudaMemcpyHostToDevice, k.s),
                "H2D staging");
    }
    if (c->h_stage_scale && U > 0)
        NG_CUDA(cudaMemcpyAsync(c->d_stage_scale, c->h_stage_scale, U * 4ull, cudaMemcpyHostToDevice, k.s),
                "H2D scales");
    NG_CUDA(cudaEventRecord(c->ev_stage_free, k.s), "cudaEventRecord");
    c->stage_in_use = 1;
    GatherArgs g = gather_args(c, k.tokens, k.history, k.T, k.N, k.residual, k.gate, k.out);
    g.table = c->d_stage;
    g.row_scale = staged_scale(c, c->d_stage_scale);
    g.row_ids = c->d_inv;
    return launch_gather(c, g, k.s, full_grid(c));
}

// UVA: the same kernel reading host rows over PCIe.  A bounded grid suffices to keep
// PCIe busy and leaves the other SMs to whatever runs beside the lookup.
// Whether an HBM batch of N tokens is gathered in grouped order: always with
// NGRAM_FLAG_SORT, never with NGRAM_FLAG_BATCH_ORDER or TMA staging, else from
// NGRAM_SORT_MIN_TOKENS tokens on.
bool grouped_order(const ngram_ctx *c, uint32_t N) {
    const uint32_t f = c->hp.flags;
    if (f & NGRAM_FLAG_SORT) return true;
    if (f & NGRAM_FLAG_BATCH_ORDER) return false;
    if ((f & NGRAM_FLAG_TMA_STAGING) && c->dtype == NGRAM_BF16) return false;
    return N >= NGRAM_SORT_MIN_TOKENS;
}

// Grouped order: tokens grouped by bigram context (counting sort on a 13-bit hash),
// then the fused gather walks them in that order.  Same outputs; repeated rows run back
// to back so L2 serves the repeats.
// Grouped order of a batch's tokens into c->so_perm (3 kernels and a memset).
// idx_out: also write every token's row ids [N][H] in the same pass, or null.
ngram_status order_tokens(ngram_ctx *c, const Call &k, uint32_t *idx_out = nullptr) {
    NG_CHECK(dev_alloc(&c->so_bucket, c->max_tokens * 4ull, "order scratch"));
    NG_CHECK(dev_alloc(&c->so_hist, kOrderBuckets * 4ull, "order scratch"));
    NG_CHECK(dev_alloc(&c->so_perm, c->max_tokens * 4ull, "order scratch"));
    const HashArgs a = hash_args(c);
    const unsigned gn = grid_for(c, k.N, 256);
    NG_CUDA(cudaMemsetAsync(c->so_hist, 0, kOrderBuckets * 4ull, k.s), "order clear");
    const int32_t *tokens = k.tokens, *history = k.history;
    const uint32_t T = k.T, N = k.N;
    uint32_t *err = c->d_err, *bucket = c->so_bucket, *hist = c->so_hist, *perm = c->so_perm;
    const uint32_t *bucket_c = bucket;
    NG_CUDA(launch_dependent(k_order_count, gn, 256, k.s, tokens, history, T, N, a, err, bucket, hist,
                             idx_out), "k_order_count launch");
    NG_CUDA(launch_dependent(k_order_scan, 1, 1024, k.s, hist), "k_order_scan launch");
    NG_CUDA(launch_dependent(k_order_scatter, gn, 256, k.s, bucket_c, N, hist, perm), "k_order_scatter launch");
    return NGRAM_OK;
}

// NGRAM_PREHASH_FORMATS bit t: on grouped batches of at least NGRAM_PREHASH_MIN_TOKENS
// tokens in HBM, row format t hashes every token once -- k_order_count writes its row ids
// [N][H] (64 B per token) beside the bucket counts -- and the gather reads the row ids
// instead of hashing in every work item.  It pays for the formats whose work item is one
// strip of a token (bf16: 10 strips, NVFP4: 5), which otherwise hash each token once per
// strip: measured on B200 with a separate hash kernel, NVFP4 prefill 133.4 -> 140.2 M
// tokens/s, bf16 prefill 75.6 -> 76.6 M.  int8 and FP8 walk a token's strips in one warp
// and hash once anyway (with the separate kernel 110.6 -> 108.5 and 114.0 -> 112.1 M).
#ifndef NGRAM_PREHASH_FORMATS
#define NGRAM_PREHASH_FORMATS ((1u << NGRAM_BF16) | (1u << NGRAM_NVFP4))
#endif
#ifndef NGRAM_PREHASH_MIN_TOKENS
#define NGRAM_PREHASH_MIN_TOKENS 4096u
#endif

ngram_status forward_sorted(ngram_ctx *c, const Call &k, uint64_t max_blocks) {
    const bool prehash = ((NGRAM_PREHASH_FORMATS >> c->dtype) & 1u) && c->where == NGRAM_RES_HBM &&
                         k.N >= NGRAM_PREHASH_MIN_TOKENS;
    if (prehash) NG_CHECK(dev_alloc(&c->d_rowid, c->dd_cap * 4ull, "row-id buffer"));
    NG_CHECK(order_tokens(c, k, prehash ? c->d_rowid : nullptr));
    GatherArgs g = gather_args(c, k.tokens, k.history, k.T, k.N, k.residual, k.gate, k.out);
    g.perm = c->so_perm;
    if (prehash) g.row_ids = c->d_rowid;
    return launch_gather(c, g, k.s, max_blocks);
}

ngram_status forward_dedup_hbm(ngram_ctx *c, const Call &k) {
    return forward_dedup(c, k, grid_for(c, static_cast<uint64_t>(k.N) * c->H * 32ull, 256));
}

// UVA with dedup: each distinct row crosses PCIe once, read by the copy kernel.
ngram_status forward_dedup_uva(ngram_ctx *c, const Call &k) {
    return forward_dedup(c, k, static_cast<unsigned>(std::min<uint64_t>(NGRAM_UVA_COPY_CTAS, full_grid(c))));
}

// UVA without dedup: the gather kernel reads the host rows itself, on a bounded grid.
ngram_status forward_direct_uva(ngram_ctx *c, const Call &k) {
    const uint64_t blocks = std::min<uint64_t>(NGRAM_UVA_CTAS, full_grid(c));
    if (c->hp.flags & NGRAM_FLAG_SORT) return forward_sorted(c, k, blocks);
    return forward_direct(c, k, blocks);
}

ngram_status forward_uva(ngram_ctx *c, const Call &k) {
    if (c->hp.flags & NGRAM_FLAG_DEDUP) return forward_dedup_uva(c, k);
    return forward_direct_uva(c, k);
}

// AUTO: the first call of each batch-size bucket runs the three host modes (UVA, UVA with
// dedup, DMA; all write the same output), each once untimed (the first call of a mode
// also allocates its staging) and then kNAutoTimed times timed in interleaved rounds,
// keeps the mode with the lowest median time, and later calls use it.  auto_choice holds NGRAM_RES_HOST_UVA,
// NGRAM_RES_HOST_DMA or NGRAM_AUTO_UVA_DEDUP.
constexpr int kNAutoTimed = 3;

ngram_status run_mode(ngram_ctx *c, const Call &k, int mode) {
    if (mode == NGRAM_RES_HOST_UVA) return forward_direct_uva(c, k);
    if (mode == NGRAM_AUTO_UVA_DEDUP) return forward_dedup_uva(c, k);
    return forward_dma(c, k);
}

ngram_status time_mode(ngram_ctx *c, const Call &k, int mode, float *ms) {
    const auto h0 = std::chrono::steady_clock::now();
    NG_CUDA(cudaEventRecord(c->ev_t0, k.s), "cudaEventRecord");
    NG_CHECK(run_mode(c, k, mode));
    NG_CUDA(cudaEventRecord(c->ev_t1, k.s), "cudaEventRecord");
    NG_CHECK(wait_event(c, c->ev_t1, "AUTO: timing"));
    NG_CUDA(cudaEventElapsedTime(ms, c->ev_t0, c->ev_t1), "cudaEventElapsedTime");
    if (mode == NGRAM_RES_HOST_DMA) {      // DMA blocks the host while it stages rows
        const float wall =
            std::chrono::duration<float, std::milli>(std::chrono::steady_clock::now() - h0).count();
        *ms = std::max(*ms, wall);
    }
    return NGRAM_OK;
}

ngram_status forward_auto(ngram_ctx *c, const Call &k) {
    const uint32_t b = ceil_log2(k.N);
    if (c->auto_choice[b] == NGRAM_RES_HOST_UVA) return forward_direct_uva(c, k);
    if (c->auto_choice[b] == NGRAM_AUTO_UVA_DEDUP) return forward_dedup_uva(c, k);
    if (c->auto_choice[b] == NGRAM_RES_HOST_DMA) return forward_dma(c, k);
    NG_CHECK(event_once(&c->ev_t0, cudaEventDefault));
    NG_CHECK(event_once(&c->ev_t1, cudaEventDefault));
    const int modes[3] = {NGRAM_RES_HOST_UVA, NGRAM_AUTO_UVA_DEDUP, NGRAM_RES_HOST_DMA};
    for (int m = 0; m < 3; ++m) NG_CHECK(run_mode(c, k, modes[m]));    // warm-up: staging, caches
    // timed rounds interleave the modes, so a slow spell of the host or the link costs
    // every mode alike instead of the one that happened to run then
    float t[3][kNAutoTimed];
    for (int r = 0; r < kNAutoTimed; ++r)
        for (int m = 0; m < 3; ++m) NG_CHECK(time_mode(c, k, modes[m], &t[m][r]));
    int best = NGRAM_RES_HOST_UVA;
    float t_best = 0.f;
    for (int m = 0; m < 3; ++m) {
        std::sort(t[m], t[m] + kNAutoTimed);
        const float med = t[m][kNAutoTimed / 2];
        if (m == 0 || med < t_best) { best = modes[m]; t_best = med; }
    }
    c->auto_choice[b] = best;
    return NGRAM_OK;
}

}  // namespace

extern "C" {

ngram_status ngram_default_hash_params(ngram_hash_params *hp) {
    if (hp == nullptr) return fail(NGRAM_EINVAL, "hp is NULL");
    hp->base_seed = NGRAM_DEFAULT_BASE_SEED;
    hp->n_bigram_heads = 8;
    hp->n_trigram_heads = 8;
    hp->pad_id = NGRAM_DEFAULT_PAD_ID;
    hp->vocab_size = kTokenMask;
    hp->flags = 0;
    hp->reserved = 0;
    return NGRAM_OK;
}

const char *ngram_last_error(void) { return g_last_error.c_str(); }

const char *ngram_status_string(ngram_status s) {
    switch (s) {
        case NGRAM_OK: return "NGRAM_OK";
        case NGRAM_EINVAL: return "NGRAM_EINVAL";
        case NGRAM_ENOMEM: return "NGRAM_ENOMEM";
        case NGRAM_ECUDA: return "NGRAM_ECUDA";
        case NGRAM_EUNSUPPORTED: return "NGRAM_EUNSUPPORTED";
        case NGRAM_ETIMEOUT: return "NGRAM_ETIMEOUT";
        case NGRAM_EDEVICE: return "NGRAM_EDEVICE";
    }
    return "NGRAM_UNKNOWN";
}

ngram_status ngram_host_alloc(void **out, uint64_t bytes) {
    if (out == nullptr) return fail(NGRAM_EINVAL, "out is NULL");
    *out = nullptr;
    if (bytes == 0) return fail(NGRAM_EINVAL, "bytes must be > 0");
    NG_CUDA(cudaHostAlloc(out, bytes, cudaHostAllocMapped | cudaHostAllocPortable), "cudaHostAlloc");
    return NGRAM_OK;
}

ngram_status ngram_host_free(void *p) {
    if (p == nullptr) return NGRAM_OK;
    NG_CUDA(cudaFreeHost(p), "cudaFreeHost");
    return NGRAM_OK;
}

ngram_status ngram_row_bytes(ngram_dtype dtype, uint32_t d, uint32_t *out) {
    if (out == nullptr) return fail(NGRAM_EINVAL, "out is NULL");
    const float one = 1.0f;
    NG_CHECK(check_format(dtype, d, dtype == NGRAM_BF16 ? nullptr : &one));
    *out = row_bytes_of(dtype, d);
    return NGRAM_OK;
}

ngram_status ngram_init(ngram_ctx **out, const void *table, const float *row_scale, uint64_t R,
                        uint32_t d, ngram_dtype dtype, ngram_residency where,
                        const ngram_hash_params *hp, uint32_t max_tokens) {
    if (out == nullptr) return fail(NGRAM_EINVAL, "out is NULL");
    *out = nullptr;
    if (table == nullptr) return fail(NGRAM_EINVAL, "table is NULL");
    if (!aligned16(table)) return fail(NGRAM_EINVAL, "table must be 16-byte aligned");
    if (R == 0 || R > 0xFFFFFFFFull) return fail(NGRAM_EINVAL, "R must be in [1, 2^32 - 1]");
    NG_CHECK(check_format(dtype, d, row_scale));
    if (where != NGRAM_RES_HBM && where != NGRAM_RES_HOST_UVA && where != NGRAM_RES_HOST_DMA &&
        where != NGRAM_RES_HOST_AUTO)
        return fail(NGRAM_EINVAL, "unknown residency %d", static_cast<int>(where));
    if (max_tokens == 0) return fail(NGRAM_EINVAL, "max_tokens must be >= 1");
    ngram_hash_params p;
    if (hp != nullptr) p = *hp; else ngram_default_hash_params(&p);
    NG_CHECK(check_hash_params(p));
    const uint32_t H = p.n_bigram_heads + p.n_trigram_heads;
    const uint32_t n_strips = (d / 8 + 31) / 32;
    if (static_cast<uint64_t>(max_tokens) * n_strips > 0xFFFFFFFFull ||
        static_cast<uint64_t>(max_tokens) * NGRAM_MAX_HEADS > (1ull << 30))
        return fail(NGRAM_EINVAL, "max_tokens %u too large for d = %u", max_tokens, d);
    if ((p.flags & NGRAM_FLAG_DEDUP) && where != NGRAM_RES_HBM && where != NGRAM_RES_HOST_UVA)
        return fail(NGRAM_EINVAL, "NGRAM_FLAG_DEDUP applies to HBM and HOST_UVA residency (DMA always dedups, AUTO tries both)");
    if ((p.flags & NGRAM_FLAG_SORT) && where != NGRAM_RES_HBM && where != NGRAM_RES_HOST_UVA)
        return fail(NGRAM_EINVAL, "NGRAM_FLAG_SORT applies to HBM and HOST_UVA residency");
    if ((p.flags & NGRAM_FLAG_SORT) &&
        (p.flags & (NGRAM_FLAG_DEDUP | NGRAM_FLAG_TMA_STAGING | NGRAM_FLAG_BATCH_ORDER)))
        return fail(NGRAM_EINVAL, "NGRAM_FLAG_SORT does not combine with DEDUP, TMA_STAGING or BATCH_ORDER");
    if ((p.flags & NGRAM_FLAG_TOKEN_GATE) && (p.flags & NGRAM_FLAG_TMA_STAGING))
        return fail(NGRAM_EINVAL, "NGRAM_FLAG_TOKEN_GATE does not combine with TMA_STAGING");

    // ---- CUDA from here on
    ngram_ctx *c = new ngram_ctx();
    memset(c, 0, sizeof(*c));
    c->table = table;
    c->table_dev = table;
    c->row_scale = scale_per_row(dtype) ? row_scale : nullptr;
    c->row_scale_dev = c->row_scale;
    c->R = R;
    c->d = d;
    c->row_bytes = row_bytes_of(dtype, d);
    c->dtype = dtype;
    c->where = where;
    c->hp = p;
    c->H = H;
    c->max_tokens = max_tokens;
    c->barrett_m = (R == 1) ? 0ull
                            : static_cast<uint64_t>((static_cast<unsigned __int128>(1) << 64) / R);
    c->wait_ms = 10000;
    c->dd_cap = max_tokens * H;
    c->dd_pcap = 1u << std::max<uint32_t>(10u, ceil_log2(2ull * c->dd_cap));
    ngram_status st = NGRAM_OK;
    cudaError_t e = cudaGetDevice(&c->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
    if (e == cudaSuccess) {
        int *bps = &c->gather_blocks_per_sm;
        switch (dtype) {
            case NGRAM_BF16: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(bps, k_gather_bf16<16>, 256, 0); break;
            case NGRAM_INT8_ROWSCALE: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(bps, k_gather_int8<16>, 256, 0); break;
            case NGRAM_FP8_E4M3_ROWSCALE: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(bps, k_gather_fp8<16>, 256, 0); break;
            case NGRAM_NVFP4: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(bps, k_gather_nvfp4<16>, 256, 0); break;
        }
    }
    if (e == cudaSuccess) e = cudaMalloc(&c->d_err, 4 * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemset(c->d_err, 0, 4 * sizeof(uint32_t));
    if (e == cudaSuccess && dtype == NGRAM_NVFP4) {   // the global scale, from host or device memory
        e = cudaMalloc(&c->d_gscale, sizeof(float));
        if (e == cudaSuccess) e = cudaMemcpy(c->d_gscale, row_scale, sizeof(float), cudaMemcpyDefault);
        c->row_scale_dev = c->d_gscale;
    }
    if (e != cudaSuccess) st = cuda_fail(e, "ngram_init");
    if (st == NGRAM_OK && where != NGRAM_RES_HBM) {
        cudaPointerAttributes attr;
        e = cudaPointerGetAttributes(&attr, table);
        if (e != cudaSuccess) {
            st = cuda_fail(e, "cudaPointerGetAttributes(table)");
        } else if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) {
            st = fail(NGRAM_EINVAL, "host residency needs a host table, got device memory");
        } else if (where != NGRAM_RES_HOST_DMA) {
            // UVA / AUTO: the kernel reads the table itself, so it must be pinned and mapped
            if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr)
                st = fail(NGRAM_EINVAL, "UVA needs pinned, mapped host memory (ngram_host_alloc)");
            else
                c->table_dev = attr.devicePointer;
            if (st == NGRAM_OK && c->row_scale != nullptr) {
                e = cudaPointerGetAttributes(&attr, row_scale);
                if (e != cudaSuccess || attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr)
                    st = fail(NGRAM_EINVAL, "UVA needs row_scale in pinned, mapped host memory");
                else
                    c->row_scale_dev = static_cast<const float *>(attr.devicePointer);
            }
        }
    }
    if (st != NGRAM_OK) {
        free_all(c);
        delete c;
        return st;
    }
    if (c->gather_blocks_per_sm < 1) c->gather_blocks_per_sm = 1;
    *out = c;
    return NGRAM_OK;
}

ngram_status ngram_set_wait_timeout(ngram_ctx *c, uint32_t ms) {
    if (c == nullptr) return fail(NGRAM_EINVAL, "ctx is NULL");
    if (ms == 0) return fail(NGRAM_EINVAL, "timeout must be > 0 ms");
    c->wait_ms = ms;
    return NGRAM_OK;
}

ngram_status ngram_forward(ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                           uint32_t n_seq, uint32_t T, const uint16_t *residual, const void *gate,
                           uint16_t *out, ngram_stream_t stream) {
    uint64_t N = 0;
    NG_CHECK(check_batch(c, tokens, n_seq, T, &N));
    if (N == 0) return NGRAM_OK;
    if (residual == nullptr || gate == nullptr || out == nullptr)
        return fail(NGRAM_EINVAL, "residual, gate and out must be non-NULL");
    if (!aligned16(residual) || !aligned16(gate) || !aligned16(out))
        return fail(NGRAM_EINVAL, "residual, gate and out must be 16-byte aligned");
    if (out != residual) {
        const uint64_t bytes = N * c->d * 2ull;
        const uintptr_t a = reinterpret_cast<uintptr_t>(out), b = reinterpret_cast<uintptr_t>(residual);
        if (a < b + bytes && b < a + bytes)
            return fail(NGRAM_EINVAL, "out overlaps residual without being equal to it");
    }
    const Call k{tokens, history, T, static_cast<uint32_t>(N), residual, gate, out,
                 reinterpret_cast<cudaStream_t>(stream)};
    switch (c->where) {
        case NGRAM_RES_HBM:
            if (c->hp.flags & NGRAM_FLAG_DEDUP) return forward_dedup_hbm(c, k);
            if (grouped_order(c, k.N)) return forward_sorted(c, k, full_grid(c));
            return forward_direct(c, k, full_grid(c));
        case NGRAM_RES_HOST_UVA: return forward_uva(c, k);
        case NGRAM_RES_HOST_DMA: return forward_dma(c, k);
        case NGRAM_RES_HOST_AUTO: return forward_auto(c, k);
    }
    return fail(NGRAM_EINVAL, "bad residency");
}

ngram_status ngram_forward_host(ngram_ctx *c, const int32_t *tokens_h, const int32_t *history_h,
                                uint32_t n_seq, uint32_t T, const uint16_t *residual_h,
                                const float *gate, uint16_t *out_h, ngram_stream_t stream) {
    uint64_t N = 0;
    NG_CHECK(check_batch(c, tokens_h, n_seq, T, &N));
    if (N == 0) return NGRAM_OK;
    if (residual_h == nullptr || gate == nullptr || out_h == nullptr)
        return fail(NGRAM_EINVAL, "residual, gate and out must be non-NULL");
    if (!aligned16(gate)) return fail(NGRAM_EINVAL, "gate must be 16-byte aligned");
    {   // the chunks' copies in and out may run in any order across streams
        const uint64_t bytes = N * c->d * 2ull;
        const uintptr_t a = reinterpret_cast<uintptr_t>(out_h), b = reinterpret_cast<uintptr_t>(residual_h);
        if (a < b + bytes && b < a + bytes) return fail(NGRAM_EINVAL, "out overlaps residual");
    }
    if ((c->hp.flags & (NGRAM_FLAG_DEDUP | NGRAM_FLAG_TMA_STAGING | NGRAM_FLAG_SORT |
                        NGRAM_FLAG_TOKEN_GATE)) ||  // chunks keep batch order
        (c->where != NGRAM_RES_HBM && c->where != NGRAM_RES_HOST_UVA))
        return fail(NGRAM_EUNSUPPORTED,
                    "ngram_forward_host pipelines the fused gather: HBM or HOST_UVA residency, no flags");
    NG_CHECK(ensure_host_path(c));
    constexpr int S = NGRAM_HOST_BUFFERS;
    cudaStream_t caller = reinterpret_cast<cudaStream_t>(stream);
    const uint64_t row = 2ull * c->d;
    const uint64_t max_blocks = (c->where == NGRAM_RES_HOST_UVA)
        ? std::min<uint64_t>(NGRAM_UVA_CTAS, full_grid(c)) : full_grid(c);
    // every pipeline stream starts after the caller's earlier work; stream 0 uploads the
    // tokens once the previous call's kernels (on every stream) have stopped reading them
    NG_CUDA(cudaEventRecord(c->hp_entry, caller), "cudaEventRecord");
    for (int i = 0; i < S; ++i) NG_CUDA(cudaStreamWaitEvent(c->hp_s[i], c->hp_entry, 0), "cudaStreamWaitEvent");
    for (int i = 1; i < S; ++i) NG_CUDA(cudaStreamWaitEvent(c->hp_s[0], c->hp_d2h[i], 0), "cudaStreamWaitEvent");
    NG_CUDA(cudaMemcpyAsync(c->hp_tok, tokens_h, N * 4, cudaMemcpyHostToDevice, c->hp_s[0]), "H2D tokens");
    if (history_h)
        NG_CUDA(cudaMemcpyAsync(c->hp_hist, history_h, n_seq * 8ull, cudaMemcpyHostToDevice, c->hp_s[0]),
                "H2D history");
    NG_CUDA(cudaEventRecord(c->hp_h2d[0], c->hp_s[0]), "cudaEventRecord");
    for (int i = 1; i < S; ++i) NG_CUDA(cudaStreamWaitEvent(c->hp_s[i], c->hp_h2d[0], 0), "cudaStreamWaitEvent");
    GatherArgs g = gather_args(c, c->hp_tok, history_h ? c->hp_hist : nullptr, T, 0, nullptr, gate,
                               nullptr);
    // chunk i runs on stream i % S, start to end: H2D residual -> gather -> D2H out.  The
    // S streams overlap each other's copies in both directions; stream order alone makes
    // a stream's buffers safe to reuse.
    std::vector<uint32_t> sizes;
    host_chunks(N, c->hp_chunk, sizes);
    uint64_t t0 = 0;
    for (size_t chunk_i = 0; chunk_i < sizes.size(); t0 += sizes[chunk_i], ++chunk_i) {
        const int b = static_cast<int>(chunk_i % S);
        cudaStream_t st = c->hp_s[b];
        const uint32_t n = sizes[chunk_i];
        NG_CUDA(cudaMemcpyAsync(c->hp_res[b], residual_h + t0 * c->d, n * row, cudaMemcpyHostToDevice, st),
                "H2D residual");
        g.tok_begin = static_cast<uint32_t>(t0);
        g.N = n;
        g.residual = c->hp_res[b];
        g.out = c->hp_out[b];
        NG_CHECK(launch_gather(c, g, st, max_blocks));
        NG_CUDA(cudaMemcpyAsync(out_h + t0 * c->d, c->hp_out[b], n * row, cudaMemcpyDeviceToHost, st),
                "D2H out");
    }
    // the caller's stream resumes once every stream's last output chunk is on the host
    for (int i = 0; i < S; ++i) {
        NG_CUDA(cudaEventRecord(c->hp_d2h[i], c->hp_s[i]), "cudaEventRecord");
        NG_CUDA(cudaStreamWaitEvent(caller, c->hp_d2h[i], 0), "cudaStreamWaitEvent");
    }
    return NGRAM_OK;
}

ngram_status ngram_prefetch(ngram_ctx *c, uint32_t slot, const int32_t *tokens, const int32_t *history,
                            uint32_t n_seq, uint32_t T, ngram_stream_t stream) {
    uint64_t N = 0;
    NG_CHECK(check_batch(c, tokens, n_seq, T, &N));
    if (slot >= NGRAM_STAGE_SLOTS)
        return fail(NGRAM_EINVAL, "slot %u out of range (%u slots)", slot, NGRAM_STAGE_SLOTS);
    if (c->where == NGRAM_RES_HOST_DMA)
        return fail(NGRAM_EUNSUPPORTED, "ngram_prefetch reads the table from the GPU: HBM, HOST_UVA or HOST_AUTO");
    auto &sl = c->slot[slot];
    sl.epoch = 0;                    // the slot holds no batch until this call has issued its work
    sl.n_seq = n_seq;
    sl.T = T;
    if (N == 0) {
        sl.epoch = ++c->prefetch_epoch;
        return NGRAM_OK;
    }
    NG_CHECK(ensure_dedup_scratch(c));
    NG_CHECK(dev_alloc(&sl.inv, c->dd_cap * 4ull, "staging slot"));
    NG_CHECK(dev_alloc(&sl.stage, static_cast<size_t>(c->dd_cap) * c->row_bytes, "staging slot"));
    if (scale_per_row(c->dtype)) NG_CHECK(dev_alloc(&sl.stage_scale, c->dd_cap * 4ull, "staging slot"));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint32_t M = static_cast<uint32_t>(N) * c->H;
    NG_CHECK(launch_hash_dedup(c, tokens, history, T, static_cast<uint32_t>(N), c->d_uniq, sl.inv, c->d_count, s));
    // each distinct row crosses once; from host memory a few CTAs keep PCIe busy
    const unsigned grid = (c->where == NGRAM_RES_HBM) ? grid_for(c, M * 32ull, 256)
                                                      : static_cast<unsigned>(NGRAM_UVA_COPY_CTAS);
    k_compact_rows<<<grid, 256, 0, s>>>(static_cast<const uint8_t *>(c->table_dev), staged_scale_src(c),
                                        c->d_uniq, c->d_count, c->row_bytes, sl.stage, sl.stage_scale);
    NG_CUDA(cudaGetLastError(), "k_compact_rows launch");
    sl.epoch = ++c->prefetch_epoch;
    return NGRAM_OK;
}

ngram_status ngram_forward_staged(ngram_ctx *c, uint32_t slot, const uint16_t *residual,
                                  const void *gate, uint16_t *out, ngram_stream_t stream) {
    if (c == nullptr) return fail(NGRAM_EINVAL, "ctx is NULL");
    if (slot >= NGRAM_STAGE_SLOTS)
        return fail(NGRAM_EINVAL, "slot %u out of range (%u slots)", slot, NGRAM_STAGE_SLOTS);
    const auto &sl = c->slot[slot];
    if (sl.epoch == 0) return fail(NGRAM_EINVAL, "slot %u holds no prefetched batch", slot);
    const uint64_t N = static_cast<uint64_t>(sl.n_seq) * sl.T;
    if (N == 0) return NGRAM_OK;
    if (residual == nullptr || gate == nullptr || out == nullptr)
        return fail(NGRAM_EINVAL, "residual, gate and out must be non-NULL");
    if (!aligned16(residual) || !aligned16(gate) || !aligned16(out))
        return fail(NGRAM_EINVAL, "residual, gate and out must be 16-byte aligned");
    if (out != residual) {
        const uint64_t bytes = N * c->d * 2ull;
        const uintptr_t a = reinterpret_cast<uintptr_t>(out), b = reinterpret_cast<uintptr_t>(residual);
        if (a < b + bytes && b < a + bytes)
            return fail(NGRAM_EINVAL, "out overlaps residual without being equal to it");
    }
    GatherArgs g = gather_args(c, nullptr, nullptr, sl.T, static_cast<uint32_t>(N), residual, gate, out);
    g.table = sl.stage;
    g.row_scale = staged_scale(c, sl.stage_scale);
    g.row_ids = sl.inv;
    return launch_gather(c, g, reinterpret_cast<cudaStream_t>(stream), full_grid(c));
}

ngram_status ngram_auto_choice(const ngram_ctx *c, uint32_t n_tokens, int *where_out) {
    if (c == nullptr || where_out == nullptr) return fail(NGRAM_EINVAL, "ctx / where_out is NULL");
    if (n_tokens == 0) return fail(NGRAM_EINVAL, "n_tokens must be > 0");
    const int ch = c->auto_choice[ceil_log2(n_tokens)];
    *where_out = ch ? ch : -1;
    return NGRAM_OK;
}

ngram_status ngram_hash_indices(ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                                uint32_t n_seq, uint32_t T, uint32_t *idx_out,
                                ngram_stream_t stream) {
    uint64_t N = 0;
    NG_CHECK(check_batch(c, tokens, n_seq, T, &N));
    if (N == 0) return NGRAM_OK;
    if (idx_out == nullptr) return fail(NGRAM_EINVAL, "idx_out is NULL");
    return launch_hash(c, tokens, history, T, static_cast<uint32_t>(N), idx_out,
                       reinterpret_cast<cudaStream_t>(stream));
}

ngram_status ngram_dedup_rows(ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                              uint32_t n_seq, uint32_t T, uint32_t *uniq_out, uint32_t *inv_out,
                              uint32_t *count_out, ngram_stream_t stream) {
    uint64_t N = 0;
    NG_CHECK(check_batch(c, tokens, n_seq, T, &N));
    if (count_out == nullptr) return fail(NGRAM_EINVAL, "count_out is NULL");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {                               // empty batch: U = 0, nothing else written
        NG_CUDA(cudaMemsetAsync(count_out, 0, 4, s), "cudaMemsetAsync");
        return NGRAM_OK;
    }
    if (uniq_out == nullptr || inv_out == nullptr)
        return fail(NGRAM_EINVAL, "uniq_out and inv_out must be non-NULL");
    NG_CHECK(ensure_dedup_scratch(c));
    return launch_hash_dedup(c, tokens, history, T, static_cast<uint32_t>(N), uniq_out, inv_out, count_out, s);
}

ngram_status ngram_fill_synthetic(void *table, float *row_scale, uint64_t R, uint32_t d,
                                  ngram_dtype dtype, uint64_t seed, ngram_stream_t stream) {
    return ngram_fill_synthetic_cols(table, row_scale, R, d, 0, dtype, seed, stream);
}

ngram_status ngram_fill_synthetic_cols(void *table, float *row_scale, uint64_t R, uint32_t d,
                                       uint32_t col0, ngram_dtype dtype, uint64_t seed,
                                       ngram_stream_t stream) {
    if (table == nullptr) return fail(NGRAM_EINVAL, "table is NULL");
    if (!aligned16(table)) return fail(NGRAM_EINVAL, "table must be 16-byte aligned");
    if (R == 0 || R > 0xFFFFFFFFull) return fail(NGRAM_EINVAL, "R must be in [1, 2^32 - 1]");
    NG_CHECK(check_format(dtype, d, row_scale));
    NG_CHECK(check_format(dtype, col0 + d, row_scale));     // col0: a multiple of the d rule
    int dev = 0, sms = 0;
    NG_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    NG_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "cudaDeviceGetAttribute");
    // a pinned, mapped host table is written through its device alias
    void *dst = table;
    float *dst_scale = row_scale;
    cudaPointerAttributes attr;
    NG_CUDA(cudaPointerGetAttributes(&attr, table), "cudaPointerGetAttributes(table)");
    if (attr.type == cudaMemoryTypeHost) {
        if (attr.devicePointer == nullptr) return fail(NGRAM_EINVAL, "host table is not mapped");
        dst = attr.devicePointer;
        if (row_scale != nullptr) {
            NG_CUDA(cudaPointerGetAttributes(&attr, row_scale), "cudaPointerGetAttributes(row_scale)");
            if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr)
                return fail(NGRAM_EINVAL, "host table needs a mapped host row_scale");
            dst_scale = static_cast<float *>(attr.devicePointer);
        }
    } else if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) {
        return fail(NGRAM_EINVAL, "table must be device memory or pinned, mapped host memory");
    }
    uint64_t blocks = static_cast<uint64_t>(sms) * 8;
    if (blocks > R) blocks = R;
    const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const unsigned nb = static_cast<unsigned>(blocks);
    switch (dtype) {
        case NGRAM_BF16: k_fill_bf16<<<nb, 256, 0, s>>>(static_cast<uint16_t *>(dst), R, d, col0, k0, k1); break;
        case NGRAM_INT8_ROWSCALE: k_fill_int8<<<nb, 256, 0, s>>>(static_cast<int8_t *>(dst), dst_scale, R, d, col0, k0, k1); break;
        case NGRAM_FP8_E4M3_ROWSCALE: k_fill_fp8<<<nb, 256, 0, s>>>(static_cast<uint8_t *>(dst), dst_scale, R, d, col0, k0, k1); break;
        case NGRAM_NVFP4: k_fill_fp4<<<nb, 256, 0, s>>>(static_cast<uint8_t *>(dst), dst_scale, R, d, col0, k0, k1); break;
    }
    NG_CUDA(cudaGetLastError(), "k_fill launch");
    return NGRAM_OK;
}

// ---------------------------------------------------------------- column-sharded table
ngram_status ngram_forward_shard(ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                                 uint32_t n_seq, uint32_t T, uint32_t d_full, uint32_t col0,
                                 const uint16_t *residual, const void *gate, uint16_t *const *outs,
                                 uint32_t n_outs, ngram_stream_t stream) {
    uint64_t N = 0;
    NG_CHECK(check_batch(c, tokens, n_seq, T, &N));
    if (c->where != NGRAM_RES_HBM)
        return fail(NGRAM_EUNSUPPORTED, "ngram_forward_shard: HBM residency only");
    if (c->hp.flags & (NGRAM_FLAG_DEDUP | NGRAM_FLAG_TMA_STAGING))
        return fail(NGRAM_EUNSUPPORTED, "ngram_forward_shard: no DEDUP or TMA_STAGING");
    if (static_cast<uint64_t>(col0) + c->d > d_full)
        return fail(NGRAM_EINVAL, "shard columns [%u, %u) exceed d_full %u", col0, col0 + c->d, d_full);
    if (col0 % 8 != 0 || d_full % 8 != 0)
        return fail(NGRAM_EINVAL, "col0 and d_full must be multiples of 8");
    if (n_outs == 0 || n_outs > 8 || outs == nullptr)
        return fail(NGRAM_EINVAL, "n_outs must be in [1, 8] with outs non-NULL");
    if (N == 0) return NGRAM_OK;
    if (residual == nullptr || gate == nullptr) return fail(NGRAM_EINVAL, "residual and gate must be non-NULL");
    if (!aligned16(residual) || !aligned16(gate)) return fail(NGRAM_EINVAL, "residual and gate must be 16-byte aligned");
    for (uint32_t p = 0; p < n_outs; ++p)
        if (outs[p] == nullptr || !aligned16(outs[p])) return fail(NGRAM_EINVAL, "outs[%u] NULL or misaligned", p);
    const bool tok_gate = (c->hp.flags & NGRAM_FLAG_TOKEN_GATE) != 0;
    const Call k{tokens, history, T, static_cast<uint32_t>(N), residual, gate, nullptr,
                 reinterpret_cast<cudaStream_t>(stream)};
    GatherArgs g = gather_args(c, k.tokens, k.history, k.T, k.N, residual + col0,
                               tok_gate ? static_cast<const void *>(static_cast<const uint16_t *>(gate) + col0)
                                        : static_cast<const void *>(static_cast<const float *>(gate) + col0),
                               nullptr);
    // 8 columns per lane for every format
    g.n_strips = (c->d / 8 + 31) / 32;
    g.strips_per_item = 1;
    g.groups_per_token = g.n_strips;
    g.ld = d_full;
    g.n_outs = n_outs;
    for (uint32_t p = 0; p < n_outs; ++p) g.outs[p] = outs[p] + col0;
    if (grouped_order(c, k.N)) {
        NG_CHECK(order_tokens(c, k));
        g.perm = c->so_perm;
    }
    const uint64_t items = static_cast<uint64_t>(g.N) * g.groups_per_token;
    uint64_t blocks = (items + 7) / 8;
    const uint64_t cap = static_cast<uint64_t>(c->num_sms) * NGRAM_C8_MIN_BLOCKS;
    if (blocks > cap) blocks = cap;
    const unsigned nb = static_cast<unsigned>(blocks);
    if (tok_gate) launch_shard<true>(c->dtype, g, nb, k.s, c->row_bytes);
    else launch_shard<false>(c->dtype, g, nb, k.s, c->row_bytes);
    NG_CUDA(cudaGetLastError(), "k_gather_c8 (shard) launch");
    return NGRAM_OK;
}

ngram_status ngram_device_alloc(void **out, uint64_t bytes) {
    if (out == nullptr) return fail(NGRAM_EINVAL, "out is NULL");
    *out = nullptr;
    if (bytes == 0) return fail(NGRAM_EINVAL, "bytes must be > 0");
    const cudaError_t e = cudaMalloc(out, bytes);
    if (e != cudaSuccess) {
        *out = nullptr;
        return cuda_fail(e, "cudaMalloc");
    }
    return NGRAM_OK;
}

ngram_status ngram_device_free(void *p) {
    if (p == nullptr) return NGRAM_OK;
    NG_CUDA(cudaFree(p), "cudaFree");
    return NGRAM_OK;
}

ngram_status ngram_ipc_get_handle(const void *dev_ptr, uint8_t handle[64]) {
    if (dev_ptr == nullptr || handle == nullptr) return fail(NGRAM_EINVAL, "dev_ptr and handle must be non-NULL");
    cudaIpcMemHandle_t h;
    NG_CUDA(cudaIpcGetMemHandle(&h, const_cast<void *>(dev_ptr)), "cudaIpcGetMemHandle");
    static_assert(sizeof(h) == 64, "cudaIpcMemHandle_t is 64 bytes");
    memcpy(handle, &h, 64);
    return NGRAM_OK;
}

ngram_status ngram_ipc_open(const uint8_t handle[64], void **dev_ptr) {
    if (dev_ptr == nullptr || handle == nullptr) return fail(NGRAM_EINVAL, "dev_ptr and handle must be non-NULL");
    *dev_ptr = nullptr;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, 64);
    NG_CUDA(cudaIpcOpenMemHandle(dev_ptr, h, cudaIpcMemLazyEnablePeerAccess), "cudaIpcOpenMemHandle");
    return NGRAM_OK;
}

ngram_status ngram_ipc_close(void *dev_ptr) {
    if (dev_ptr == nullptr) return fail(NGRAM_EINVAL, "dev_ptr is NULL");
    NG_CUDA(cudaIpcCloseMemHandle(dev_ptr), "cudaIpcCloseMemHandle");
    return NGRAM_OK;
}

// ---------------------------------------------------------------- backward
}  // extern "C"

namespace {

ngram_status ensure_backward_sort(ngram_ctx *c) {
    const uint64_t M = c->dd_cap;
    const uint64_t n_tiles = (M + kSortTile - 1) / kSortTile;
    const uint64_t L = kSortRadix * n_tiles;
    const uint64_t nb = (L + kScanChunk - 1) / kScanChunk;
    for (int b = 0; b < 2; ++b) {
        NG_CHECK(dev_alloc(&c->bw_k[b], M * 4, "backward scratch"));
        NG_CHECK(dev_alloc(&c->bw_v[b], M * 4, "backward scratch"));
    }
    NG_CHECK(dev_alloc(&c->bw_hist, L * 4, "backward scratch"));
    NG_CHECK(dev_alloc(&c->bw_tot, nb * 4, "backward scratch"));
    NG_CHECK(dev_alloc(&c->bw_seg, (M + 1) * 4, "backward scratch"));
    NG_CHECK(dev_alloc(&c->bw_word, 8, "backward scratch"));     // scan total, item counter
    // queried once, not per call, so that a call may be captured in a CUDA graph
    if (c->bw_rows_per_sm[0] == 0) {
        constexpr int kS = NGRAM_ROWS_GRAD_STRIPS;
        NG_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c->bw_rows_per_sm[1], k_rows_grad<true, kS>, 256, 0),
                "occupancy");
        NG_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c->bw_rows_per_sm[0], k_rows_grad<false, kS>, 256, 0),
                "occupancy");
    }
    return NGRAM_OK;
}

// Exclusive scan of a[0..n) in place.
ngram_status scan_exclusive(ngram_ctx *c, uint32_t *a, uint32_t n, cudaStream_t s) {
    const uint32_t nb = (n + kScanChunk - 1) / kScanChunk;
    NG_CUDA(launch_dependent(k_scan_local, nb, 256, s, a, n, a, c->bw_tot), "scan launch");
    NG_CUDA(launch_dependent(k_dedup_scan_blocks, 1, 1024, s, c->bw_tot, nb, c->bw_word), "scan launch");
    NG_CUDA(launch_dependent(k_scan_add, (n + 255) / 256, 256, s, a, n, c->bw_tot), "scan launch");
    return NGRAM_OK;
}

// Stable sort of the M occurrences by key (their row's position u < M); the values are
// the occurrences' tokens (p / H).  Returns the sorted keys and values.
ngram_status sort_occurrences(ngram_ctx *c, const uint32_t *keys, uint32_t M, cudaStream_t s,
                              const uint32_t **skeys, const uint32_t **svals) {
    const uint32_t bits = std::max<uint32_t>(1u, ceil_log2(M));
    const uint32_t passes = (bits + 7) / 8;
    const uint32_t n_tiles = (M + kSortTile - 1) / kSortTile;
    const unsigned grid = static_cast<unsigned>(std::min<uint64_t>(n_tiles, static_cast<uint64_t>(c->num_sms) * 8));
    const uint32_t *kin = keys, *vin = nullptr;
    for (uint32_t pass = 0; pass < passes; ++pass) {
        const uint32_t shift = 8 * pass;
        NG_CUDA(launch_dependent(k_radix_hist, grid, 256, s, kin, M, shift, n_tiles, c->bw_hist),
                "radix sort launch");
        NG_CHECK(scan_exclusive(c, c->bw_hist, kSortRadix * n_tiles, s));
        const int o = static_cast<int>(pass & 1u);
        NG_CUDA(launch_dependent(k_radix_scatter, grid, 256, s, kin, vin, c->H, M, shift, n_tiles, c->bw_hist,
                                 c->bw_k[o], c->bw_v[o]),
                "radix sort launch");
        kin = c->bw_k[o];
        vin = c->bw_v[o];
    }
    *skeys = kin;
    *svals = vin;
    return NGRAM_OK;
}

template <class Rows, bool kTok>
cudaError_t launch_gate_grad_fmt(const GatherArgs &g, unsigned grid, cudaStream_t s, const uint16_t *dy,
                                 float *dg, double *part, uint32_t rb) {
    if (g.h.n_heads == 16) return launch_dependent(k_gate_grad<16, Rows, kTok>, grid, 256, s, g, dy, dg, part, rb);
    return launch_dependent(k_gate_grad<0, Rows, kTok>, grid, 256, s, g, dy, dg, part, rb);
}

template <bool kTok>
cudaError_t launch_gate_grad(ngram_dtype t, const GatherArgs &g, unsigned grid, cudaStream_t s,
                             const uint16_t *dy, float *dg, double *part, uint32_t rb) {
    switch (t) {
        case NGRAM_BF16: return launch_gate_grad_fmt<RowsBf16, kTok>(g, grid, s, dy, dg, part, rb);
        case NGRAM_INT8_ROWSCALE: return launch_gate_grad_fmt<Rows8bit<Int8Codes>, kTok>(g, grid, s, dy, dg, part, rb);
        case NGRAM_FP8_E4M3_ROWSCALE: return launch_gate_grad_fmt<Rows8bit<E4m3Codes>, kTok>(g, grid, s, dy, dg, part, rb);
        case NGRAM_NVFP4: return launch_gate_grad_fmt<RowsNvfp4, kTok>(g, grid, s, dy, dg, part, rb);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

extern "C" {

ngram_status ngram_backward_rows(ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                                 uint32_t n_seq, uint32_t T, const uint16_t *grad_out,
                                 const void *gate, uint32_t *uniq_out, uint32_t *count_out,
                                 float *grad_rows, ngram_stream_t stream) {
    uint64_t N = 0;
    NG_CHECK(check_batch(c, tokens, n_seq, T, &N));
    if (count_out == nullptr) return fail(NGRAM_EINVAL, "count_out is NULL");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        NG_CUDA(cudaMemsetAsync(count_out, 0, 4, s), "cudaMemsetAsync");
        return NGRAM_OK;
    }
    if (grad_out == nullptr || gate == nullptr || uniq_out == nullptr || grad_rows == nullptr)
        return fail(NGRAM_EINVAL, "grad_out, gate, uniq_out and grad_rows must be non-NULL");
    if (!aligned16(grad_out) || !aligned16(gate) || !aligned16(grad_rows))
        return fail(NGRAM_EINVAL, "grad_out, gate and grad_rows must be 16-byte aligned");
    NG_CHECK(ensure_dedup_scratch(c));
    NG_CHECK(ensure_backward_sort(c));
    const uint32_t M = static_cast<uint32_t>(N) * c->H;
    NG_CUDA(cudaMemsetAsync(c->bw_word + 1, 0, 4, s), "cudaMemsetAsync");     // k_rows_grad's item counter
    NG_CHECK(launch_hash_dedup(c, tokens, history, T, static_cast<uint32_t>(N), uniq_out, c->d_inv, count_out, s));
    const uint32_t *skeys = nullptr, *stok = nullptr;
    NG_CHECK(sort_occurrences(c, c->d_inv, M, s, &skeys, &stok));
    NG_CUDA(launch_dependent(k_seg_starts, grid_for(c, M, 256), 256, s, skeys, M, c->bw_seg), "k_seg_starts launch");
    const bool tok_gate = (c->hp.flags & NGRAM_FLAG_TOKEN_GATE) != 0;
    constexpr int kS = NGRAM_ROWS_GRAD_STRIPS;
    const int per_sm = c->bw_rows_per_sm[tok_gate ? 1 : 0];
    const unsigned grid = static_cast<unsigned>(c->num_sms) * static_cast<unsigned>(std::max(1, per_sm));
    if (tok_gate)
        NG_CUDA(launch_dependent(k_rows_grad<true, kS>, grid, 256, s, count_out, c->bw_seg, stok, grad_out,
                                 nullptr, static_cast<const uint16_t *>(gate), c->d, grad_rows, c->bw_word + 1),
                "k_rows_grad launch");
    else
        NG_CUDA(launch_dependent(k_rows_grad<false, kS>, grid, 256, s, count_out, c->bw_seg, stok, grad_out,
                                 static_cast<const float *>(gate), nullptr, c->d, grad_rows, c->bw_word + 1),
                "k_rows_grad launch");
    return NGRAM_OK;
}

ngram_status ngram_backward_gate(ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                                 uint32_t n_seq, uint32_t T, const uint16_t *grad_out,
                                 float *grad_gate, ngram_stream_t stream) {
    uint64_t N = 0;
    NG_CHECK(check_batch(c, tokens, n_seq, T, &N));
    if (grad_gate == nullptr) return fail(NGRAM_EINVAL, "grad_gate is NULL");
    if (!aligned16(grad_gate)) return fail(NGRAM_EINVAL, "grad_gate must be 16-byte aligned");
    if (c->where == NGRAM_RES_HOST_DMA)
        return fail(NGRAM_EUNSUPPORTED, "ngram_backward_gate reads the table from the GPU: HBM, HOST_UVA or HOST_AUTO");
    const bool tok_gate = (c->hp.flags & NGRAM_FLAG_TOKEN_GATE) != 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        if (!tok_gate) NG_CUDA(cudaMemsetAsync(grad_gate, 0, c->d * 4ull, s), "cudaMemsetAsync");
        return NGRAM_OK;
    }
    if (grad_out == nullptr) return fail(NGRAM_EINVAL, "grad_out is NULL");
    if (!aligned16(grad_out)) return fail(NGRAM_EINVAL, "grad_out must be 16-byte aligned");
    const GatherArgs g = gather_args(c, tokens, history, T, static_cast<uint32_t>(N), nullptr, nullptr, nullptr);
    const unsigned grid = static_cast<unsigned>(c->num_sms) * 2u;
    if (tok_gate) {
        NG_CUDA(launch_gate_grad<true>(c->dtype, g, grid, s, grad_out, grad_gate, nullptr, c->row_bytes),
                "k_gate_grad launch");
    } else {
        const uint64_t max_chunks = (c->max_tokens + kGateChunk - 1) / kGateChunk;
        const uint64_t max_groups = (max_chunks + kGateGroup - 1) / kGateGroup;
        // chunk partials, then group partials
        NG_CHECK(dev_alloc(&c->bw_part, (max_chunks + max_groups) * 8ull * c->d, "backward scratch"));
        const uint32_t n_chunks = static_cast<uint32_t>((N + kGateChunk - 1) / kGateChunk);
        const uint32_t n_groups = (n_chunks + kGateGroup - 1) / kGateGroup;
        double *groups = c->bw_part + max_chunks * c->d;
        NG_CUDA(launch_gate_grad<false>(c->dtype, g, grid, s, grad_out, nullptr, c->bw_part, c->row_bytes),
                "k_gate_grad launch");
        NG_CUDA(launch_dependent(k_gate_reduce_groups, dim3((c->d + 255) / 256, n_groups), 256, s,
                                 c->bw_part, n_chunks, c->d, groups),
                "k_gate_reduce launch");
        NG_CUDA(launch_dependent(k_gate_reduce, (c->d + 255) / 256, 256, s, groups, n_groups, c->d, grad_gate),
                "k_gate_reduce launch");
    }
    NG_CUDA(cudaGetLastError(), "k_gate_grad launch");
    return NGRAM_OK;
}

ngram_status ngram_selftest_wait_timeout(ngram_ctx *c, uint32_t limit_ms, ngram_stream_t stream) {
    if (c == nullptr) return fail(NGRAM_EINVAL, "ctx is NULL");
    if (limit_ms == 0 || limit_ms > 2000) return fail(NGRAM_EINVAL, "limit_ms must be in [1, 2000]");
    k_selftest_wait<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(c->d_err, limit_ms * 1000000ull);
    NG_CUDA(cudaGetLastError(), "k_selftest_wait launch");
    return NGRAM_OK;
}

ngram_status ngram_get_device_error(ngram_ctx *c, uint32_t info[4], int clear) {
    if (c == nullptr) return fail(NGRAM_EINVAL, "ctx is NULL");
    uint32_t h[4] = {0, 0, 0, 0};
    NG_CUDA(cudaDeviceSynchronize(), "ngram_get_device_error");
    NG_CUDA(cudaMemcpy(h, c->d_err, sizeof(h), cudaMemcpyDeviceToHost), "ngram_get_device_error");
    if (clear) NG_CUDA(cudaMemset(c->d_err, 0, sizeof(h)), "ngram_get_device_error");
    if (info != nullptr) memcpy(info, h, sizeof(h));
    if (h[0] == 1)
        return fail(NGRAM_EDEVICE, "token id %d out of [0, %u) at %s %u", static_cast<int32_t>(h[2]),
                    c->hp.vocab_size, (h[1] & 0x80000000u) ? "history entry" : "flat position",
                    h[1] & 0x7FFFFFFFu);
    if (h[0] != 0)
        return fail(NGRAM_EDEVICE, "a kernel wait ran past its deadline (code %u)", h[0]);
    return NGRAM_OK;
}

void ngram_destroy(ngram_ctx *c) {
    if (c == nullptr) return;
    free_all(c);
    delete c;
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// Dedup without any device allocation.
//
// Some callers cannot call cudaMalloc: a serving process whose device memory was handed
// in full to another allocator at start-up (a cudaMalloc there fails, or carves memory
// out of a pool that is accounted for elsewhere), or a latency-critical loop that
// cannot afford the implicit device synchronisation an allocation may cause.  They
// cannot create an ngram_ctx either (it owns a device error word), so this entry point
// takes the hash parameters directly and keeps all of its scratch in one file-scope
// device array, sized for at most kNoAllocMaxEntries (token, head) entries.
//
// Layout of the array (32-bit words): idx | slot | pos [E each], keys | first | uid
// [P each], block sums [E / 1024], error word [4].
// ------------------------------------------------------------------------------------
namespace {

constexpr uint32_t kNoAllocMaxEntries = 65536u;                   // 4096 tokens x 16 heads
constexpr uint32_t kNoAllocSlots = 2u * kNoAllocMaxEntries;        // hash-table slots
constexpr uint32_t kNoAllocBlocks = kNoAllocMaxEntries / kScanBlock;
constexpr size_t kNoAllocWords = 3ull * kNoAllocMaxEntries + 3ull * kNoAllocSlots + kNoAllocBlocks + 4;

static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocWords];

// Device address of g_noalloc_scratch per device, looked up once per device and again
// whenever the device's current context is not the one the address was taken in (a
// cudaDeviceReset destroys the primary context; the array of the next one may sit at
// another address).  The context is identified by cuCtxGetId, reached through
// cudaGetDriverEntryPoint (no link against libcuda); where that is unavailable, or no
// context is current yet, the address is looked up again on that call.
typedef CUresult (*PfnCtxGetCurrent)(CUcontext *);
typedef CUresult (*PfnCtxGetId)(CUcontext, unsigned long long *);

struct NoallocAddr {
    uint32_t *ptr = nullptr;
    unsigned long long ctx_id = 0;   // 0: unknown
};

std::mutex g_noalloc_mu;
NoallocAddr g_noalloc_addr[256];
PfnCtxGetCurrent g_ctx_get_current = nullptr;
PfnCtxGetId g_ctx_get_id = nullptr;
bool g_ctx_fns_tried = false;

// Unique id of the calling thread's current context, or 0 when it cannot be had.
unsigned long long current_ctx_id() {
    if (!g_ctx_fns_tried) {
        g_ctx_fns_tried = true;
        void *a = nullptr, *b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess && qb == cudaDriverEntryPointSuccess) {
            g_ctx_get_current = reinterpret_cast<PfnCtxGetCurrent>(a);
            g_ctx_get_id = reinterpret_cast<PfnCtxGetId>(b);
        }
        cudaGetLastError();                  // a failed query leaves no sticky error
    }
    if (g_ctx_get_current == nullptr) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

ngram_status noalloc_scratch(uint32_t **out) {
    int dev = -1;
    NG_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 0 || dev >= 256) return fail(NGRAM_EUNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocAddr &a = g_noalloc_addr[dev];
    const unsigned long long id = current_ctx_id();
    if (a.ptr == nullptr || id == 0 || id != a.ctx_id) {
        a = NoallocAddr();
        void *p = nullptr;
        NG_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(noalloc scratch)");
        a.ptr = static_cast<uint32_t *>(p);
        a.ctx_id = current_ctx_id();         // the lookup above made the primary context current
    }
    *out = a.ptr;
    return NGRAM_OK;
}

}  // namespace

extern "C" ngram_status ngram_dedup_rows_noalloc(const ngram_hash_params *hp, uint64_t R,
                                                  const int32_t *tokens, const int32_t *history,
                                                  uint32_t n_seq, uint32_t T, uint32_t *uniq_out,
                                                  uint32_t *inv_out, uint32_t *count_out,
                                                  ngram_stream_t stream) {
    if (R == 0 || R > 0xFFFFFFFFull) return fail(NGRAM_EINVAL, "R must be in [1, 2^32 - 1]");
    ngram_hash_params p;
    if (hp != nullptr) p = *hp; else ngram_default_hash_params(&p);
    NG_CHECK(check_hash_params(p));
    if (count_out == nullptr) return fail(NGRAM_EINVAL, "count_out is NULL");
    const uint32_t H = p.n_bigram_heads + p.n_trigram_heads;
    const uint64_t N = static_cast<uint64_t>(n_seq) * T;
    if (H == 0 || N > kNoAllocMaxEntries / H)          // N * H could wrap: compare by division
        return fail(NGRAM_EINVAL,
                    "ngram_dedup_rows_noalloc: %llu tokens x %u heads exceed its fixed scratch of %u "
                    "entries; use ngram_dedup_rows", static_cast<unsigned long long>(N), H,
                    kNoAllocMaxEntries);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        NG_CUDA(cudaMemsetAsync(count_out, 0, 4, s), "cudaMemsetAsync");
        return NGRAM_OK;
    }
    if (tokens == nullptr || uniq_out == nullptr || inv_out == nullptr)
        return fail(NGRAM_EINVAL, "tokens, uniq_out and inv_out must be non-NULL");
    uint32_t *base = nullptr;
    NG_CHECK(noalloc_scratch(&base));
    const uint32_t E = kNoAllocMaxEntries, P = kNoAllocSlots;
    uint32_t *idx = base, *slot = base + E, *pos = base + 2 * E;
    uint32_t *keys = base + 3 * E, *first = keys + P, *uid = first + P;
    uint32_t *bsum = uid + P, *err = bsum + kNoAllocBlocks;

    const uint32_t M = static_cast<uint32_t>(N) * H;
    const uint32_t log2p = std::max<uint32_t>(10u, ceil_log2(2ull * M));   // <= log2(P)
    const uint32_t NB = (M + kScanBlock - 1) / kScanBlock;
    int dev = 0, sms = 0;
    NG_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    NG_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "cudaDeviceGetAttribute");
    uint64_t gm = (M + 255) / 256;
    if (gm > static_cast<uint64_t>(sms) * 8) gm = static_cast<uint64_t>(sms) * 8;

    HashArgs a;
    a.base_seed = p.base_seed;
    a.R = R;
    a.barrett_m = (R == 1) ? 0ull : static_cast<uint64_t>((static_cast<unsigned __int128>(1) << 64) / R);
    a.n_bigram = p.n_bigram_heads;
    a.n_heads = H;
    a.pad_id = p.pad_id;
    a.vocab = p.vocab_size;
    // the array keeps the previous call's contents: reset what must start cleared
    NG_CUDA(cudaMemsetAsync(err, 0, 16, s), "noalloc clear");
    NG_CUDA(cudaMemsetAsync(keys, 0xFF, (1ull << log2p) * 4, s), "noalloc clear");
    NG_CUDA(cudaMemsetAsync(first, 0xFF, (1ull << log2p) * 4, s), "noalloc clear");
    k_hash_indices<<<static_cast<unsigned>(gm), 256, 0, s>>>(a, tokens, history, T,
                                                              static_cast<uint32_t>(N), err, idx);
    k_dedup_insert<<<static_cast<unsigned>(gm), 256, 0, s>>>(idx, M, keys, first, slot, log2p);
    k_dedup_scan_local<<<NB, 256, 0, s>>>(slot, first, M, pos, bsum);
    k_dedup_scan_blocks<<<1, 1024, 0, s>>>(bsum, NB, count_out);
    k_dedup_emit<<<static_cast<unsigned>(gm), 256, 0, s>>>(idx, slot, first, pos, bsum, M, uniq_out, uid);
    k_dedup_inverse<<<static_cast<unsigned>(gm), 256, 0, s>>>(slot, uid, M, inv_out);
    NG_CUDA(cudaGetLastError(), "ngram_dedup_rows_noalloc launch");
    return NGRAM_OK;
}
