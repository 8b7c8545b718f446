/*
 * ngram.h -- C ABI of libngram.so, the B200 (sm_100a) hashed n-gram embedding lookup.
 *
 * The operation ("Qwen Brought Back N-Grams. All 51 Billion Parameters of Them.",
 * section "N-grams, of all things", and its "Key Takeaways"): for every token, hash
 * the local bigram and trigram context into one table of R rows of width d
 * (20,000,000 x 2560 in the full model), gather 16 rows, sum them, and add the sum to
 * the residual stream.  The sum enters through an elementwise gate, as in the
 * equation of Key point 1 of "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with
 * Heterogeneous Memory Prefetch":  out = residual + g (elementwise) sum_h E[idx_h].
 *
 * Definitions this library fixes where the pages are silent:
 *   - Context of token t in sequence s (t counted from 0 inside the sequence):
 *       w0 = w_t,  w1 = w_{t-1},  w2 = w_{t-2}.  Positions before 0 come from
 *       history[s] = {w_-2, w_-1} (oldest first) when history is non-NULL, else they
 *       are pad_id.  Contexts never cross from one sequence row into another.
 *       A token id outside [0, vocab_size) is read as pad_id and flags the device
 *       error word (see ngram_get_device_error).
 *   - Keys: bigram k2 = (w1 << 21) | w0, trigram k3 = (w2 << 42) | (w1 << 21) | w0.
 *   - Heads: h = 0 .. n_bigram_heads-1 hash k2, the next n_trigram_heads hash k3
 *       (defaults 8 + 8 = the 16 rows per token the pages give).
 *   - Hash: mix(z) = the splitmix64 output function applied to state z + 0x9E3779B97F4A7C15;
 *       seed_h = (h+1)-th splitmix64 output from base_seed;
 *       idx_h  = mix(key ^ seed_h) mod R   (exact 64-bit remainder).
 *   - Sum: fp32, in head order 0..H-1; colliding heads each contribute their row.
 *   - Output: y = fp32(residual) + g * sum (separately rounded multiply and add),
 *       stored as bf16 rounded to nearest even.
 *
 * Memory: every pointer argument of the compute calls is a device pointer (or, for
 * the table in the host-resident modes, a pinned host pointer).  The caller owns
 * every buffer it passes.  bf16 arrays are passed as uint16_t bit patterns.
 * Streams: all compute calls are asynchronous on the stream given (NULL = legacy
 * default stream).  The only other streams are ngram_forward_host's internal copy
 * streams, which start after the given stream and which the given stream waits for;
 * no call makes the given stream wait on anything else.
 * Errors: every call returns an ngram_status; invalid arguments are reported before
 * any CUDA work is issued, and nothing aborts the process.  ngram_last_error() gives
 * the text of the last failure on the calling thread.
 */
#ifndef NGRAM_H_
#define NGRAM_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols; everything else in the library is hidden. */
#if defined(__GNUC__)
#define NGRAM_API __attribute__((visibility("default")))
#else
#define NGRAM_API
#endif

/* Same underlying type as cudaStream_t / CUstream. */
typedef struct CUstream_st *ngram_stream_t;

typedef enum {
    NGRAM_OK = 0,
    NGRAM_EINVAL = 1,          /* bad argument; nothing was launched */
    NGRAM_ENOMEM = 2,          /* a device or pinned allocation failed */
    NGRAM_ECUDA = 3,           /* a CUDA runtime call failed (text in ngram_last_error) */
    NGRAM_EUNSUPPORTED = 4,    /* valid request this build does not implement */
    NGRAM_ETIMEOUT = 5,        /* a bounded host-side wait ran out */
    NGRAM_EDEVICE = 6          /* a kernel flagged bad input (device error word set) */
} ngram_status;

/* Row formats.  bf16 is the table as the pages size it (20M x 2560, ~95 GiB); the
 * 8-bit and 4-bit formats are the smaller tables the pages weigh ("Qwen3.8-Flash-Next:
 * A 51B N-gram Embedding Table with Heterogeneous Memory Prefetch": ~51 GB INT8 in Key
 * point 3, ~25.5 GB at FP4 in its architecture figure; "Qwen3.8-Flash-Next: A 125B MoE
 * for the Local Stack?", section "Hardware math for self-hosting": FP8 and 4-bit).  In
 * every scaled format the value of a code is q * s with q exact in fp32, and the sum over
 * heads is acc = fma(q, s, acc) in fp32, head order, one rounding per head. */
typedef enum {
    NGRAM_BF16 = 0,            /* table [R][d] bf16; d % 8 == 0 */
    NGRAM_INT8_ROWSCALE = 1,   /* table [R][d] int8 + row_scale [R] fp32; value = q * scale;
                                  d % 16 == 0 */
    NGRAM_FP8_E4M3_ROWSCALE = 2, /* table [R][d] FP8 E4M3 codes (OCP: bias 7, S.1111.111 NaN,
                                  no infinities) + row_scale [R] fp32; value = e4m3(q) * scale;
                                  d % 16 == 0 */
    NGRAM_NVFP4 = 3            /* table [R][rb] bytes, rb = d/2 + ceil16(d/16): d/2 bytes of
                                  FP4 E2M1 codes (OCP MX: bias 1, magnitudes 0, 0.5, 1, 1.5,
                                  2, 3, 4, 6; column 2j in the low nibble of byte j), then one
                                  E4M3 scale byte per 16 columns, then zero padding to rb.
                                  row_scale points at ONE fp32 global scale gs.  value =
                                  e2m1(q) * e4m3(block scale) * gs.  In the sum, each head
                                  adds e2m1(q) * e4m3(bs) (exact) to an fp32 accumulator with
                                  one rounding, and gs multiplies the 16-head sum once, in
                                  fp32; d % 32 == 0 */
} ngram_dtype;

typedef enum {
    NGRAM_RES_HBM = 0,         /* table in this GPU's memory */
    NGRAM_RES_HOST_UVA = 1,    /* table in pinned host memory, read by the kernel over PCIe */
    NGRAM_RES_HOST_DMA = 2,    /* table in pinned host memory, rows staged by copy engine */
    NGRAM_RES_HOST_AUTO = 3    /* host-resident; the fastest of UVA / UVA with dedup / DMA,
                                  chosen by timing */
} ngram_residency;

/* ngram_auto_choice's value for HOST_UVA with NGRAM_FLAG_DEDUP (not a residency). */
#define NGRAM_AUTO_UVA_DEDUP 4

/* HBM or HOST_UVA residency: dedup the batch's rows first (ngram_dedup_rows), copy each
 * distinct row once into an HBM staging buffer, and gather from staging through the
 * inverse map.  Same results bit for bit.  With HOST_UVA the copy kernel reads each
 * distinct row once over PCIe (a few CTAs), where the plain UVA gather reads every
 * occurrence.  Staging (max_tokens * H rows in HBM) and the dedup scratch are allocated by
 * the first call that needs them. */
#define NGRAM_FLAG_DEDUP 0x1u
/* Stage the rows through shared memory with TMA bulk copies (cp.async.bulk into an
 * mbarrier ring) instead of register loads: bf16 rows in column chunks, the 8- and 4-bit
 * formats as whole rows (a producer warp copies, consumer warps decode; HBM residency).
 * Same results bit for bit; measured slower on B200 (bf16 522-895 us vs 455 us on the
 * full-size gather; NVFP4 52-76 M vs 121 M tokens/s for the register gather of that time,
 * 138 M now), kept for comparison.  Every wait is
 * bounded (1 s; then device error code 2).  Not with NGRAM_FLAG_TOKEN_GATE. */
#define NGRAM_FLAG_TMA_STAGING 0x2u
/* Grouped order: before the gather, group the batch's tokens by bigram context
 * (counting sort on a 13-bit hash of (w_{t-1}, w_t): 3 small kernels and a memset, ~11 us)
 * and gather in that order, so tokens that read the same rows run back to back and L2
 * serves the repeats.  Same results bit for bit.  Scratch (8 bytes per max_tokens + 32 KB)
 * is allocated by the first call that groups.
 *   HBM residency groups by default when N >= NGRAM_SORT_MIN_TOKENS (measured on B200
 *   with Zipf tokens: break-even near 12,288 tokens, 3-6% faster from 16,384 up).
 *   NGRAM_FLAG_SORT groups every batch (HBM or HOST_UVA); NGRAM_FLAG_BATCH_ORDER never
 *   groups. */
#define NGRAM_FLAG_SORT 0x4u
#define NGRAM_FLAG_BATCH_ORDER 0x8u
#define NGRAM_SORT_MIN_TOKENS 16384u
/* A gate per token: the `gate` argument of ngram_forward, ngram_forward_staged and the
 * backward calls is bf16 [N][d] (16-byte aligned, token-major like residual) instead of
 * fp32 [d] -- the output of a gating network computed from the hidden state
 * ("Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with Heterogeneous Memory
 * Prefetch", Summary).  y = fp32(residual) + fp32(gate[t][c]) * sum, rounded as with the
 * shared gate.  Not with TMA_STAGING (EINVAL) nor ngram_forward_host (EUNSUPPORTED). */
#define NGRAM_FLAG_TOKEN_GATE 0x10u
#define NGRAM_FLAGS_KNOWN (NGRAM_FLAG_DEDUP | NGRAM_FLAG_TMA_STAGING | NGRAM_FLAG_SORT | \
                           NGRAM_FLAG_BATCH_ORDER | NGRAM_FLAG_TOKEN_GATE)

#define NGRAM_MAX_HEADS 16u
#define NGRAM_TOKEN_BITS 21u
#define NGRAM_DEFAULT_BASE_SEED 0x6E6772616D5F7631ull   /* ASCII "ngram_v1" */
#define NGRAM_DEFAULT_PAD_ID 0x1FFFFFu                   /* 2^21 - 1 */

typedef struct {
    uint64_t base_seed;        /* head seeds are the splitmix64 outputs from this state */
    uint32_t n_bigram_heads;   /* default 8 */
    uint32_t n_trigram_heads;  /* default 8; n_bigram + n_trigram in [1, 16] */
    uint32_t pad_id;           /* default 2^21 - 1; must be < 2^21 */
    uint32_t vocab_size;       /* token ids must lie in [0, vocab_size); <= 2^21 - 1 */
    uint32_t flags;            /* NGRAM_FLAG_* bits, default 0 */
    uint32_t reserved;         /* must be 0 */
} ngram_hash_params;

typedef struct ngram_ctx ngram_ctx;

/* Fill hp with the defaults: base_seed "ngram_v1", 8 + 8 heads, pad 2^21-1, and
 * vocab_size 2^21-1.  Returns NGRAM_EINVAL if hp is NULL. */
NGRAM_API ngram_status ngram_default_hash_params(ngram_hash_params *hp);

/* Pinned host memory the GPU can read directly (cudaHostAlloc, mapped + portable), for a
 * host-resident table ("Which is why the offload matters more than the parameter
 * count" on the aibacon page: rows parked in pinned host memory, gathered over unified
 * addressing).  ngram_fill_synthetic can fill it.  Free with ngram_host_free. */
NGRAM_API ngram_status ngram_host_alloc(void **out, uint64_t bytes);
NGRAM_API ngram_status ngram_host_free(void *p);

/* Bytes of one table row in the dtype's layout (2d bf16; d int8 and fp8;
 * d/2 + ceil16(d/16) nvfp4), after the same d checks as ngram_init.  Host only, no CUDA
 * call.  EINVAL for an unknown dtype, a d the dtype does not allow, or out == NULL. */
NGRAM_API ngram_status ngram_row_bytes(ngram_dtype dtype, uint32_t d, uint32_t *out);

/* Create a lookup context on the current CUDA device.
 *   table      the R rows in the dtype's layout (ngram_dtype), 16-byte aligned; not owned, must
 *              outlive the context.  Device memory for NGRAM_RES_HBM; pinned, mapped
 *              host memory (ngram_host_alloc) for HOST_UVA and HOST_AUTO; any host
 *              memory for HOST_DMA (host threads read it).
 *   row_scale  int8 / fp8: [R] fp32 in the same kind of memory as the table; not owned.
 *              nvfp4: ONE fp32 (host or device memory), copied by this call.  bf16: NULL.
 *   R          rows, 1 <= R < 2^32.   d: row width (columns), a multiple of 8 (bf16),
 *              16 (int8, fp8) or 32 (nvfp4).
 *   where      residency of the table:
 *              HBM       one fused kernel per call;
 *              HOST_UVA  the same kernel reads the rows from host memory over PCIe;
 *              HOST_DMA  rows are deduplicated on the GPU, the distinct rows are copied
 *                        by host threads (OpenMP: OMP_NUM_THREADS / OMP_WAIT_POLICY
 *                        apply) into pinned staging and moved to HBM by the copy engine
 *                        in 8 MB chunks (copy and host gather overlap), then gathered
 *                        from HBM; the call blocks the host until the rows are staged
 *                        (bounded wait, see ngram_set_wait_timeout);
 *              HOST_AUTO the first call of each batch-size bucket (ceil(log2 N)) runs
 *                        UVA, UVA with dedup (NGRAM_FLAG_DEDUP) and DMA, each once
 *                        untimed and then three times timed in interleaved rounds
 *                        (synchronously); later calls use the mode with the lowest
 *                        median time
 *                        (ngram_auto_choice reports it).
 *   hp         hash parameters (NULL = defaults).
 *   max_tokens largest n_seq * T a later call may pass (>= 1).
 * The context owns a 16-byte device error word; dedup scratch and staging buffers are
 * allocated by the first call that needs them (a call that returns NGRAM_ENOMEM keeps what
 * it allocated and launches nothing that needs the rest; a later call allocates the rest).  EINVAL on bad arguments (checked
 * before any CUDA call, except the memory-kind checks of host residency),
 * ECUDA/ENOMEM on CUDA failures.  On failure *out is set to NULL. */
NGRAM_API ngram_status ngram_init(ngram_ctx **out, const void *table, const float *row_scale,
                        uint64_t R, uint32_t d, ngram_dtype dtype, ngram_residency where,
                        const ngram_hash_params *hp, uint32_t max_tokens);

/* The fused lookup: for all N = n_seq * T tokens,
 *   out[t][c] = bf16( residual[t][c] + gate[c] * sum_h table[idx_h(t)][c] ).
 *   tokens    device int32 [n_seq][T] (row-major).
 *   history   device int32 [n_seq][2] = {w_-2, w_-1} per sequence, or NULL (PAD).
 *   residual  device bf16 [N][d], 16-byte aligned.
 *   gate      device fp32 [d], 16-byte aligned (the static gate W_g); with
 *             NGRAM_FLAG_TOKEN_GATE device bf16 [N][d] (one gate per token).
 *   out       device bf16 [N][d], 16-byte aligned; may equal residual (in place),
 *             must not otherwise overlap it.
 * Launches on stream: the fused gather kernel.  A grouped batch (HBM: NGRAM_FLAG_SORT, or by
 * default from NGRAM_SORT_MIN_TOKENS tokens) is preceded by the grouped-order step (a memset
 * and 3 small kernels); for bf16 and NVFP4 tables from 4,096 tokens its first kernel also
 * hashes every token once (64 B of row ids per token), so that the gather's work items read
 * row ids instead of hashing per column strip.  N == 0
 * launches nothing.  The grouping and row-id scratch belong to the context: order the
 * context's ngram_forward calls (one stream, or events); ngram_prefetch uses other scratch
 * and may run beside them.  EINVAL if N > max_tokens, a pointer is NULL or misaligned.  Bad
 * token ids are reported asynchronously through ngram_get_device_error.
 *   Stream order: the gather and the order kernels of an HBM lookup are launched as
 *   programmatic dependents (the launch may overlap the previous kernel of the stream; each
 *   waits for that kernel to complete before touching memory), and they let the next such
 *   kernel be scheduled as soon as they start.  Results are those of plain stream order.
 *   The hash, dedup, radix-sort and backward kernels of the other entry points are
 *   launched the same way.  The host-resident lookups on a bounded grid, and the copy of
 *   host rows into staging, launch plainly. */
NGRAM_API ngram_status ngram_forward(ngram_ctx *ctx, const int32_t *tokens, const int32_t *history,
                           uint32_t n_seq, uint32_t T, const uint16_t *residual,
                           const void *gate, uint16_t *out, ngram_stream_t stream);

/* Prefetch: stage the rows a coming batch will read, ahead of its lookup.  The pages
 * describe prefetching the n-gram vectors of upcoming tokens over PCIe while the GPU
 * computes ("Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with Heterogeneous Memory
 * Prefetch", Key point 3).
 *   ngram_prefetch hashes and dedups the batch on the GPU, then copies each distinct row
 *   once from the table into HBM staging slot `slot` (0 .. NGRAM_STAGE_SLOTS-1); with a
 *   host-resident table (HOST_UVA / HOST_AUTO) the copy kernel reads host memory over PCIe
 *   on 8 CTAs, leaving the other SMs to the work it overlaps.  Asynchronous on `stream`
 *   (typically a side stream).
 *   ngram_forward_staged then computes ngram_forward for that batch from HBM staging
 *   (bit-identical results), on `stream`; the caller orders it after the prefetch
 *   (e.g. cudaStreamWaitEvent).
 * The slots and the dedup scratch belong to the context: prefetches on one context must
 * be ordered with each other, and a slot must not be refilled while a staged forward
 * still reads it.  Each slot holds max_tokens * H rows (allocated by its first
 * prefetch).  A slot that no prefetch has filled, or whose last prefetch failed to
 * allocate or launch its work, holds no batch: ngram_forward_staged on it returns
 * NGRAM_EINVAL (a prefetch refused for its arguments leaves the slot as it was).  HOST_DMA
 * residency:
 * NGRAM_EUNSUPPORTED. */
#define NGRAM_STAGE_SLOTS 2u
NGRAM_API ngram_status ngram_prefetch(ngram_ctx *ctx, uint32_t slot, const int32_t *tokens,
                                      const int32_t *history, uint32_t n_seq, uint32_t T,
                                      ngram_stream_t stream);
NGRAM_API ngram_status ngram_forward_staged(ngram_ctx *ctx, uint32_t slot, const uint16_t *residual,
                                            const void *gate, uint16_t *out, ngram_stream_t stream);

/* Backward of out = residual + gate * sum_h E[idx_h(t)], given grad_out = dL/dout (device
 * bf16 [N][d], 16-byte aligned).  The gradient with respect to residual is grad_out itself.
 *
 * ngram_backward_rows: the gradient with respect to the table, which only the rows the
 * batch read have.  uniq_out (device uint32 [N*H]) receives the distinct rows in order of
 * first occurrence (the list ngram_dedup_rows gives), count_out (device uint32 [1]) their
 * number U, and grad_rows (device fp32 [N*H][d], 16-byte aligned; rows 0..U-1 written)
 * row u's gradient: over the occurrences i = t * H + h of uniq_out[u] in ascending order,
 *   shared gate:    grad = fp32(gate * S),  S = the fp32 sum of grad_out[t] in that order;
 *   per-token gate: grad = the chain acc = fma(gate[t], grad_out[t], acc) in that order.
 * A row read by several heads of one token counts once per head.  The order is fixed by a
 * stable radix sort of the occurrences (no floating-point atomics), so the result is the
 * same bit for bit on every run.  Scratch (about 20 bytes per max_tokens * H entry) is
 * allocated by the first call.  The table itself is not read.
 *
 * ngram_backward_gate: the gradient with respect to the gate (recomputes the head sums
 * e[t] exactly as ngram_forward does; HBM, HOST_UVA or HOST_AUTO residency, else
 * NGRAM_EUNSUPPORTED):
 *   shared gate:    grad_gate device fp32 [d] = fp32 of the sum over every token of
 *                   grad_out[t] * e[t]: each product exact in fp64, summed in fp64 over
 *                   fixed chunks of 16 tokens and then over the chunks in order (same
 *                   result on every run and any GPU size); scratch N/16 * d fp64;
 *   per-token gate: grad_gate device fp32 [N][d] = fp32(grad_out[t] * e[t]).
 * Both are asynchronous on stream; N == 0: count_out set to 0 / grad_gate zeroed
 * (shared) or untouched (per-token).  EINVAL as for ngram_forward. */
NGRAM_API ngram_status ngram_backward_rows(ngram_ctx *ctx, const int32_t *tokens,
                                           const int32_t *history, uint32_t n_seq, uint32_t T,
                                           const uint16_t *grad_out, const void *gate,
                                           uint32_t *uniq_out, uint32_t *count_out,
                                           float *grad_rows, ngram_stream_t stream);
NGRAM_API ngram_status ngram_backward_gate(ngram_ctx *ctx, const int32_t *tokens,
                                           const int32_t *history, uint32_t n_seq, uint32_t T,
                                           const uint16_t *grad_out, float *grad_gate,
                                           ngram_stream_t stream);

/* Bound, in milliseconds, of every host-side wait of the context (default 10,000).  A
 * wait that runs out returns NGRAM_ETIMEOUT; work already enqueued stays enqueued and
 * the context stays usable once the stream drains. */
NGRAM_API ngram_status ngram_set_wait_timeout(ngram_ctx *ctx, uint32_t ms);

/* Residency HOST_AUTO picked for batches of n_tokens (its ceil(log2) bucket):
 * NGRAM_RES_HOST_UVA, NGRAM_AUTO_UVA_DEDUP or NGRAM_RES_HOST_DMA, or -1 while
 * undecided. */
NGRAM_API ngram_status ngram_auto_choice(const ngram_ctx *ctx, uint32_t n_tokens, int *where_out);

/* Per-batch row dedup (the optional dedup step): with idx the [N][H] row indices of
 * the batch (as ngram_hash_indices computes them), writes
 *   uniq_out  device uint32 [N*H]: the distinct rows, in order of first appearance in
 *             idx, in entries [0, U);
 *   inv_out   device uint32 [N*H]: inv[i] = position of idx[i]'s row in uniq, so that
 *             uniq[inv[i]] == idx[i] for every entry (colliding heads keep their own);
 *   count_out device uint32 [1]: U (an empty batch writes 0 and may pass NULL arrays).
 * The result is a pure function of the batch.  Several kernel launches on stream; the
 * context's scratch (allocated on first use, ~24 bytes per entry of max_tokens * H) is
 * reused by every call, so calls on one context must not overlap on the GPU. */
NGRAM_API ngram_status ngram_dedup_rows(ngram_ctx *ctx, const int32_t *tokens,
                                        const int32_t *history, uint32_t n_seq, uint32_t T,
                                        uint32_t *uniq_out, uint32_t *inv_out,
                                        uint32_t *count_out, ngram_stream_t stream);

/* ngram_dedup_rows for callers that cannot allocate device memory.  The pages have no
 * counterpart to this call; it exists for users of this library.  Callers that cannot
 * call cudaMalloc include a serving process whose device memory was handed in full to
 * another allocator at start-up, and a latency-critical loop that cannot accept the
 * device synchronisation an allocation may cause.  They cannot create an ngram_ctx
 * either (the context owns a device error word), so this call takes the hash
 * parameters (NULL = defaults) and the row count R directly.  Its outputs are exactly
 * those of ngram_dedup_rows.
 *   Allocation: none.  All scratch lives in one static device array of 2.25 MiB that
 *     every GPU which loads libngram.so holds until the process exits.
 *   Limit: n_seq * T * heads <= 65,536 entries (4,096 tokens at 16 heads); larger
 *     batches return NGRAM_EINVAL with a message naming the limit.
 *   Set-up: the first call on each device looks the array's device address up (with
 *     that device current); make that first call before any stream capture.  The
 *     address is kept per device together with the id of the context it was taken in;
 *     a call that finds another context current (after cudaDeviceReset) looks it up
 *     again, so make the first call after a reset before any stream capture too.
 *   Sharing: every call on a device uses the same array and leaves its contents
 *     behind; the call clears what must start empty.  Calls that overlap on the GPU
 *     (other streams, other host threads) race on the array: serialise them.
 *   Bad token ids read as PAD, as in ngram_forward, but are not reported (there is no
 *     context to hold the error word). */
NGRAM_API ngram_status ngram_dedup_rows_noalloc(const ngram_hash_params *hp, uint64_t R,
                                                const int32_t *tokens, const int32_t *history,
                                                uint32_t n_seq, uint32_t T, uint32_t *uniq_out,
                                                uint32_t *inv_out, uint32_t *count_out,
                                                ngram_stream_t stream);

/* ngram_forward with the per-token inputs and the output in HOST memory (the weights --
 * table and gate -- stay resident on the device).  The batch is cut into chunks of about
 * 16 MB of residual dealt round-robin to three internal streams; each stream copies its
 * chunk in, gathers it and copies it out, and the streams overlap each other, so PCIe
 * carries input and output at the same time.
 *   tokens_h   host int32 [n_seq][T]; history_h host int32 [n_seq][2] or NULL;
 *   residual_h host bf16 [N][d];  gate: DEVICE fp32 [d];  out_h: host bf16 [N][d], must
 *   not overlap residual_h.  Pinned host memory gives the overlap; pageable memory works
 *   but its copies do not overlap.
 * Ordering: starts after the work already on `stream`; `stream` waits for the last
 * output chunk, so synchronising `stream` means out_h is complete.  Host buffers must
 * stay valid until then.  HBM or HOST_UVA residency without flags (BATCH_ORDER aside),
 * else
 * NGRAM_EUNSUPPORTED.  The device copies of the inputs (max_tokens tokens, two chunks
 * of residual and output) are allocated by the first call. */
NGRAM_API ngram_status ngram_forward_host(ngram_ctx *ctx, const int32_t *tokens_h,
                                          const int32_t *history_h, uint32_t n_seq, uint32_t T,
                                          const uint16_t *residual_h, const float *gate,
                                          uint16_t *out_h, ngram_stream_t stream);

/* The index step alone: idx_out (device uint32 [N][H], H = heads) receives the row
 * index of every (token, head), computed exactly as ngram_forward computes them. */
NGRAM_API ngram_status ngram_hash_indices(ngram_ctx *ctx, const int32_t *tokens, const int32_t *history,
                                uint32_t n_seq, uint32_t T, uint32_t *idx_out,
                                ngram_stream_t stream);

/* Fill a table (device memory, or pinned mapped host memory written through its
 * device alias) with the synthetic values used by the tests and benchmarks
 * (the pages' table is learned; no weights exist here).  Element (row, col) is a
 * pure function of (seed, row, col) through Philox4x32-10 (Salmon et al., SC'11):
 *   bf16: counter (col/2, row, 1, 0), key (seed lo32, seed hi32); words (x0,x1) for
 *         even col, (x2,x3) for odd; S = sum of their four 16-bit halves;
 *         value = bf16_rne(float(2S - 262140) * 0x1.1bc77ap-22)   (std 0.02).
 *   int8: counter (col/4, row, 2, 0), word x[col%4]; q = (sum of its bytes - 510) >> 2;
 *         row_scale[row] = 0x1.1bc5f4p-11 * (0.75 + (x0 >> 8) * 2^-25) with x0 from
 *         counter (0, row, 3, 0), each fp32 step rounded separately.
 *   fp8:  counter (col/4, row, 4, 0), word w = x[col%4]; code = sign bit 31, exponent
 *         field 4 + bits[3:4] + bits[5:6] (4..10, never NaN), mantissa bits[0:2];
 *         row_scale[row] = 0x1.4dp-8 * (0.75 + (x0 >> 8) * 2^-25), x0 from counter
 *         (0, row, 5, 0), each fp32 step rounded separately.
 *   nvfp4: code of column c = nibble c%8 of word x[(c/8)%4] of counter (c/32, row, 6, 0)
 *         (so code bytes 16k..16k+15 are the 16 output bytes of counter k in order);
 *         scale of block b = word w = x[b%4] of counter (b/4, row, 7, 0): exponent field
 *         5 + bits[0:1] + bit[2] (5..9), mantissa bits[3:5], positive; padding bytes 0;
 *         row_scale[0] = 0x1.4fp-9 (the global scale; a buffer of one fp32).
 * Asynchronous on stream. */
NGRAM_API ngram_status ngram_fill_synthetic(void *table, float *row_scale, uint64_t R, uint32_t d,
                                  ngram_dtype dtype, uint64_t seed, ngram_stream_t stream);

/* ngram_fill_synthetic for columns [col0, col0 + d) of the synthetic table: a column shard
 * (the values of a column do not depend on the table's full width).  col0 must be a
 * multiple of the format's d rule (8 bf16, 16 int8 / fp8, 32 nvfp4); the shard's rows use
 * the format's layout for width d; int8 / fp8 row scales are the full table's. */
NGRAM_API ngram_status ngram_fill_synthetic_cols(void *table, float *row_scale, uint64_t R,
                                                 uint32_t d, uint32_t col0, ngram_dtype dtype,
                                                 uint64_t seed, ngram_stream_t stream);

/* Column-sharded table.  The pages' serving stack keeps "each rank's shard" of the table per
 * GPU at TP4 ("Qwen Brought Back N-Grams. All 51 Billion Parameters of Them.", section
 * "Which is why the offload matters more than the parameter count"; the shard axis is not
 * given).  Here rank r of P holds columns [col0, col0 + d) of every row (a context made over
 * its [R][d] shard, e.g. filled with ngram_fill_synthetic_cols), and every rank holds the
 * full-width residual (tensor-parallel activations).  ngram_forward_shard computes the
 * shard's columns of out = residual + gate * sum_h E[idx_h] for all N tokens and stores them
 * into each of the n_outs output buffers -- this rank's and, through peer mappings
 * (ngram_ipc_open), the other ranks' -- so the lookup and the all-gather of its output are
 * one kernel over NVLink.
 *   residual  device bf16 [N][d_full]; gate fp32 [d_full] (or bf16 [N][d_full] with
 *             NGRAM_FLAG_TOKEN_GATE); outs[p] device-accessible bf16 [N][d_full];
 *   d_full, col0 multiples of 8; col0 + d <= d_full; 1 <= n_outs <= 8.
 * Columns outside the shard are not touched.  The results are bit-identical to
 * ngram_forward over the full table.  The caller orders the ranks' calls before any read of
 * the outputs (e.g. a one-element NCCL all-reduce on the same stream after this call).  HBM
 * residency, no DEDUP / TMA_STAGING (else NGRAM_EUNSUPPORTED). */
NGRAM_API ngram_status ngram_forward_shard(ngram_ctx *ctx, const int32_t *tokens, const int32_t *history,
                                           uint32_t n_seq, uint32_t T, uint32_t d_full, uint32_t col0,
                                           const uint16_t *residual, const void *gate,
                                           uint16_t *const *outs, uint32_t n_outs,
                                           ngram_stream_t stream);

/* CUDA IPC of a device buffer between the processes of one node, for ngram_forward_shard's
 * peer outputs: ngram_ipc_get_handle writes the 64-byte handle of the allocation that
 * starts at dev_ptr (cudaMalloc memory, not a sub-allocation); ngram_ipc_open maps another
 * process's handle into this one (peer access enabled); ngram_ipc_close unmaps it. */
NGRAM_API ngram_status ngram_device_alloc(void **out, uint64_t bytes);   /* cudaMalloc */
NGRAM_API ngram_status ngram_device_free(void *p);                        /* cudaFree; NULL ok */
NGRAM_API ngram_status ngram_ipc_get_handle(const void *dev_ptr, uint8_t handle[64]);
NGRAM_API ngram_status ngram_ipc_open(const uint8_t handle[64], void **dev_ptr);
NGRAM_API ngram_status ngram_ipc_close(void *dev_ptr);

/* Self-test of the kernels' bounded waits: launches one wait that nothing ends (an
 * mbarrier expecting an arrival that never comes), through the same bounded-wait code the
 * TMA-staged gathers use, with a limit of limit_ms (1 .. 2000) instead of their 1 s.  The
 * wait gives up, the kernel sets the context's device error word to code 2 (as a staged
 * gather whose copies never land would) and returns; the context stays usable.  For tests
 * of the failure path; nothing faults or hangs.  Asynchronous on stream. */
NGRAM_API ngram_status ngram_selftest_wait_timeout(ngram_ctx *ctx, uint32_t limit_ms, ngram_stream_t stream);

/* Synchronise the context's device, read and optionally clear its error word.
 * info (may be NULL) receives {code, flat position, bad id, 0}.  Code 1: a token id was
 * out of range (a position with bit 31 set names history entry (position & 0x7FFFFFFF)
 * = 2*s + j).  Code 2: a kernel wait ran past its 1 s deadline (TMA-staged gather).
 * Returns NGRAM_OK if no kernel flagged anything, NGRAM_EDEVICE if one did. */
NGRAM_API ngram_status ngram_get_device_error(ngram_ctx *ctx, uint32_t info[4], int clear);

/* Text of the last failure on the calling thread ("" if none). */
NGRAM_API const char *ngram_last_error(void);

/* Constant name of a status code. */
NGRAM_API const char *ngram_status_string(ngram_status s);

/* Free the context's own allocations (never the caller's buffers).  NULL is a no-op.
 * The caller must make sure no work using ctx is still running. */
NGRAM_API void ngram_destroy(ngram_ctx *ctx);

#ifdef __cplusplus
}
#endif

#endif /* NGRAM_H_ */
