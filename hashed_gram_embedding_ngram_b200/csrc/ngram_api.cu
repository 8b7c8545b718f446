// ngram_api.cu -- host side of libngram.so: argument checks, context, launches.
//
// Every entry point validates its arguments before touching CUDA and reports through
// an ngram_status; nothing here aborts the process.  All compute is asynchronous on
// the caller's stream.  The operation and the definitions it follows are stated in
// include/ngram.h.
#include <cstdio>
#include <cstring>
#include <cstdarg>
#include <string>

#include <cuda_runtime.h>

#include "ngram.h"
#include "device_common.cuh"
#include "fill.cuh"
#include "gather.cuh"

using namespace ngram;

struct ngram_ctx {
    const void *table;
    const float *row_scale;
    uint64_t R;
    uint32_t d;
    ngram_dtype dtype;
    ngram_residency where;
    ngram_hash_params hp;
    uint32_t max_tokens;
    uint64_t barrett_m;
    int device;
    int num_sms;
    int gather_blocks_per_sm;
    uint32_t *d_err;            // 4 words, owned
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

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
    if (hp.flags != 0 || hp.reserved != 0)
        return fail(NGRAM_EINVAL, "flags/reserved must be 0");
    return NGRAM_OK;
}

HashArgs hash_args(const ngram_ctx *c) {
    HashArgs a;
    a.base_seed = c->hp.base_seed;
    a.R = c->R;
    a.barrett_m = c->barrett_m;
    a.n_bigram = c->hp.n_bigram_heads;
    a.n_heads = c->hp.n_bigram_heads + c->hp.n_trigram_heads;
    a.pad_id = c->hp.pad_id;
    a.vocab = c->hp.vocab_size;
    return a;
}

// Common checks of the token batch of one call.
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
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (cur != c->device)
        return fail(NGRAM_EINVAL, "current device %d is not the context's device %d", cur, c->device);
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

ngram_status ngram_init(ngram_ctx **out, const void *table, const float *row_scale, uint64_t R,
                        uint32_t d, ngram_dtype dtype, ngram_residency where,
                        const ngram_hash_params *hp, uint32_t max_tokens) {
    if (out == nullptr) return fail(NGRAM_EINVAL, "out is NULL");
    *out = nullptr;
    if (table == nullptr) return fail(NGRAM_EINVAL, "table is NULL");
    if (!aligned16(table)) return fail(NGRAM_EINVAL, "table must be 16-byte aligned");
    if (R == 0 || R > 0xFFFFFFFFull) return fail(NGRAM_EINVAL, "R must be in [1, 2^32 - 1]");
    if (dtype != NGRAM_BF16 && dtype != NGRAM_INT8_ROWSCALE)
        return fail(NGRAM_EINVAL, "unknown dtype %d", static_cast<int>(dtype));
    if (dtype == NGRAM_BF16 && (d == 0 || d % 8 != 0))
        return fail(NGRAM_EINVAL, "bf16 rows need d %% 8 == 0 and d > 0, got %u", d);
    if (dtype == NGRAM_INT8_ROWSCALE && (d == 0 || d % 16 != 0))
        return fail(NGRAM_EINVAL, "int8 rows need d %% 16 == 0 and d > 0, got %u", d);
    if (dtype == NGRAM_INT8_ROWSCALE && row_scale == nullptr)
        return fail(NGRAM_EINVAL, "int8 rows need row_scale");
    if (dtype == NGRAM_BF16 && row_scale != nullptr)
        return fail(NGRAM_EINVAL, "row_scale is only for int8 rows");
    if (where != NGRAM_RES_HBM && where != NGRAM_RES_HOST_UVA && where != NGRAM_RES_HOST_DMA &&
        where != NGRAM_RES_HOST_AUTO)
        return fail(NGRAM_EINVAL, "unknown residency %d", static_cast<int>(where));
    if (max_tokens == 0) return fail(NGRAM_EINVAL, "max_tokens must be >= 1");
    ngram_hash_params p;
    if (hp != nullptr) p = *hp; else ngram_default_hash_params(&p);
    ngram_status st = check_hash_params(p);
    if (st != NGRAM_OK) return st;
    const uint32_t n_strips = (d / 8 + 31) / 32;
    if (static_cast<uint64_t>(max_tokens) * n_strips > 0xFFFFFFFFull ||
        static_cast<uint64_t>(max_tokens) * NGRAM_MAX_HEADS > 0xFFFFFFFFull)
        return fail(NGRAM_EINVAL, "max_tokens %u too large for d = %u", max_tokens, d);
    if (where != NGRAM_RES_HBM)
        return fail(NGRAM_EUNSUPPORTED, "host-resident tables are not built yet");

    // ---- CUDA from here on
    ngram_ctx *c = new ngram_ctx();
    c->table = table;
    c->row_scale = row_scale;
    c->R = R;
    c->d = d;
    c->dtype = dtype;
    c->where = where;
    c->hp = p;
    c->max_tokens = max_tokens;
    c->barrett_m = (R == 1) ? 0ull
                            : static_cast<uint64_t>((static_cast<unsigned __int128>(1) << 64) / R);
    c->d_err = nullptr;
    cudaError_t e = cudaGetDevice(&c->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
    if (e == cudaSuccess)
        e = (dtype == NGRAM_BF16)
                ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c->gather_blocks_per_sm,
                                                                k_gather_bf16<16>, 256, 0)
                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c->gather_blocks_per_sm,
                                                                k_gather_int8<16>, 256, 0);
    if (e == cudaSuccess) e = cudaMalloc(&c->d_err, 4 * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemset(c->d_err, 0, 4 * sizeof(uint32_t));
    if (e != cudaSuccess) {
        ngram_status s = cuda_fail(e, "ngram_init");
        if (c->d_err) cudaFree(c->d_err);
        delete c;
        return s;
    }
    if (c->gather_blocks_per_sm < 1) c->gather_blocks_per_sm = 1;
    *out = c;
    return NGRAM_OK;
}

ngram_status ngram_forward(ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                           uint32_t n_seq, uint32_t T, const uint16_t *residual, const float *gate,
                           uint16_t *out, ngram_stream_t stream) {
    uint64_t N = 0;
    ngram_status st = check_batch(c, tokens, n_seq, T, &N);
    if (st != NGRAM_OK || N == 0) return st;
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

    GatherArgs g;
    g.h = hash_args(c);
    g.table = c->table;
    g.row_scale = c->row_scale;
    g.tokens = tokens;
    g.history = history;
    g.residual = residual;
    g.gate = gate;
    g.out = out;
    g.err = c->d_err;
    g.T = T;
    g.N = static_cast<uint32_t>(N);
    g.d = c->d;
    const uint32_t cols_per_lane = (c->dtype == NGRAM_BF16) ? 8u : 16u;
    g.n_strips = (c->d / cols_per_lane + 31) / 32;
    const uint32_t resident_warps = static_cast<uint32_t>(c->num_sms) * c->gather_blocks_per_sm * 8u;
    // Few tokens: one strip per warp (lowest latency).  Many: a warp keeps its token.
    g.strips_per_item = (static_cast<uint64_t>(N) * g.n_strips <= 2ull * resident_warps) ? 1u : g.n_strips;
    g.groups_per_token = (g.n_strips + g.strips_per_item - 1) / g.strips_per_item;
    const uint64_t items = N * g.groups_per_token;
    const uint64_t max_blocks = static_cast<uint64_t>(c->num_sms) * c->gather_blocks_per_sm;
    uint64_t blocks = (items + 7) / 8;
    if (blocks > max_blocks) blocks = max_blocks;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const unsigned nb = static_cast<unsigned>(blocks);
    if (c->dtype == NGRAM_BF16) {
        if (g.h.n_heads == 16) k_gather_bf16<16><<<nb, 256, 0, s>>>(g);
        else k_gather_bf16<0><<<nb, 256, 0, s>>>(g);
    } else {
        if (g.h.n_heads == 16) k_gather_int8<16><<<nb, 256, 0, s>>>(g);
        else k_gather_int8<0><<<nb, 256, 0, s>>>(g);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "gather kernel launch");
    return NGRAM_OK;
}

ngram_status ngram_hash_indices(ngram_ctx *c, const int32_t *tokens, const int32_t *history,
                                uint32_t n_seq, uint32_t T, uint32_t *idx_out,
                                ngram_stream_t stream) {
    uint64_t N = 0;
    ngram_status st = check_batch(c, tokens, n_seq, T, &N);
    if (st != NGRAM_OK || N == 0) return st;
    if (idx_out == nullptr) return fail(NGRAM_EINVAL, "idx_out is NULL");
    const HashArgs a = hash_args(c);
    const uint64_t total = N * a.n_heads;
    uint64_t blocks = (total + 255) / 256;
    const uint64_t cap = static_cast<uint64_t>(c->num_sms) * 8;
    if (blocks > cap) blocks = cap;
    k_hash_indices<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        a, tokens, history, T, static_cast<uint32_t>(N), c->d_err, idx_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "k_hash_indices launch");
    return NGRAM_OK;
}

ngram_status ngram_fill_synthetic(void *table, float *row_scale, uint64_t R, uint32_t d,
                                  ngram_dtype dtype, uint64_t seed, ngram_stream_t stream) {
    if (table == nullptr) return fail(NGRAM_EINVAL, "table is NULL");
    if (!aligned16(table)) return fail(NGRAM_EINVAL, "table must be 16-byte aligned");
    if (R == 0 || R > 0xFFFFFFFFull) return fail(NGRAM_EINVAL, "R must be in [1, 2^32 - 1]");
    if (dtype == NGRAM_BF16 && (d == 0 || d % 8 != 0))
        return fail(NGRAM_EINVAL, "bf16 rows need d %% 8 == 0 and d > 0, got %u", d);
    if (dtype == NGRAM_INT8_ROWSCALE && (d == 0 || d % 16 != 0 || row_scale == nullptr))
        return fail(NGRAM_EINVAL, "int8 rows need d %% 16 == 0 and a row_scale buffer");
    if (dtype != NGRAM_BF16 && dtype != NGRAM_INT8_ROWSCALE)
        return fail(NGRAM_EINVAL, "unknown dtype %d", static_cast<int>(dtype));
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "ngram_fill_synthetic");
    uint64_t blocks = static_cast<uint64_t>(sms) * 8;
    if (blocks > R) blocks = R;
    const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == NGRAM_BF16)
        k_fill_bf16<<<static_cast<unsigned>(blocks), 256, 0, s>>>(static_cast<uint16_t *>(table), R, d, k0, k1);
    else
        k_fill_int8<<<static_cast<unsigned>(blocks), 256, 0, s>>>(static_cast<int8_t *>(table), row_scale, R, d, k0, k1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "k_fill launch");
    return NGRAM_OK;
}

ngram_status ngram_get_device_error(ngram_ctx *c, uint32_t info[4], int clear) {
    if (c == nullptr) return fail(NGRAM_EINVAL, "ctx is NULL");
    uint32_t h[4] = {0, 0, 0, 0};
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(h, c->d_err, sizeof(h), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear) e = cudaMemset(c->d_err, 0, sizeof(h));
    if (e != cudaSuccess) return cuda_fail(e, "ngram_get_device_error");
    if (info != nullptr) memcpy(info, h, sizeof(h));
    if (h[0] != 0)
        return fail(NGRAM_EDEVICE, "token id %d out of [0, %u) at %s %u", static_cast<int32_t>(h[2]),
                    c->hp.vocab_size, (h[1] & 0x80000000u) ? "history entry" : "flat position",
                    h[1] & 0x7FFFFFFFu);
    return NGRAM_OK;
}

void ngram_destroy(ngram_ctx *c) {
    if (c == nullptr) return;
    if (c->d_err) cudaFree(c->d_err);
    delete c;
}

}  // extern "C"
