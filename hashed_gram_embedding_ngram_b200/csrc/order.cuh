// order.cuh -- process a batch's tokens grouped by their bigram context, so that tokens
// that read the same rows run back to back and the repeats are served by L2.
//
// With Zipf-distributed text ("Why N-Gram Lookup Works Without Latency Penalties" in
// Section 1 of "Qwen 3.8 Flash-Next Deep Dive ...": frequent patterns recur) many
// tokens share a bigram context (w_{t-1}, w_t): they read the same 8 bigram rows, and if
// w_{t-2} also matches, the same 16.  In batch order such repeats are far apart and L2
// rarely still holds the row; grouped, the second read is an L2 hit.
//
// A counting sort on a 13-bit hash of the bigram key (w1 << 21 | w0) makes perm[N]: a
// histogram, one exclusive scan over the 8,192 buckets (in shared memory), and a
// scatter with per-bucket atomic cursors.  The order inside a bucket depends on timing,
// which is harmless: every token's output is computed and written the same way in any
// order.  Each kernel waits for the previous grid of its stream before touching memory
// (grid_dependency_wait), so the three may be launched as programmatic dependents.
#pragma once

#include "device_common.cuh"

namespace ngram {

constexpr uint32_t kOrderBucketsLog2 = 13;
constexpr uint32_t kOrderBuckets = 1u << kOrderBucketsLog2;

// Bucket counts, one thread per token.  With idx_out, the same thread also writes the
// token's row ids idx_out[t][h] = head_row(h, context) for h < H (the hash-once step of
// the gather, folded into this pass over the contexts).
__global__ void __launch_bounds__(256) k_order_count(const int32_t *__restrict__ tokens,
                                                     const int32_t *__restrict__ history,
                                                     uint32_t T, uint32_t N, const HashArgs a,
                                                     uint32_t *err, uint32_t *__restrict__ bucket_of,
                                                     uint32_t *hist, uint32_t *__restrict__ idx_out) {
    allow_dependents();
    grid_dependency_wait();
    for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < N; t += gridDim.x * blockDim.x) {
        uint32_t w0, w1, w2;
        token_context(tokens, history, t, T, a, err, w0, w1, w2);
        const uint64_t k2 = (static_cast<uint64_t>(w1) << 21) | w0;
        const uint32_t b = static_cast<uint32_t>(splitmix64_step(k2) >> (64 - kOrderBucketsLog2));
        bucket_of[t] = b;
        atomicAdd(hist + b, 1u);
        if (idx_out != nullptr) {
            uint32_t *dst = idx_out + static_cast<size_t>(t) * a.n_heads;
            for (uint32_t h = 0; h < a.n_heads; ++h) dst[h] = head_row(h, w0, w1, w2, a);
        }
    }
}

// Exclusive scan of the bucket counts in place by one CTA of 1024 threads: coalesced
// copy into shared memory, each thread scans 8 consecutive buckets, warp and block
// offsets, coalesced copy back.
__global__ void __launch_bounds__(1024) k_order_scan(uint32_t *hist) {
    __shared__ uint32_t sh[kOrderBuckets];
    __shared__ uint32_t warp_tot[32];
    constexpr uint32_t kPer = kOrderBuckets / 1024;
    allow_dependents();
    grid_dependency_wait();
    for (uint32_t i = threadIdx.x; i < kOrderBuckets; i += 1024) sh[i] = hist[i];
    __syncthreads();
    const uint32_t base = threadIdx.x * kPer;
    uint32_t local = 0;
#pragma unroll
    for (uint32_t j = 0; j < kPer; ++j) local += sh[base + j];
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= static_cast<uint32_t>(o)) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    uint32_t run = incl - local;
    for (uint32_t w = 0; w < warp; ++w) run += warp_tot[w];
#pragma unroll
    for (uint32_t j = 0; j < kPer; ++j) {
        const uint32_t c = sh[base + j];
        sh[base + j] = run;
        run += c;
    }
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < kOrderBuckets; i += 1024) hist[i] = sh[i];
}

__global__ void __launch_bounds__(256) k_order_scatter(const uint32_t *__restrict__ bucket_of,
                                                       uint32_t N, uint32_t *cursor,
                                                       uint32_t *__restrict__ perm) {
    allow_dependents();
    grid_dependency_wait();
    for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < N; t += gridDim.x * blockDim.x)
        perm[atomicAdd(cursor + bucket_of[t], 1u)] = t;
}

}  // namespace ngram
