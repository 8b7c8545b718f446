// dedup.cuh -- per-batch row dedup: the distinct rows of a batch and an inverse map.
//
// The lookup reads 16 rows per token ("Qwen Brought Back N-Grams. All 51 Billion
// Parameters of Them.", "Key Takeaways"); with Zipf-distributed text the same bigram
// and trigram contexts recur, so a batch reads some rows several times.  Rows that
// must cross PCIe (the host-resident table of "Qwen3.8-Flash-Next: A 51B N-gram
// Embedding Table with Heterogeneous Memory Prefetch", Key point 3) should cross once.
//
// Given idx[M] (M = N * H row ids), produce
//   uniq[U]  the distinct ids in order of first appearance in idx,
//   inv[M]   for every entry, the position of its row in uniq (uniq[inv[i]] == idx[i]),
//   count    U.
// The order is a pure function of idx (no dependence on thread timing), so staging
// buffers built from it are identical from run to run.
//
// Steps (each a grid-wide pass):
//   1. insert: open-addressing table of P >= 2M slots (linear probing, atomicCAS);
//      every entry records its slot and atomicMin's its own index into first[slot];
//   2. scan_local: flag[i] = (first[slot[i]] == i) (a first occurrence); exclusive scan
//      of the flags inside each 1024-entry block, block totals to block_sum;
//   3. scan_blocks: one CTA scans the block totals (and writes U);
//   4. emit: each first occurrence i takes u = its global rank: uniq[u] = idx[i],
//      uid[slot[i]] = u;
//   5. inverse: inv[i] = uid[slot[i]].
// Steps 1-5 open with allow_dependents(); grid_dependency_wait(): each may be launched as a
// programmatic dependent of the step before and waits for it before touching memory.
#pragma once

#include "device_common.cuh"

namespace ngram {

constexpr uint32_t kEmptyKey = 0xFFFFFFFFu;   // never a row id (R <= 2^32 - 1)
constexpr uint32_t kScanBlock = 1024;         // entries per scan block (256 threads x 4)

__device__ __forceinline__ uint32_t dedup_home(uint32_t row, uint32_t log2p) {
    return (row * 0x9E3779B1u) >> (32u - log2p);          // Fibonacci hashing
}

__global__ void __launch_bounds__(256) k_dedup_insert(const uint32_t *__restrict__ idx, uint32_t M,
                                                      uint32_t *keys, uint32_t *first,
                                                      uint32_t *__restrict__ slot_of, uint32_t log2p) {
    allow_dependents();
    grid_dependency_wait();
    const uint32_t mask = (1u << log2p) - 1u;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < M; i += gridDim.x * blockDim.x) {
        const uint32_t row = idx[i];
        uint32_t s = dedup_home(row, log2p);
        // the table holds at most M < P/2 keys, so a free slot is found within P probes
        for (uint32_t probe = 0; probe <= mask; ++probe) {
            const uint32_t prev = atomicCAS(keys + s, kEmptyKey, row);
            if (prev == kEmptyKey || prev == row) break;
            s = (s + 1u) & mask;
        }
        slot_of[i] = s;
        atomicMin(first + s, i);
    }
}

// Block-local exclusive scan of the first-occurrence flags (256 threads x 4 entries).
__global__ void __launch_bounds__(256) k_dedup_scan_local(const uint32_t *__restrict__ slot_of,
                                                          const uint32_t *__restrict__ first,
                                                          uint32_t M, uint32_t *__restrict__ pos,
                                                          uint32_t *__restrict__ block_sum) {
    allow_dependents();
    grid_dependency_wait();
    __shared__ uint32_t warp_tot[8];
    const uint32_t base = blockIdx.x * kScanBlock + threadIdx.x * 4u;
    uint32_t f[4], run = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t i = base + j;
        f[j] = (i < M && first[slot_of[i]] == i) ? 1u : 0u;
        run += f[j];
    }
    // inclusive warp scan of the per-thread totals
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    uint32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= static_cast<uint32_t>(o)) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    uint32_t warp_off = 0;
    for (uint32_t w = 0; w < warp; ++w) warp_off += warp_tot[w];
    uint32_t p = warp_off + incl - run;                 // exclusive prefix of this thread
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t i = base + j;
        if (i < M) pos[i] = p;
        p += f[j];
    }
    if (threadIdx.x == 255) block_sum[blockIdx.x] = warp_off + incl;
}

// Exclusive scan of the block totals by one CTA; writes U to *count.
__global__ void __launch_bounds__(1024) k_dedup_scan_blocks(uint32_t *block_sum, uint32_t nb,
                                                            uint32_t *count) {
    allow_dependents();
    grid_dependency_wait();
    __shared__ uint32_t warp_tot[32];
    __shared__ uint32_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    for (uint32_t base = 0; base < nb; base += 1024) {
        const uint32_t i = base + threadIdx.x;
        const uint32_t v = (i < nb) ? block_sum[i] : 0u;
        uint32_t incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= static_cast<uint32_t>(o)) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        uint32_t warp_off = 0;
        for (uint32_t w = 0; w < warp; ++w) warp_off += warp_tot[w];
        const uint32_t c = carry;
        if (i < nb) block_sum[i] = c + warp_off + incl - v;
        __syncthreads();
        if (threadIdx.x == 1023) carry = c + warp_off + incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) *count = carry;
}

__global__ void __launch_bounds__(256) k_dedup_emit(const uint32_t *__restrict__ idx,
                                                    const uint32_t *__restrict__ slot_of,
                                                    const uint32_t *__restrict__ first,
                                                    const uint32_t *__restrict__ pos,
                                                    const uint32_t *__restrict__ block_off, uint32_t M,
                                                    uint32_t *__restrict__ uniq,
                                                    uint32_t *__restrict__ uid) {
    allow_dependents();
    grid_dependency_wait();
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < M; i += gridDim.x * blockDim.x) {
        const uint32_t s = slot_of[i];
        if (first[s] == i) {
            const uint32_t u = block_off[i / kScanBlock] + pos[i];
            uniq[u] = idx[i];
            uid[s] = u;
        }
    }
}

__global__ void __launch_bounds__(256) k_dedup_inverse(const uint32_t *__restrict__ slot_of,
                                                       const uint32_t *__restrict__ uid, uint32_t M,
                                                       uint32_t *__restrict__ inv) {
    allow_dependents();
    grid_dependency_wait();
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < M; i += gridDim.x * blockDim.x)
        inv[i] = uid[slot_of[i]];
}

// Copy the U unique rows (and per-row scales) of the table into a dense staging buffer.
// The copy is flat over the U * nv 16-byte vectors (vector f = row u, column vector v):
// a warp owns 512 consecutive vectors at a time and a lane issues its 16 loads before its
// first store, so every warp keeps 8 KB in flight whatever the row width.  Read from host
// memory over PCIe, the link's throughput follows the bytes in flight (the latency grows
// with the queue), so a few CTAs reach the link's rate only with this depth.
constexpr uint32_t kCompactBatch = 16;

__global__ void __launch_bounds__(256) k_compact_rows(const uint8_t *__restrict__ table,
                                                      const float *__restrict__ row_scale,
                                                      const uint32_t *__restrict__ uniq,
                                                      const uint32_t *__restrict__ count,
                                                      uint32_t row_bytes, uint8_t *__restrict__ stage,
                                                      float *__restrict__ stage_scale) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t U = *count;
    const uint32_t nv = row_bytes >> 4;
    const uint64_t total = static_cast<uint64_t>(U) * nv;
    const uint64_t warp = (static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const uint64_t n_warps = (static_cast<uint64_t>(gridDim.x) * blockDim.x) >> 5;
    uint4 *dst = reinterpret_cast<uint4 *>(stage);
    for (uint64_t base = warp * 32u * kCompactBatch; base < total; base += n_warps * 32u * kCompactBatch) {
        uint4 x[kCompactBatch];
#pragma unroll
        for (uint32_t j = 0; j < kCompactBatch; ++j) {
            const uint64_t f = base + 32u * j + lane;
            if (f < total) {
                // 32-bit division whenever the vector index fits (every batch up to 2^32 vectors)
                const uint32_t u = (total >> 32) ? static_cast<uint32_t>(f / nv)
                                                 : static_cast<uint32_t>(f) / nv;
                const uint32_t v = static_cast<uint32_t>(f - static_cast<uint64_t>(u) * nv);
                x[j] = ld_stream_v4(table + static_cast<size_t>(uniq[u]) * row_bytes + 16u * v);
            }
        }
#pragma unroll
        for (uint32_t j = 0; j < kCompactBatch; ++j) {
            const uint64_t f = base + 32u * j + lane;
            if (f < total) dst[f] = x[j];
        }
    }
    if (row_scale != nullptr) {
        for (uint32_t u = blockIdx.x * blockDim.x + threadIdx.x; u < U; u += gridDim.x * blockDim.x)
            stage_scale[u] = row_scale[uniq[u]];
    }
}

}  // namespace ngram
