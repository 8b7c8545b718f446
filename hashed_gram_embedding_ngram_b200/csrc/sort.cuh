// sort.cuh -- a stable LSD radix sort of (key, value) pairs and a generic exclusive scan,
// used by the backward pass to list every distinct row's occurrences in ascending order.
//
// The table gradient sums, for each distinct row, the contributions of its occurrences
// in ascending occurrence order (i = token * H + head), so the result is the same bit for
// bit on every run.  Sorting the occurrence indices by their row's position u in the
// distinct-row list with a stable sort leaves each row's occurrences in ascending order.
//
// Radix sort: 8-bit digits, least significant first, one pass per digit.  A tile of
// kSortTile = 2048 consecutive keys is handled by one CTA of 256 threads in 8 rounds of
// 256 keys (round r holds keys r * 256 .. r * 256 + 255 of the tile, thread j key j), so
// keys are ranked in tile order:
//   hist:    the digit counts of every tile, stored digit-major ([digit][tile]) so that
//            one exclusive scan of the whole array gives every (digit, tile) its output
//            offset;
//   scatter: per round, __match_any_sync groups the lanes of a warp with equal digits
//            (the lane's rank = its peers below it), each warp's count per digit goes to
//            shared memory, and a key's position is the tile's offset for its digit +
//            the keys of that digit in earlier rounds + in earlier warps of this round +
//            its rank in the warp.  Stable by construction.
// Every kernel opens with allow_dependents(); grid_dependency_wait(), so the passes may be
// launched as programmatic dependents of one another.
#pragma once

#include <cstdint>

#include "device_common.cuh"

namespace ngram {

constexpr uint32_t kSortTile = 2048;      // keys per tile (256 threads x 8 rounds)
constexpr uint32_t kSortRadix = 256;      // 8-bit digits
constexpr uint32_t kScanChunk = 1024;     // entries per block of the generic scan

__global__ void __launch_bounds__(256) k_radix_hist(const uint32_t *__restrict__ keys, uint32_t M,
                                                    uint32_t shift, uint32_t n_tiles,
                                                    uint32_t *__restrict__ hist) {
    allow_dependents();
    grid_dependency_wait();
    __shared__ uint32_t h[kSortRadix];
    for (uint32_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        h[threadIdx.x] = 0;
        __syncthreads();
        const uint32_t base = tile * kSortTile;
#pragma unroll
        for (uint32_t r = 0; r < kSortTile / 256u; ++r) {
            const uint32_t p = base + r * 256u + threadIdx.x;
            if (p < M) atomicAdd(h + ((keys[p] >> shift) & (kSortRadix - 1u)), 1u);
        }
        __syncthreads();
        hist[threadIdx.x * n_tiles + tile] = h[threadIdx.x];
        __syncthreads();
    }
}

// vals_in == nullptr: the value of key p is p / val_div (the first pass over occurrences
// p = token * H + head takes the token, val_div = H).
__global__ void __launch_bounds__(256) k_radix_scatter(const uint32_t *__restrict__ keys_in,
                                                       const uint32_t *__restrict__ vals_in,
                                                       uint32_t val_div, uint32_t M, uint32_t shift,
                                                       uint32_t n_tiles,
                                                       const uint32_t *__restrict__ offsets,
                                                       uint32_t *__restrict__ keys_out,
                                                       uint32_t *__restrict__ vals_out) {
    allow_dependents();
    grid_dependency_wait();
    __shared__ uint32_t run[kSortRadix];          // keys of each digit placed so far + offset
    __shared__ uint16_t wcnt[8][kSortRadix];      // this round's count per (warp, digit)
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (uint32_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        run[threadIdx.x] = offsets[threadIdx.x * n_tiles + tile];
        const uint32_t base = tile * kSortTile;
        for (uint32_t r = 0; r < kSortTile / 256u; ++r) {
#pragma unroll
            for (uint32_t w = 0; w < 8; ++w) wcnt[w][threadIdx.x] = 0;
            __syncthreads();
            const uint32_t p = base + r * 256u + threadIdx.x;
            const bool valid = p < M;
            const uint32_t key = valid ? keys_in[p] : 0u;
            // invalid lanes take digit 256, which no valid lane has
            const uint32_t digit = valid ? ((key >> shift) & (kSortRadix - 1u)) : kSortRadix;
            const uint32_t peers = __match_any_sync(0xFFFFFFFFu, digit);
            const uint32_t rank = __popc(peers & lt_mask);
            if (valid && rank == 0) wcnt[warp][digit] = static_cast<uint16_t>(__popc(peers));
            __syncthreads();
            if (valid) {
                uint32_t pos = run[digit] + rank;
                for (uint32_t w = 0; w < warp; ++w) pos += wcnt[w][digit];
                keys_out[pos] = key;
                vals_out[pos] = vals_in ? vals_in[p] : p / val_div;
            }
            __syncthreads();
            uint32_t add = 0;
#pragma unroll
            for (uint32_t w = 0; w < 8; ++w) add += wcnt[w][threadIdx.x];
            run[threadIdx.x] += add;
            __syncthreads();
        }
    }
}

// Exclusive scan of in[0..n) into out (in may equal out), three steps: each block of
// kScanChunk entries scans locally and records its total; one CTA scans the totals
// (k_dedup_scan_blocks); k_scan_add adds them back.
__global__ void __launch_bounds__(256) k_scan_local(const uint32_t *in, uint32_t n, uint32_t *out,
                                                    uint32_t *__restrict__ block_total) {
    allow_dependents();
    grid_dependency_wait();
    __shared__ uint32_t warp_tot[8];
    const uint32_t base = blockIdx.x * kScanChunk + threadIdx.x * 4u;
    uint32_t v[4], run = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[j] = (base + j < n) ? in[base + j] : 0u;
        run += v[j];
    }
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    uint32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= static_cast<uint32_t>(o)) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    uint32_t p = incl - run;
    for (uint32_t w = 0; w < warp; ++w) p += warp_tot[w];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (base + j < n) out[base + j] = p;
        p += v[j];
    }
    if (threadIdx.x == 255) block_total[blockIdx.x] = p;
}

__global__ void __launch_bounds__(256) k_scan_add(uint32_t *out, uint32_t n,
                                                  const uint32_t *__restrict__ block_off) {
    allow_dependents();
    grid_dependency_wait();
    const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] += block_off[i / kScanChunk];
}

}  // namespace ngram
