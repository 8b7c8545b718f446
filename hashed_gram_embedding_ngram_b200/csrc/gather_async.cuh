// gather_async.cuh -- the NVFP4 gather with each warp's next item copied into shared
// memory by cp.async while the warp decodes the current one (same operation and
// arithmetic as k_gather_nvfp4, so the same bits).
//
// k_gather_nvfp4 keeps a token's 16 code fragments and scale bytes in registers from the
// loads to the decode, so while a warp decodes nothing of its own is in flight, and the
// registers the loads hold cap the warps per SM.  Here every lane copies, per head, its
// 8 code bytes and the 4-byte word holding its block scale (cp.async.ca, 8 + 4 bytes)
// into a warp-private slot of a double buffer in shared memory, for the item after the
// one it is decoding; it then waits only for the older group (cp.async.wait_group 1).
// A lane reads back only the bytes it copied itself, so no barrier is needed between the
// lanes, and no wait spins.
#pragma once

#include "gather_int8.cuh"

namespace ngram {

#ifndef NGRAM_ASYNC_MIN_BLOCKS        // resident CTAs per SM the register budget targets
#define NGRAM_ASYNC_MIN_BLOCKS 2
#endif
constexpr uint32_t kAsyncWarps = 8;   // warps per CTA (256 threads)
// shared memory per warp: 2 buffers x 16 heads x 32 lanes x (8 code + 4 scale) bytes
constexpr uint32_t kAsyncWarpBytes = 2u * 16u * 32u * 12u;

__device__ __forceinline__ void cp_async_8(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_older() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

template <int kH, bool kTokGate = false>
__global__ void __launch_bounds__(256, NGRAM_ASYNC_MIN_BLOCKS) k_gather_nvfp4_async(const GatherArgs g) {
    extern __shared__ __align__(16) uint8_t async_smem[];
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t wib = threadIdx.x >> 5;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t nvec = g.d >> 4;                       // scale blocks per row
    const uint32_t code_bytes = g.d >> 1;
    const size_t rb = code_bytes + 16u * ((nvec + 15u) >> 4);
    const uint32_t n_items = g.N * g.groups_per_token;
    const uint8_t *__restrict__ table = static_cast<const uint8_t *>(g.table);
    const float gs = __ldg(g.row_scale);
    // this warp's slots: codes [buf][head][lane] (8 B), scale words [buf][head][lane] (4 B)
    uint8_t *wbase = async_smem + wib * kAsyncWarpBytes;
    const uint32_t codes_s = static_cast<uint32_t>(__cvta_generic_to_shared(wbase));
    const uint32_t scales_s = codes_s + 2u * 16u * 32u * 8u;
    const uint2 *codes_p = reinterpret_cast<const uint2 *>(wbase);
    const uint32_t *scales_p = reinterpret_cast<const uint32_t *>(wbase + 2u * 16u * 32u * 8u);

    // copy this lane's fragments of item `item` into buffer `b` (lanes >= the row's
    // blocks copy nothing); returns nothing, the copies join the open group
    auto issue = [&](uint32_t item, uint32_t b) {
        const uint32_t pos = item / g.groups_per_token;
        const uint32_t grp = item - pos * g.groups_per_token;
        const uint32_t tok = g.perm ? __ldg(g.perm + pos) : pos;
        const uint32_t my_row = warp_head_row(g, tok, lane, H);
        const uint32_t v = grp * g.strips_per_item * 32u + lane;   // one strip per item
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            const uint32_t row = __shfl_sync(0xFFFFFFFFu, my_row, h);
            if ((kH || h < static_cast<int>(H)) && v < nvec) {
                const uint8_t *r = table + static_cast<size_t>(row) * rb;
                const uint32_t slot = (b * 16u + h) * 32u + lane;
                cp_async_8(codes_s + slot * 8u, r + v * 8u);
                cp_async_4(scales_s + slot * 4u, r + code_bytes + (v & ~3u));
            }
        }
    };

    uint32_t item = warp, k = 0;
    if (item < n_items) issue(item, 0);
    cp_async_commit();
    for (; item < n_items; item += n_warps, ++k) {
        const uint32_t b = k & 1u;
        const uint32_t pos = item / g.groups_per_token;
        const uint32_t grp = item - pos * g.groups_per_token;
        const uint32_t tok = g.perm ? __ldg(g.perm + pos) : pos;
        const uint32_t v = grp * g.strips_per_item * 32u + lane;
        const bool active = v < nvec;
        const size_t tok_off = static_cast<size_t>(tok) * g.d;
        uint4 r0 = make_uint4(0u, 0u, 0u, 0u), r1 = r0;
        if (active) {                        // the residual load overlaps the next issue
            r0 = ld_na_v4(g.residual + tok_off + v * 16u);
            r1 = ld_na_v4(g.residual + tok_off + v * 16u + 8u);
        }
        if (item + n_warps < n_items) issue(item + n_warps, b ^ 1u);
        cp_async_commit();
        cp_async_wait_older();               // this item's copies (this lane's) have landed
        if (!active) continue;
        float2 acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            if (kH || h < static_cast<int>(H)) {
                const uint32_t slot = (b * 16u + h) * 32u + lane;
                const uint2 e = codes_p[slot];
                const uint32_t bs = (scales_p[slot] >> (8u * (v & 3u))) & 0xFFu;
                const float cs = __fmul_rn(e4m3_to_float(bs), gs);
                const float2 s2 = make_float2(cs, cs);
                float2 q[4];
                e2m1x8_to_float(e.x, q);
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[j] = fma2(q[j], s2, acc[j]);
                e2m1x8_to_float(e.y, q);
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[4 + j] = fma2(q[j], s2, acc[4 + j]);
            }
        }
        store_gated16<kTokGate>(g, tok_off, v, r0, r1, acc);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
}

}  // namespace ngram
