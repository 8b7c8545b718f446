// gather_nvfp4.cuh -- the gather for NVFP4 rows: FP4 E2M1 codes with one E4M3 scale per
// 16 columns and one fp32 scale for the whole table.
//
// The 4-bit table of "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with
// Heterogeneous Memory Prefetch" (its architecture figure: 51B parameters, ~25.5 GB at
// FP4; "Qwen3.8-Flash-Next: A 125B MoE for the Local Stack?", section "Hardware math for
// self-hosting", weighs 4-bit n-gram tables too).  Same operation as k_gather_bf16, with
// row value  q * bs * gs,  q the E2M1 value of the code, bs its E4M3 block scale and gs the
// table's fp32 global scale: per head in order acc = fma(q, bs, acc) -- both as f16 into
// one fp32 fma (fma.rn.f32.f16), q * bs exact, one rounding -- and the global scale
// multiplies the sum once, e = fp32(gs * acc).  The block scales of heads 2k and 2k+1
// go to f16 in one conversion (cvt.rn.f16x2.e4m3x2 of the two bytes), which measured
// 3.7% faster than one conversion per head.
//
// Row layout (rb = d/2 + ceil16(d/16) bytes, a multiple of 16 for d % 32 == 0): d/2 code
// bytes, column 2j in the low nibble of byte j; then d/16 block-scale bytes; then zero
// padding.  A lane owns 16 columns = one scale block: 8 code bytes and 1 scale byte per
// head, so a 32-lane strip covers 512 columns as in the 8-bit gather.
#pragma once

#include "gather_int8.cuh"

namespace ngram {

#ifndef NGRAM_NVFP4_MIN_BLOCKS        // resident CTAs per SM the register budget targets
#define NGRAM_NVFP4_MIN_BLOCKS 2
#endif

template <int kH, bool kTokGate = false>
__global__ void __launch_bounds__(256, NGRAM_NVFP4_MIN_BLOCKS) k_gather_nvfp4(const GatherArgs g) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t nvec = g.d >> 4;                       // scale blocks per row
    const uint32_t code_bytes = g.d >> 1;
    const size_t rb = code_bytes + 16u * ((nvec + 15u) >> 4);
    const uint32_t n_items = g.N * g.groups_per_token;
    const uint8_t *__restrict__ table = static_cast<const uint8_t *>(g.table);
    const uint64_t seed = head_seed(lane, g.h);           // arithmetic only: before the wait
    if (g.trigger_early) allow_dependents();
    grid_dependency_wait();
    const float gs = __ldg(g.row_scale);                  // the global scale

    for (uint32_t item = warp; item < n_items; item += n_warps) {
        const uint32_t pos = item / g.groups_per_token;
        const uint32_t grp = item - pos * g.groups_per_token;
        const uint32_t tok = g.perm ? __ldg(g.perm + pos) : pos;
        const uint32_t my_row = warp_head_row(g, tok, lane, H, seed);
        uint32_t rows[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) rows[h] = __shfl_sync(0xFFFFFFFFu, my_row, h);
        const uint32_t s_begin = grp * g.strips_per_item;
        const uint32_t s_end = min(s_begin + g.strips_per_item, g.n_strips);
        const size_t tok_off = static_cast<size_t>(tok) * g.d;
        for (uint32_t s = s_begin; s < s_end; ++s) {
            const uint32_t v = s * 32u + lane;
            if (v >= nvec) continue;                      // the last strip may be ragged
            // issue every load of this block before the first multiply-add
            uint2 e[16];
            uint32_t bs[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                if (kH || h < static_cast<int>(H)) {
                    const uint8_t *row = table + static_cast<size_t>(rows[h]) * rb;
                    e[h] = ld_stream_v2(row + v * 8u);
                    bs[h] = ld_stream_u8(row + code_bytes + v);
                }
            }
            const uint4 r0 = ld_na_v4(g.residual + tok_off + v * 16u);
            const uint4 r1 = ld_na_v4(g.residual + tok_off + v * 16u + 8u);

            float2 acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = make_float2(0.0f, 0.0f);
            // the block scales of heads 2k and 2k+1 converted together (one f16 pair)
#pragma unroll
            for (int h = 0; h < 16; h += 2) {
                if (kH || h < static_cast<int>(H)) {
                    const bool two = kH || h + 1 < static_cast<int>(H);
                    const uint32_t s2 = e4m3x2_to_half2_bits(bs[h], two ? bs[h + 1] : 0u);
                    e2m1x8_fma<false>(e[h].x, s2, acc);
                    e2m1x8_fma<false>(e[h].y, s2, acc + 4);
                    if (two) {
                        e2m1x8_fma<true>(e[h + 1].x, s2, acc);
                        e2m1x8_fma<true>(e[h + 1].y, s2, acc + 4);
                    }
                }
            }
            const float2 g2 = make_float2(gs, gs);       // the global scale, once per sum
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = mul2(acc[k], g2);
            store_gated16<kTokGate>(g, tok_off, v, r0, r1, acc);
        }
    }
}

}  // namespace ngram
