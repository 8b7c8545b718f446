// gather_c8.cuh -- the fused gather with 8 columns per lane, for any row format of
// rows.cuh (same operation and arithmetic as k_gather_bf16 / k_gather_int8 /
// k_gather_fp8 / k_gather_nvfp4, so the same bits).
//
// A lane holds one 8-column fragment per head in flight (16 B of bf16, 8 B of int8 / FP8,
// 4 B of E2M1 codes + a block-scale byte), half of what the 16-column gathers of the 8- and
// 4-bit formats hold, so a CTA needs fewer registers and more CTAs fit on an SM.  Over a
// whole table the 16-column gathers measured faster on B200 (the 8-bit and 4-bit decode
// wants the longer fragment); this kernel serves the column-sharded table, where one
// layout for every format keeps the shard widths simple.
//
// kShard: the table holds a column shard (columns col0 .. col0 + d - 1 of a wider table, as
// the per-rank shards of the SGLang TP4 setup on "Qwen Brought Back N-Grams. All 51 Billion
// Parameters of Them.", section "Which is why the offload matters more than the parameter
// count").  The residual and the outputs are full rows of g.ld elements; the kernel
// computes the shard's columns and stores them into every buffer of g.outs -- this GPU's
// output and, through peer mappings, the other ranks' -- so the gather and the all-gather
// of the output are one kernel.
#pragma once

#include "rows.cuh"

namespace ngram {

#ifndef NGRAM_C8_MIN_BLOCKS           // resident CTAs per SM the register budget targets
#define NGRAM_C8_MIN_BLOCKS 3
#endif

template <int kH, class Rows, bool kTokGate, bool kShard = false>
__global__ void __launch_bounds__(256, NGRAM_C8_MIN_BLOCKS) k_gather_c8(const GatherArgs g,
                                                                        uint32_t row_bytes) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t nvec = g.d >> 3;
    const uint32_t n_items = g.N * g.groups_per_token;
    const uint8_t *__restrict__ table = static_cast<const uint8_t *>(g.table);
    const float gs = (g.row_scale != nullptr && !Rows::kRowScale) ? __ldg(g.row_scale) : 0.0f;

    for (uint32_t item = warp; item < n_items; item += n_warps) {
        const uint32_t pos = item / g.groups_per_token;
        const uint32_t grp = item - pos * g.groups_per_token;
        const uint32_t tok = g.perm ? __ldg(g.perm + pos) : pos;
        const uint32_t my_row = warp_head_row(g, tok, lane, H);
        const float my_scale = (Rows::kRowScale && lane < H) ? __ldg(g.row_scale + my_row) : 0.0f;
        uint32_t rows[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) rows[h] = __shfl_sync(0xFFFFFFFFu, my_row, h);
        const uint32_t s_begin = grp * g.strips_per_item;
        const uint32_t s_end = min(s_begin + g.strips_per_item, g.n_strips);
        const size_t tok_off = static_cast<size_t>(tok) * (kShard ? g.ld : g.d);
        for (uint32_t s = s_begin; s < s_end; ++s) {
            const uint32_t v = s * 32u + lane;
            const bool active = v < nvec;
            typename Rows::Frag f[16];
            if (active) {
#pragma unroll
                for (int h = 0; h < 16; ++h)
                    if (kH || h < static_cast<int>(H))
                        f[h] = Rows::load(table + static_cast<size_t>(rows[h]) * row_bytes, v, g.d);
            }
            float sc[16];
#pragma unroll
            for (int h = 0; h < 16; ++h)
                sc[h] = Rows::kRowScale ? __shfl_sync(0xFFFFFFFFu, my_scale, h) : 0.0f;
            if (!active) continue;
            const uint4 r = ld_na_v4(g.residual + tok_off + v * 8u);
            float2 acc[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int h = 0; h < 16; ++h)
                if (kH || h < static_cast<int>(H)) Rows::add(acc, f[h], sc[h], gs);
            Rows::finish(acc, gs);
            float gv[8];
            load_gate8<kTokGate>(g, tok_off, v, gv);
            // y = r + (g * acc): the product is rounded on its own (scalar, never fused)
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
            uint32_t o[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float y0 = __fadd_rn(bf16_lo(rw[p]), __fmul_rn(gv[2 * p], acc[p].x));
                const float y1 = __fadd_rn(bf16_hi(rw[p]), __fmul_rn(gv[2 * p + 1], acc[p].y));
                o[p] = pack_bf16x2(y0, y1);
            }
            const uint4 ov = make_uint4(o[0], o[1], o[2], o[3]);
            if (kShard) {
                for (uint32_t p = 0; p < g.n_outs; ++p)
                    *reinterpret_cast<uint4 *>(g.outs[p] + tok_off + v * 8u) = ov;
            } else {
                *reinterpret_cast<uint4 *>(g.out + tok_off + v * 8u) = ov;
            }
        }
    }
}

}  // namespace ngram
