// gather_int8.cuh -- the gather for int8 rows with one fp32 scale per row.
//
// Same operation as k_gather_bf16 ("Qwen Brought Back N-Grams. All 51 Billion
// Parameters of Them.", section "N-grams, of all things": hash, gather 16 rows, sum,
// add to the residual through the gate of "Qwen3.8-Flash-Next: A 51B N-gram Embedding
// Table with Heterogeneous Memory Prefetch", Key point 1) for the INT8 table that
// page's Key point 3 sizes at ~51 GB: every row value is q * scale[row].
#pragma once

#include "gather.cuh"

namespace ngram {

// int8 byte j (0..3) of word w -> exact fp32 value.  The sign bit is flipped (q + 128
// in [0, 255]), the byte is placed in the mantissa of 2^23 with one byte permute, and
// 2^23 + 128 is subtracted; every step is exact.
__device__ __forceinline__ float int8_at(uint32_t biased, uint32_t j) {
    return __fsub_rn(__uint_as_float(__byte_perm(biased, 0x4B000000u, 0x7540u + j)), 8388736.0f);
}

// int8 rows with one fp32 scale per row: value = q * scale[row].  A lane owns 16
// columns (one 16-byte vector of the row); the per-row scales are loaded once per token
// by the hashing lanes and broadcast with the row indices.  Sum per head in order:
// acc = acc + (q * s), each step rounded separately, then the same bf16 epilogue.
template <int kH>
__global__ void __launch_bounds__(256, 2) k_gather_int8(const GatherArgs g) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t nvec = g.d >> 4;
    const uint32_t n_items = g.N * g.groups_per_token;
    const int8_t *__restrict__ table = static_cast<const int8_t *>(g.table);

    for (uint32_t item = warp; item < n_items; item += n_warps) {
        const uint32_t tok = item / g.groups_per_token;
        const uint32_t grp = item - tok * g.groups_per_token;
        const uint32_t my_row = warp_head_row(g, tok, lane, H);
        const float my_scale = (lane < H) ? __ldg(g.row_scale + my_row) : 0.0f;
        uint32_t rows[16];
        float sc[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            rows[h] = __shfl_sync(0xFFFFFFFFu, my_row, h);
            sc[h] = __shfl_sync(0xFFFFFFFFu, my_scale, h);
        }
        const uint32_t s_begin = grp * g.strips_per_item;
        const uint32_t s_end = min(s_begin + g.strips_per_item, g.n_strips);
        const size_t tok_off = static_cast<size_t>(tok) * g.d;
        for (uint32_t s = s_begin; s < s_end; ++s) {
            const uint32_t v = s * 32u + lane;
            if (v >= nvec) continue;
            uint4 e[16];
#pragma unroll
            for (int h = 0; h < 16; ++h)
                if (kH || h < static_cast<int>(H))
                    e[h] = ld_stream_v4(table + static_cast<size_t>(rows[h]) * g.d + v * 16u);
            const uint4 r0 = ld_na_v4(g.residual + tok_off + v * 16u);
            const uint4 r1 = ld_na_v4(g.residual + tok_off + v * 16u + 8u);

            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                if (kH || h < static_cast<int>(H)) {
                    const uint32_t wv[4] = {e[h].x ^ 0x80808080u, e[h].y ^ 0x80808080u,
                                            e[h].z ^ 0x80808080u, e[h].w ^ 0x80808080u};
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            acc[4 * k + j] = __fadd_rn(acc[4 * k + j],
                                                       __fmul_rn(int8_at(wv[k], j), sc[h]));
                }
            }
            const float4 *gp = reinterpret_cast<const float4 *>(g.gate) + 4u * v;
            const float4 g0 = __ldg(gp), g1 = __ldg(gp + 1), g2 = __ldg(gp + 2), g3 = __ldg(gp + 3);
            const float gv[16] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w,
                                  g2.x, g2.y, g2.z, g2.w, g3.x, g3.y, g3.z, g3.w};
            const uint32_t rw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            uint32_t o[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const float y0 = __fadd_rn(bf16_lo(rw[p]), __fmul_rn(gv[2 * p], acc[2 * p]));
                const float y1 = __fadd_rn(bf16_hi(rw[p]), __fmul_rn(gv[2 * p + 1], acc[2 * p + 1]));
                o[p] = pack_bf16x2(y0, y1);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(g.out + tok_off + v * 16u);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
    }
}

}  // namespace ngram
