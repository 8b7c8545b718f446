// gather_int8.cuh -- the gather for 8-bit rows with one fp32 scale per row: int8, and FP8
// E4M3.
//
// Same operation as k_gather_bf16 ("Qwen Brought Back N-Grams. All 51 Billion
// Parameters of Them.", section "N-grams, of all things": hash, gather 16 rows, sum,
// add to the residual through the gate of "Qwen3.8-Flash-Next: A 51B N-gram Embedding
// Table with Heterogeneous Memory Prefetch", Key point 1) for the INT8 table that
// page's Key point 3 sizes at ~51 GB, and for FP8 rows ("Qwen3.8-Flash-Next: A 125B MoE
// for the Local Stack?", section "Hardware math for self-hosting", weighs FP8 and 4-bit
// n-gram tables): every row value is q * scale[row], q the code's exact value.
#pragma once

#include "gather.cuh"

namespace ngram {

// Row decoders: the four codes of one 32-bit word (byte k = column k) -> exact fp32
// columns (0, 1) and (2, 3).
struct Int8Codes {
    // The sign bit of each byte is flipped (q + 128 in [0, 255]), one byte permute places
    // the byte in the mantissa of 2^23 (the float 2^23 + 128 + q), and 2^23 + 128 is
    // subtracted; every step is exact.
    static __device__ __forceinline__ void decode(uint32_t w, float2 &c01, float2 &c23) {
        const uint32_t u = w ^ 0x80808080u;
        const float2 bias = make_float2(8388736.0f, 8388736.0f);       // 2^23 + 128
        c01 = sub2(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540u)),
                               __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541u))), bias);
        c23 = sub2(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542u)),
                               __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543u))), bias);
    }
};

struct E4m3Codes {
    static __device__ __forceinline__ void decode(uint32_t w, float2 &c01, float2 &c23) {
        e4m3x4_to_float(w, c01, c23);
    }
};

// y = r + (g * acc) for columns 16v .. 16v+15 of one token (residual words r0, r1 loaded
// before the sum); the product is rounded on its own (scalar, never fused).
template <bool kTokGate>
__device__ __forceinline__ void store_gated16(const GatherArgs &g, size_t tok_off, uint32_t v,
                                              const uint4 &r0, const uint4 &r1, const float2 acc[8]) {
    float gv[16];
    load_gate8<kTokGate>(g, tok_off, 2u * v, gv);
    load_gate8<kTokGate>(g, tok_off, 2u * v + 1u, gv + 8);
    const uint32_t rw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    uint32_t o[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const float y0 = __fadd_rn(bf16_lo(rw[p]), __fmul_rn(gv[2 * p], acc[p].x));
        const float y1 = __fadd_rn(bf16_hi(rw[p]), __fmul_rn(gv[2 * p + 1], acc[p].y));
        o[p] = pack_bf16x2(y0, y1);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(g.out + tok_off + v * 16u);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// 8-bit rows with one fp32 scale per row: value = q * scale[row].  A lane owns 16
// columns (one 16-byte vector of the row); the per-row scales are loaded once per token
// by the hashing lanes and broadcast with the row indices.  Sum per head in order with
// one fused multiply-add per head, acc = fma(q, s, acc) (one rounding per head), then
// the same bf16 epilogue as the bf16 rows.
template <int kH, class Codes, bool kTokGate>
__device__ __forceinline__ void gather_rowscale(const GatherArgs &g) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t nvec = g.d >> 4;
    const uint32_t n_items = g.N * g.groups_per_token;
    const uint8_t *__restrict__ table = static_cast<const uint8_t *>(g.table);
    const uint64_t seed = head_seed(lane, g.h);           // arithmetic only: before the wait
    if (g.trigger_early) allow_dependents();
    grid_dependency_wait();

    for (uint32_t item = warp; item < n_items; item += n_warps) {
        const uint32_t pos = item / g.groups_per_token;
        const uint32_t grp = item - pos * g.groups_per_token;
        const uint32_t tok = g.perm ? __ldg(g.perm + pos) : pos;
        const uint32_t my_row = warp_head_row(g, tok, lane, H, seed);
        // the scale load is issued here but first used after the row loads are in flight
        const float my_scale = (lane < H) ? __ldg(g.row_scale + my_row) : 0.0f;
        uint32_t rows[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) rows[h] = __shfl_sync(0xFFFFFFFFu, my_row, h);
        const uint32_t s_begin = grp * g.strips_per_item;
        const uint32_t s_end = min(s_begin + g.strips_per_item, g.n_strips);
        const size_t tok_off = static_cast<size_t>(tok) * g.d;
        for (uint32_t s = s_begin; s < s_end; ++s) {
            const uint32_t v = s * 32u + lane;
            const bool active = v < nvec;             // the last strip may be ragged
            uint4 e[16];
            if (active) {
#pragma unroll
                for (int h = 0; h < 16; ++h)
                    if (kH || h < static_cast<int>(H))
                        e[h] = ld_stream_v4(table + static_cast<size_t>(rows[h]) * g.d + v * 16u);
            }
            // every lane takes part in the shuffles, after the row loads are issued
            float sc[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) sc[h] = __shfl_sync(0xFFFFFFFFu, my_scale, h);
            if (!active) continue;
            const uint4 r0 = ld_na_v4(g.residual + tok_off + v * 16u);
            const uint4 r1 = ld_na_v4(g.residual + tok_off + v * 16u + 8u);

            // acc[k] holds columns (2k, 2k+1); per head, acc = fma(q, s, acc) on both lanes
            float2 acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                if (kH || h < static_cast<int>(H)) {
                    const uint32_t wv[4] = {e[h].x, e[h].y, e[h].z, e[h].w};
                    const float2 s2 = make_float2(sc[h], sc[h]);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float2 lo, hi;
                        Codes::decode(wv[k], lo, hi);
                        acc[2 * k] = fma2(lo, s2, acc[2 * k]);
                        acc[2 * k + 1] = fma2(hi, s2, acc[2 * k + 1]);
                    }
                }
            }
            store_gated16<kTokGate>(g, tok_off, v, r0, r1, acc);
        }
    }
}

template <int kH, bool kTokGate = false>
__global__ void __launch_bounds__(256, 2) k_gather_int8(const GatherArgs g) {
    gather_rowscale<kH, Int8Codes, kTokGate>(g);
}

template <int kH, bool kTokGate = false>
__global__ void __launch_bounds__(256, 2) k_gather_fp8(const GatherArgs g) {
    gather_rowscale<kH, E4m3Codes, kTokGate>(g);
}

}  // namespace ngram
