// rows.cuh -- the row formats as policies over 8 columns of one row: load the bytes of
// columns 8v .. 8v+7, and add their values to fp32 accumulators in head order.
//
// Each policy decodes and accumulates exactly as the format's own gather does (bf16:
// acc = acc + v; int8 / FP8: acc = fma(q, s_row, acc); NVFP4: acc = fma(q, block scale,
// acc), then finish() multiplies the sum by the global scale once), so every kernel built
// on them -- add() for each head in order, then finish() -- computes the head sum bit for
// bit as the forward does.  Formats: "Qwen Brought Back N-Grams. All
// 51 Billion Parameters of Them." (bf16 table, section "N-grams, of all things");
// "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with Heterogeneous Memory Prefetch"
// (INT8, Key point 3; FP4, architecture figure); "Qwen3.8-Flash-Next: A 125B MoE for the
// Local Stack?" (FP8 and 4-bit, section "Hardware math for self-hosting").
#pragma once

#include "gather_int8.cuh"

namespace ngram {

__device__ __forceinline__ uint32_t ld_stream_u32(const void *p) {
    uint32_t r;
    asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

// ---------------------------------------------------------------- row formats, 8 columns
struct RowsBf16 {
    static constexpr bool kRowScale = false;
    typedef uint4 Frag;
    static __device__ __forceinline__ Frag load(const uint8_t *row, uint32_t v, uint32_t /*d*/) {
        return ld_stream_v4(row + v * 16u);
    }
    static __device__ __forceinline__ Frag load_smem(const uint8_t *row, uint32_t v, uint32_t) {
        return *reinterpret_cast<const uint4 *>(row + v * 16u);
    }
    static __device__ __forceinline__ void add(float2 (&acc)[4], const Frag &f, float, float) {
        acc[0] = add2(acc[0], bf16x2(f.x));
        acc[1] = add2(acc[1], bf16x2(f.y));
        acc[2] = add2(acc[2], bf16x2(f.z));
        acc[3] = add2(acc[3], bf16x2(f.w));
    }
    static __device__ __forceinline__ void finish(float2 (&)[4], float) {}
};

template <class Codes>
struct Rows8bit {                       // int8 / FP8 E4M3 codes with a per-row scale
    static constexpr bool kRowScale = true;
    typedef uint2 Frag;
    static __device__ __forceinline__ Frag load(const uint8_t *row, uint32_t v, uint32_t) {
        return ld_stream_v2(row + v * 8u);
    }
    static __device__ __forceinline__ Frag load_smem(const uint8_t *row, uint32_t v, uint32_t) {
        return *reinterpret_cast<const uint2 *>(row + v * 8u);
    }
    static __device__ __forceinline__ void add(float2 (&acc)[4], const Frag &f, float s, float) {
        const float2 s2 = make_float2(s, s);
        float2 lo, hi;
        Codes::decode(f.x, lo, hi);
        acc[0] = fma2(lo, s2, acc[0]);
        acc[1] = fma2(hi, s2, acc[1]);
        Codes::decode(f.y, lo, hi);
        acc[2] = fma2(lo, s2, acc[2]);
        acc[3] = fma2(hi, s2, acc[3]);
    }
    static __device__ __forceinline__ void finish(float2 (&)[4], float) {}
};

struct RowsNvfp4 {                      // E2M1 codes, E4M3 block scale, global scale gs
    static constexpr bool kRowScale = false;
    struct Frag {
        uint32_t codes, bs;
    };
    static __device__ __forceinline__ Frag load(const uint8_t *row, uint32_t v, uint32_t d) {
        return Frag{ld_stream_u32(row + v * 4u), ld_stream_u8(row + (d >> 1) + (v >> 1))};
    }
    static __device__ __forceinline__ Frag load_smem(const uint8_t *row, uint32_t v, uint32_t d) {
        return Frag{*reinterpret_cast<const uint32_t *>(row + v * 4u), row[(d >> 1) + (v >> 1)]};
    }
    static __device__ __forceinline__ void add(float2 (&acc)[4], const Frag &f, float, float) {
        e2m1x8_fma(f.codes, e4m3_to_half_bits(f.bs), acc);      // acc += q * bs, one rounding
    }
    static __device__ __forceinline__ void finish(float2 (&acc)[4], float gs) {
        const float2 g2 = make_float2(gs, gs);                    // the global scale, once
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = mul2(acc[k], g2);
    }
};

}  // namespace ngram
