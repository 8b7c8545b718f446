// fill.cuh -- synthetic table initialisation (set-up, not on the timed path).
//
// The pages' table is learned ("Qwen Brought Back N-Grams. All 51 Billion
// Parameters of Them.", section "N-grams, of all things"); no weights exist here, so
// element (row, col) is a pure function of (seed, row, col) through Philox4x32-10.
// The exact mapping is stated in include/ngram.h (ngram_fill_synthetic).
#pragma once

#include "device_common.cuh"

namespace ngram {

constexpr float kBf16Scale = 0x1.1bc77ap-22f;   // 0.02 / std(2S - 262140)
constexpr float kInt8Scale = 0x1.1bc5f4p-11f;   // 0.02 / std(q)
constexpr float kFp8Scale = 0x1.4dp-8f;         // ~0.02 / std of the E4M3 values below
constexpr float kFp4GlobalScale = 0x1.4fp-9f;   // ~0.02 / std of E2M1 x block scale

// bf16 value from the two Philox words (a, b) of its column parity.
__device__ __forceinline__ float synth_bf16_value(uint32_t a, uint32_t b) {
    const int32_t S = static_cast<int32_t>((a & 0xFFFFu) + (a >> 16) + (b & 0xFFFFu) + (b >> 16));
    const int32_t C = 2 * S - 262140;                     // |C| < 2^24: exact in fp32
    return __fmul_rn(__int2float_rn(C), kBf16Scale);
}

// int8 value from one Philox word: (sum of its bytes - 510) >> 2, arithmetic shift.
__device__ __forceinline__ int32_t synth_int8_value(uint32_t w) {
    const int32_t sum = static_cast<int32_t>((w & 0xFFu) + ((w >> 8) & 0xFFu) +
                                             ((w >> 16) & 0xFFu) + (w >> 24));
    return (sum - 510) >> 2;
}

// Every fill writes columns col0 .. col0 + d - 1 of the synthetic table (col0 = 0: the
// whole table; else a column shard of a wider one), the values of those columns being the
// same whatever the table's full width.
//
// One CTA per row (grid-stride over rows); each thread writes 8 columns (16 bytes)
// per step, from four Philox calls with counters (col/2, row, 1, 0).
__global__ void __launch_bounds__(256) k_fill_bf16(uint16_t *__restrict__ table, uint64_t R,
                                                   uint32_t d, uint32_t col0, uint32_t k0, uint32_t k1) {
    const uint32_t nvec = d >> 3;
    for (uint64_t row = blockIdx.x; row < R; row += gridDim.x) {
        uint4 *dst = reinterpret_cast<uint4 *>(table + row * d);
        for (uint32_t v = threadIdx.x; v < nvec; v += blockDim.x) {
            uint32_t words[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {                // column pair 4v+p: cols 8v+2p, +1
                const uint4 x = philox4x32_10(
                    make_uint4((col0 >> 1) + 4u * v + p, static_cast<uint32_t>(row), 1u, 0u), k0, k1);
                words[p] = pack_bf16x2(synth_bf16_value(x.x, x.y), synth_bf16_value(x.z, x.w));
            }
            dst[v] = make_uint4(words[0], words[1], words[2], words[3]);
        }
    }
}

// int8 rows: each thread writes 16 columns from four Philox calls with counters
// (col/4, row, 2, 0); thread 0 of the row also writes the row scale (counter
// (0, row, 3, 0)).
__global__ void __launch_bounds__(256) k_fill_int8(int8_t *__restrict__ table,
                                                   float *__restrict__ row_scale, uint64_t R,
                                                   uint32_t d, uint32_t col0, uint32_t k0, uint32_t k1) {
    const uint32_t nvec = d >> 4;
    for (uint64_t row = blockIdx.x; row < R; row += gridDim.x) {
        uint4 *dst = reinterpret_cast<uint4 *>(table + row * d);
        for (uint32_t v = threadIdx.x; v < nvec; v += blockDim.x) {
            uint32_t words[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {                // columns 16v+4p .. 16v+4p+3
                const uint4 x = philox4x32_10(
                    make_uint4((col0 >> 2) + 4u * v + p, static_cast<uint32_t>(row), 2u, 0u), k0, k1);
                const uint32_t q0 = synth_int8_value(x.x) & 0xFFu;
                const uint32_t q1 = synth_int8_value(x.y) & 0xFFu;
                const uint32_t q2 = synth_int8_value(x.z) & 0xFFu;
                const uint32_t q3 = synth_int8_value(x.w) & 0xFFu;
                words[p] = q0 | (q1 << 8) | (q2 << 16) | (q3 << 24);
            }
            dst[v] = make_uint4(words[0], words[1], words[2], words[3]);
        }
        if (threadIdx.x == 0) {
            const uint4 x = philox4x32_10(make_uint4(0u, static_cast<uint32_t>(row), 3u, 0u), k0, k1);
            const float t = __fmul_rn(__uint2float_rn(x.x >> 8), 0x1p-25f);
            row_scale[row] = __fmul_rn(kInt8Scale, __fadd_rn(0.75f, t));
        }
    }
}

// FP8 E4M3 code from one Philox word: sign bit 31, exponent field 4 + bits[3:4] +
// bits[5:6] (4..10: finite, never NaN), mantissa bits[0:2].
__device__ __forceinline__ uint32_t synth_e4m3(uint32_t w) {
    const uint32_t e = 4u + ((w >> 3) & 3u) + ((w >> 5) & 3u);
    return ((w >> 31) << 7) | (e << 3) | (w & 7u);
}

// NVFP4 block scale (E4M3) from one Philox word: positive, exponent field 5 + bits[0:1]
// + bit[2] (5..9), mantissa bits[3:5].
__device__ __forceinline__ uint32_t synth_fp4_block_scale(uint32_t w) {
    const uint32_t e = 5u + (w & 3u) + ((w >> 2) & 1u);
    return (e << 3) | ((w >> 3) & 7u);
}

// FP8 rows: each thread writes 16 codes from four Philox calls with counters
// (col/4, row, 4, 0), byte k of a word from word k; thread 0 of the row also writes the
// row scale from counter (0, row, 5, 0).
__global__ void __launch_bounds__(256) k_fill_fp8(uint8_t *__restrict__ table,
                                                  float *__restrict__ row_scale, uint64_t R,
                                                  uint32_t d, uint32_t col0, uint32_t k0, uint32_t k1) {
    const uint32_t nvec = d >> 4;
    for (uint64_t row = blockIdx.x; row < R; row += gridDim.x) {
        uint4 *dst = reinterpret_cast<uint4 *>(table + row * d);
        for (uint32_t v = threadIdx.x; v < nvec; v += blockDim.x) {
            uint32_t words[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {                // columns 16v+4p .. 16v+4p+3
                const uint4 x = philox4x32_10(
                    make_uint4((col0 >> 2) + 4u * v + p, static_cast<uint32_t>(row), 4u, 0u), k0, k1);
                words[p] = synth_e4m3(x.x) | (synth_e4m3(x.y) << 8) | (synth_e4m3(x.z) << 16) |
                           (synth_e4m3(x.w) << 24);
            }
            dst[v] = make_uint4(words[0], words[1], words[2], words[3]);
        }
        if (threadIdx.x == 0) {
            const uint4 x = philox4x32_10(make_uint4(0u, static_cast<uint32_t>(row), 5u, 0u), k0, k1);
            const float t = __fmul_rn(__uint2float_rn(x.x >> 8), 0x1p-25f);
            row_scale[row] = __fmul_rn(kFp8Scale, __fadd_rn(0.75f, t));
        }
    }
}

// NVFP4 rows of rb = d/2 + ceil16(d/16) bytes: the d/2 code bytes (column 2j in the low
// nibble of byte j), then one E4M3 scale byte per 16 columns, zero-padded to 16 bytes.
// Codes of columns 32k .. 32k+31 are the 16 bytes of Philox (k, row, 6, 0) in order (nibble
// c%8 of word (c/8)%4 is column c); the scale of block b comes from word b%4 of Philox
// (b/4, row, 7, 0).  The global scale is written to gscale[0] by the first CTA.  With a
// column offset col0 (a multiple of 32), code vector v is counter col0/32 + v and local
// block b is global block col0/16 + b.
__global__ void __launch_bounds__(256) k_fill_fp4(uint8_t *__restrict__ table,
                                                  float *__restrict__ gscale, uint64_t R,
                                                  uint32_t d, uint32_t col0, uint32_t k0, uint32_t k1) {
    const uint32_t n_blocks = d >> 4;
    const uint32_t code_vec = d >> 5;
    const uint32_t scale_vec = (n_blocks + 15u) >> 4;
    const uint64_t rb = (d >> 1) + 16ull * scale_vec;
    if (blockIdx.x == 0 && threadIdx.x == 0) gscale[0] = kFp4GlobalScale;
    for (uint64_t row = blockIdx.x; row < R; row += gridDim.x) {
        uint4 *dst = reinterpret_cast<uint4 *>(table + row * rb);
        for (uint32_t v = threadIdx.x; v < code_vec + scale_vec; v += blockDim.x) {
            if (v < code_vec) {
                dst[v] = philox4x32_10(make_uint4((col0 >> 5) + v, static_cast<uint32_t>(row), 6u, 0u),
                                       k0, k1);
                continue;
            }
            const uint32_t sv = v - code_vec;            // local blocks 16sv .. 16sv+15
            uint32_t words[4] = {0u, 0u, 0u, 0u};
            uint32_t ctr = 0xFFFFFFFFu;
            uint4 x = make_uint4(0u, 0u, 0u, 0u);
            for (uint32_t j = 0; j < 16u && 16u * sv + j < n_blocks; ++j) {
                const uint32_t B = (col0 >> 4) + 16u * sv + j;   // global block
                if ((B >> 2) != ctr) {
                    ctr = B >> 2;
                    x = philox4x32_10(make_uint4(ctr, static_cast<uint32_t>(row), 7u, 0u), k0, k1);
                }
                const uint32_t k = B & 3u;
                const uint32_t w = k == 0u ? x.x : k == 1u ? x.y : k == 2u ? x.z : x.w;
                const uint32_t byte = synth_fp4_block_scale(w) << (8u * (j & 3u));
                if (j < 4u) words[0] |= byte;
                else if (j < 8u) words[1] |= byte;
                else if (j < 12u) words[2] |= byte;
                else words[3] |= byte;
            }
            dst[v] = make_uint4(words[0], words[1], words[2], words[3]);
        }
    }
}

}  // namespace ngram
