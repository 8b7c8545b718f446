// device_common.cuh -- device helpers of libngram: context formation, the per-head
// hash, exact remainder by R, Philox4x32-10 and cache-hinted vector loads.
//
// The method ("Qwen Brought Back N-Grams. All 51 Billion Parameters of Them.",
// section "N-grams, of all things"): hash the bigram and trigram context of each
// token into one table, gather 16 rows.  The pages fix no hash; the one defined
// here is documented in include/ngram.h.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace ngram {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;   // splitmix64 state increment
constexpr uint32_t kTokenMask = (1u << 21) - 1u;

// splitmix64 output for the state reached by one increment from z (Steele, Lea &
// Flood, OOPSLA 2014): the mixer with the published constants.
__host__ __device__ __forceinline__ uint64_t splitmix64_step(uint64_t z) {
    z += kGolden;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// x mod R for R >= 2 with the Barrett constant m = floor(2^64 / R) (Barrett, CRYPTO
// '86).  q = floor(x * m / 2^64) is floor(x / R) or one less, so one conditional
// subtraction gives the exact remainder.  R == 1 is handled by the caller (m = 0).
__device__ __forceinline__ uint32_t mod_rows(uint64_t x, uint64_t R, uint64_t m) {
    if (m == 0) return 0u;                       // R == 1
    uint64_t q = __umul64hi(x, m);
    uint64_t r = x - q * R;
    if (r >= R) r -= R;
    return static_cast<uint32_t>(r);
}

// Parameters of the hash, passed by value to every kernel that hashes.
struct HashArgs {
    uint64_t base_seed;
    uint64_t R;
    uint64_t barrett_m;       // floor(2^64 / R), 0 when R == 1
    uint32_t n_bigram;
    uint32_t n_heads;         // bigram + trigram, <= 16
    uint32_t pad_id;
    uint32_t vocab;
};

// Device error word: [0] flag, [1] position (bit 31 = history entry), [2] bad id.
__device__ __forceinline__ void flag_bad_token(uint32_t *err, uint32_t pos, int32_t id) {
    if (atomicCAS(err, 0u, 1u) == 0u) {
        err[1] = pos;
        err[2] = static_cast<uint32_t>(id);
    }
}

__device__ __forceinline__ uint32_t checked_token(int32_t w, const HashArgs &a,
                                                  uint32_t *err, uint32_t pos) {
    if (w < 0 || static_cast<uint32_t>(w) >= a.vocab) {
        flag_bad_token(err, pos, w);
        return a.pad_id;
    }
    return static_cast<uint32_t>(w);
}

// w0 = w_t, w1 = w_{t-1}, w2 = w_{t-2} of flat token `tok` (= s * T + t); earlier
// positions come from history[s] = {w_-2, w_-1} or PAD.  Never crosses sequences.
__device__ __forceinline__ void token_context(const int32_t *__restrict__ tokens,
                                              const int32_t *__restrict__ history,
                                              uint32_t tok, uint32_t T, const HashArgs &a,
                                              uint32_t *err, uint32_t &w0, uint32_t &w1,
                                              uint32_t &w2) {
    const uint32_t s = tok / T;
    const uint32_t t = tok - s * T;
    w0 = checked_token(__ldg(tokens + tok), a, err, tok);
    uint32_t h_old = a.pad_id, h_new = a.pad_id;
    if (history != nullptr && t < 2) {
        h_new = checked_token(__ldg(history + 2 * s + 1), a, err, 0x80000000u | (2 * s + 1));
        if (t == 0)
            h_old = checked_token(__ldg(history + 2 * s), a, err, 0x80000000u | (2 * s));
    }
    w1 = (t >= 1) ? checked_token(__ldg(tokens + tok - 1), a, err, tok - 1) : h_new;
    w2 = (t >= 2) ? checked_token(__ldg(tokens + tok - 2), a, err, tok - 2)
                  : ((t == 1) ? h_new : h_old);
}

// seed_h = (h+1)-th splitmix64 output from base_seed.
__device__ __forceinline__ uint64_t head_seed(uint32_t h, const HashArgs &a) {
    return splitmix64_step(a.base_seed + static_cast<uint64_t>(h) * kGolden);
}

// Row index of head h for context (w0, w1, w2), given seed = head_seed(h).
__device__ __forceinline__ uint32_t head_row_seeded(uint32_t h, uint64_t seed, uint32_t w0, uint32_t w1,
                                                    uint32_t w2, const HashArgs &a) {
    const uint64_t k2 = (static_cast<uint64_t>(w1) << 21) | w0;
    const uint64_t key = (h < a.n_bigram) ? k2 : ((static_cast<uint64_t>(w2) << 42) | k2);
    return mod_rows(splitmix64_step(key ^ seed), a.R, a.barrett_m);
}

// Row index of head h for context (w0, w1, w2).
__device__ __forceinline__ uint32_t head_row(uint32_t h, uint32_t w0, uint32_t w1,
                                             uint32_t w2, const HashArgs &a) {
    return head_row_seeded(h, head_seed(h, a), w0, w1, w2, a);
}

// Programmatic dependent launch (sm_90+).  A kernel launched with programmatic stream
// serialization may start while the previous kernel of its stream is still running;
// grid_dependency_wait() returns once every prerequisite grid has completed and its
// memory operations are visible, so a kernel calls it before its first global memory
// access and keeps plain stream-order semantics.  allow_dependents() lets the next such
// kernel of the stream be scheduled early (it waits the same way before touching memory).
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Philox4x32-10 (Salmon, Moraes, Dror & Shaw, SC'11): ten rounds of two 32x32->64
// multiplies on words 0 and 2, key bumped by the Weyl constants between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int i = 0; i < 10; ++i) {
        const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// 16-byte read-only load that does not allocate in L1 (rows and residual are read
// once per use; reuse across tokens is left to L2).  NGRAM_ROW_LOAD_HINT = 1 (default)
// adds an L2 256-byte prefetch hint, measured ~0.3% faster on the full-size gather.
#ifndef NGRAM_ROW_LOAD_HINT
#define NGRAM_ROW_LOAD_HINT 1
#endif
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
#if NGRAM_ROW_LOAD_HINT == 1
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
#else
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
#endif
    return r;
}

// 8-byte and 1-byte forms of the same load (the NVFP4 rows: 8 code bytes and one block
// scale per 16 columns).
__device__ __forceinline__ uint2 ld_stream_v2(const void *p) {
    uint2 r;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v2.u32 {%0, %1}, [%2];"
        : "=r"(r.x), "=r"(r.y)
        : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_stream_u8(const void *p) {
    uint32_t r;
    asm("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

// Packed fp32 pairs (sm_100 add/sub/mul/fma .f32x2): two independent IEEE fp32
// operations, each rounded to nearest even exactly as the scalar __fadd_rn / __fsub_rn /
// __fmul_rn / __fmaf_rn, in one instruction.  A packed product whose only use is a packed
// add may be fused with it into one rounding, so wherever the definition rounds a product
// on its own the code uses the scalar __fmul_rn / __fadd_rn, and where it fuses it says
// so with fma2.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rr;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rr, ra, rb;\n\tmov.b64 {%0, %1}, rr;\n\t}"
        : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rr;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rr, ra, rb;\n\tmov.b64 {%0, %1}, rr;\n\t}"
        : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rr;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rr, ra, rb;\n\tmov.b64 {%0, %1}, rr;\n\t}"
        : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {     // a * b + c
    float2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rr;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rr, ra, rb, rc;\n\tmov.b64 {%0, %1}, rr;\n\t}"
        : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

// bf16 pair in one 32-bit word -> two fp32 values (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float2 bf16x2(uint32_t w) { return make_float2(bf16_lo(w), bf16_hi(w)); }

// Two fp32 -> bf16 pair (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Exact FP8 E4M3 and FP4 E2M1 -> fp32 through the sm_100 conversions to f16 pairs: every
// E4M3 value (448 at most, 2^-9 at least) and every E2M1 value is an f16 value, and
// f16 -> fp32 is exact.  The conversion puts the lower byte (nibble) of its input in the
// lower f16, so code k of a word lands in column k.
__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t h) {
    float a, b;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "cvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
        : "=f"(a), "=f"(b) : "r"(h));
    return make_float2(a, b);
}

// Four E4M3 codes (byte k = column k) -> columns (0, 1) and (2, 3).
__device__ __forceinline__ void e4m3x4_to_float(uint32_t w, float2 &c01, float2 &c23) {
    uint32_t h01, h23;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(h01), "=r"(h23) : "r"(w));
    c01 = half2_bits_to_float2(h01);
    c23 = half2_bits_to_float2(h23);
}

// One E4M3 code (the low byte of b) -> its f16 bits (exact), in the low 16 bits.
__device__ __forceinline__ uint32_t e4m3_to_half_bits(uint32_t b) {
    uint32_t h;
    asm("{\n\t.reg .b16 x, lo, hi;\n\t.reg .b32 t;\n\tcvt.u16.u32 x, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 t, x;\n\tmov.b32 {lo, hi}, t;\n\tcvt.u32.u16 %0, lo;\n\t}"
        : "=r"(h) : "r"(b & 0xFFu));
    return h;
}

// Two E4M3 codes (the low bytes of a and b) -> their f16 bits, a in the low half (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_half2_bits(uint32_t a, uint32_t b) {
    uint32_t h;
    asm("{\n\t.reg .b16 x;\n\tcvt.u16.u32 x, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, x;\n\t}"
        : "=r"(h) : "r"((a & 0xFFu) | ((b & 0xFFu) << 8)));
    return h;
}

// Eight E2M1 codes (nibble k = column k), each times the f16 value s, added to fp32
// accumulators: acc[j] (columns 2j, 2j+1) += q * s with one rounding (fma.rn.f32.f16: the
// f16 operands enter exactly, q * s is exact for E2M1 x E4M3).
// kHi: s is the high half of s_half (else the low half).
template <bool kHi = false>
__device__ __forceinline__ void e2m1x8_fma(uint32_t w, uint32_t s_half, float2 acc[4]) {
    uint32_t h0, h1, h2, h3;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3) : "r"(w));
    const uint32_t hh[4] = {h0, h1, h2, h3};
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (kHi)
            asm("{\n\t.reg .b16 lo, hi, s, u;\n\tmov.b32 {lo, hi}, %2;\n\tmov.b32 {u, s}, %3;\n\t"
                "fma.rn.f32.f16 %0, lo, s, %0;\n\tfma.rn.f32.f16 %1, hi, s, %1;\n\t}"
                : "+f"(acc[j].x), "+f"(acc[j].y) : "r"(hh[j]), "r"(s_half));
        else
            asm("{\n\t.reg .b16 lo, hi, s, u;\n\tmov.b32 {lo, hi}, %2;\n\tmov.b32 {s, u}, %3;\n\t"
                "fma.rn.f32.f16 %0, lo, s, %0;\n\tfma.rn.f32.f16 %1, hi, s, %1;\n\t}"
                : "+f"(acc[j].x), "+f"(acc[j].y) : "r"(hh[j]), "r"(s_half));
}

}  // namespace ngram
