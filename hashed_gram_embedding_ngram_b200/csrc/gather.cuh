// gather.cuh -- the hot path: context -> 16 hashed rows -> fp32 sum -> gate -> residual.
//
// "Qwen Brought Back N-Grams. All 51 Billion Parameters of Them.", section "N-grams,
// of all things": hash the bigram and trigram context into the table, gather 16 rows,
// sum them into one d-wide vector that is added to the residual stream.  The gate is
// the elementwise W_g of "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with
// Heterogeneous Memory Prefetch", Key point 1.
//
// Design (HBM-bound gather, no contraction, so no tensor cores):
//   * One warp owns one (token, group of 32-vector column strips) work item.  Lanes
//     0..H-1 form the context and hash one head each; the H row indices are then
//     broadcast with shuffles, so there is no shared memory and no block barrier.
//   * For each strip a lane owns one 16-byte column vector (8 bf16): it issues all H
//     row loads (16 x 16 B in flight per lane, 8 KB per warp) plus the residual load
//     before the first add, then sums in head order 0..H-1 in fp32 (packed pairs of
//     columns, each rounded like a scalar add), applies y = r + g * acc with separately
//     rounded multiply and add, and stores bf16.
//   * Work items are dealt to a persistent grid (blocks = SMs x resident blocks).  For
//     bf16 every item is one strip, so a token's strips run on several warps at once;
//     on large grouped batches the order step has already written every token's 16 row
//     ids (row_ids), which the hashing lanes then read instead of hashing per strip.
#pragma once

#include "device_common.cuh"

namespace ngram {

struct GatherArgs {
    HashArgs h;
    const void *table;          // [R][d] bf16 bits, or int8
    const float *row_scale;     // [R] (int8)
    const int32_t *tokens;      // [n_seq][T]
    const int32_t *history;     // [n_seq][2] or null
    const uint16_t *residual;   // [N][d] bf16 bits
    const float *gate;          // [d], shared by every token
    const uint16_t *gate_tok;   // [N][d] bf16 bits, a gate per token (replaces gate), or null
    uint16_t *out;              // [N][d] bf16 bits (may alias residual)
    const uint32_t *row_ids;    // [N][H] precomputed row ids into `table`, or null (hash)
    const uint32_t *perm;       // [N] processing order of the tokens, or null (batch order)
    uint32_t *err;              // device error word
    uint32_t T;
    uint32_t N;                 // tokens of this launch: flat tokens [tok_begin, tok_begin + N)
    uint32_t tok_begin;         // first flat token (contexts read tokens / history globally;
                                // residual / out are indexed from the launch's first token)
    uint32_t d;
    uint32_t n_strips;          // strips of 32 column vectors per token
    uint32_t strips_per_item;
    uint32_t groups_per_token;  // ceil(n_strips / strips_per_item)
    // column-sharded table (k_gather_c8<.., kShard = true> only): residual, gate_tok and
    // every outs[p] are rows of ld elements, already offset to this shard's first column;
    // the shard's columns of each token are stored to all n_outs buffers
    uint32_t ld;
    uint32_t n_outs;
    uint16_t *outs[8];
    // 1: the kernel lets the next programmatic-dependent kernel of its stream be scheduled as
    // soon as it starts (full-grid launches); 0: only when it ends (a bounded grid that runs
    // long beside other work, whose successor would otherwise sit resident and waiting)
    uint32_t trigger_early;
};

// 16-byte load through L2 without L1 allocation; coherent (the residual may be the
// output buffer of the same launch when the caller works in place).
__device__ __forceinline__ uint4 ld_na_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Row indices of the warp's token, one head per lane (lanes >= H hold 0): hashed
// from the context, or read from precomputed ids -- the table's own rows hashed once by
// the order step, or, on the dedup'ed / staged paths, the inverse map into the staging
// buffer that `table` then points to.  seed: head_seed(lane) (the caller computes it once
// per lane, outside its item loop).
__device__ __forceinline__ uint32_t warp_head_row(const GatherArgs &g, uint32_t tok,
                                                  uint32_t lane, uint32_t H, uint64_t seed) {
    uint32_t row = 0;
    if (lane < H) {
        const uint32_t flat = g.tok_begin + tok;
        if (g.row_ids != nullptr) {
            row = __ldg(g.row_ids + static_cast<size_t>(flat) * H + lane);
        } else {
            uint32_t w0, w1, w2;
            token_context(g.tokens, g.history, flat, g.T, g.h, g.err, w0, w1, w2);
            row = head_row_seeded(lane, seed, w0, w1, w2, g.h);
        }
    }
    return row;
}

__device__ __forceinline__ uint32_t warp_head_row(const GatherArgs &g, uint32_t tok,
                                                  uint32_t lane, uint32_t H) {
    return warp_head_row(g, tok, lane, H, head_seed(lane, g.h));
}

// The gate of columns 8v .. 8v+7 of one token: the shared fp32 gate, or (kTokGate) the
// token's bf16 gate (exact in fp32).
template <bool kTokGate>
__device__ __forceinline__ void load_gate8(const GatherArgs &g, size_t tok_off, uint32_t v, float gv[8]) {
    if (kTokGate) {
        const uint4 w = ld_na_v4(g.gate_tok + tok_off + v * 8u);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            gv[2 * p] = bf16_lo(ww[p]);
            gv[2 * p + 1] = bf16_hi(ww[p]);
        }
    } else {
        const float4 ga = __ldg(reinterpret_cast<const float4 *>(g.gate) + 2u * v);
        const float4 gb = __ldg(reinterpret_cast<const float4 *>(g.gate) + 2u * v + 1u);
        gv[0] = ga.x; gv[1] = ga.y; gv[2] = ga.z; gv[3] = ga.w;
        gv[4] = gb.x; gv[5] = gb.y; gv[6] = gb.z; gv[7] = gb.w;
    }
}

#ifndef NGRAM_LDG_MIN_BLOCKS          // resident CTAs per SM the register budget targets
#define NGRAM_LDG_MIN_BLOCKS 2
#endif

// kH: compile-time head count (16), or 0: runtime g.h.n_heads <= 16.  kTokGate: the gate
// is g.gate_tok (per token) instead of g.gate.  kMinBlocks: resident CTAs per SM the
// register budget targets (2 by default; 3 for batches whose work items fit one wave of
// 3 CTAs per SM but not of 2, the decode batches of a few hundred tokens).
template <int kH, bool kTokGate = false, int kMinBlocks = NGRAM_LDG_MIN_BLOCKS>
__global__ void __launch_bounds__(256, kMinBlocks) k_gather_bf16(const GatherArgs g) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t nvec = g.d >> 3;
    const uint32_t n_items = g.N * g.groups_per_token;
    const uint16_t *__restrict__ table = static_cast<const uint16_t *>(g.table);
    const uint64_t seed = head_seed(lane, g.h);           // arithmetic only: before the wait
    if (g.trigger_early) allow_dependents();
    grid_dependency_wait();

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
            if (v >= nvec) continue;
            // issue every load of this column vector before the first add
            uint4 e[16];
#pragma unroll
            for (int h = 0; h < 16; ++h)
                if (kH || h < static_cast<int>(H))
                    e[h] = ld_stream_v4(table + static_cast<size_t>(rows[h]) * g.d + v * 8u);
            const uint4 r = ld_na_v4(g.residual + tok_off + v * 8u);
            float gv[8];
            load_gate8<kTokGate>(g, tok_off, v, gv);

            // acc[p] holds columns (2p, 2p+1): packed pair adds round each lane exactly as
            // the scalar head-order sum
            float2 acc[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) acc[p] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                if (kH || h < static_cast<int>(H)) {
                    acc[0] = add2(acc[0], bf16x2(e[h].x));
                    acc[1] = add2(acc[1], bf16x2(e[h].y));
                    acc[2] = add2(acc[2], bf16x2(e[h].z));
                    acc[3] = add2(acc[3], bf16x2(e[h].w));
                }
            }
            // y = r + (g * acc): the product is rounded on its own (scalar, never fused)
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
            uint32_t o[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float y0 = __fadd_rn(bf16_lo(rw[p]), __fmul_rn(gv[2 * p], acc[p].x));
                const float y1 = __fadd_rn(bf16_hi(rw[p]), __fmul_rn(gv[2 * p + 1], acc[p].y));
                o[p] = pack_bf16x2(y0, y1);
            }
            *reinterpret_cast<uint4 *>(g.out + tok_off + v * 8u) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// The index step alone: one thread per (token, head).
__global__ void __launch_bounds__(256) k_hash_indices(const HashArgs a,
                                                      const int32_t *__restrict__ tokens,
                                                      const int32_t *__restrict__ history,
                                                      uint32_t T, uint32_t N, uint32_t *err,
                                                      uint32_t *__restrict__ idx_out) {
    allow_dependents();
    grid_dependency_wait();
    const uint32_t H = a.n_heads;
    const uint32_t total = N * H;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += gridDim.x * blockDim.x) {
        const uint32_t tok = i / H;
        const uint32_t h = i - tok * H;
        uint32_t w0, w1, w2;
        token_context(tokens, history, tok, T, a, err, w0, w1, w2);
        idx_out[i] = head_row(h, w0, w1, w2, a);
    }
}

}  // namespace ngram
