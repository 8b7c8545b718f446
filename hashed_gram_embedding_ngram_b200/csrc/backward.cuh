// backward.cuh -- the backward pass of out = residual + g (elementwise) sum_h E[idx_h].
//
// The table is learned ("Qwen Brought Back N-Grams. All 51 Billion Parameters of Them.",
// section "N-grams, of all things": a table the model learns), and the gate may be the
// output of a gating network ("Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with
// Heterogeneous Memory Prefetch", Summary).  Given dy = dL/dout (bf16 [N][d]):
//   * table: only the rows the batch read have a gradient.  Distinct row u (in order of
//     first occurrence, the list of the dedup step) receives, over its occurrences i =
//     token * H + head in ascending order, S = sum dy[token] in fp32 (then g * S, one
//     rounding) -- or, with a per-token gate, acc = fma(g[token], dy[token], acc).  The
//     occurrences are listed by a stable radix sort (sort.cuh), so the order, and the
//     result, are the same on every run; no floating-point atomics.
//   * gate: shared gate [d]: dg = sum over tokens of dy * e, with e the forward's fp32 head
//     sum recomputed here; each product dy * e is exact in fp64 and the sum runs in fp64
//     over fixed chunks of kGateChunk tokens (per (chunk, column) partials), then over
//     groups of kGateGroup chunks and over the groups, each in order, rounded once to fp32
//     -- a fixed order, so the same result for any grid size.
//     Per-token gate [N][d]: dg[t] = fp32(dy[t] * e[t]).
//   * residual: dL/dresidual = dy; nothing to compute.
//
// The gate-gradient kernel recomputes e with the row-format policies of rows.cuh, which
// decode and sum exactly as the forward gathers do (same operations in the same head
// order), so e is bit-identical to the forward's.  A lane owns 8 columns here.
//
// Every kernel here opens with allow_dependents(); grid_dependency_wait(), so the steps of
// a backward call may be launched as programmatic dependents of one another.
#pragma once

#include "rows.cuh"

namespace ngram {

constexpr uint32_t kGateChunk = 16;     // tokens per partial sum of the shared-gate gradient

// ---------------------------------------------------------------- gate gradient
// Work item = (chunk of kChunk tokens, strip of 32 lanes x 8 columns).  kPerToken: chunk of
// one token, dg_tok[t] = fp32(dy * e); else the fp64 sum of dy * e over the chunk's tokens
// goes to partial[chunk][d].
template <int kH, class Rows, bool kPerToken>
__global__ void __launch_bounds__(256, 2) k_gate_grad(const GatherArgs g, const uint16_t *__restrict__ dy,
                                                      float *__restrict__ dg_tok,
                                                      double *__restrict__ partial, uint32_t row_bytes) {
    allow_dependents();
    grid_dependency_wait();
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t nvec = g.d >> 3;
    const uint32_t n_strips = (nvec + 31u) >> 5;
    const uint32_t chunk = kPerToken ? 1u : kGateChunk;
    const uint32_t n_chunks = (g.N + chunk - 1u) / chunk;
    const uint32_t n_items = n_chunks * n_strips;
    const uint8_t *__restrict__ table = static_cast<const uint8_t *>(g.table);
    const float gs = (g.row_scale != nullptr && !Rows::kRowScale) ? __ldg(g.row_scale) : 0.0f;

    for (uint32_t item = warp; item < n_items; item += n_warps) {
        const uint32_t ch = item / n_strips;
        const uint32_t v = (item - ch * n_strips) * 32u + lane;
        const bool active = v < nvec;
        const uint32_t t_end = min(g.N, (ch + 1u) * chunk);
        double part[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) part[k] = 0.0;
        for (uint32_t tok = ch * chunk; tok < t_end; ++tok) {
            const uint32_t my_row = warp_head_row(g, tok, lane, H);
            const float my_scale = (Rows::kRowScale && lane < H) ? __ldg(g.row_scale + my_row) : 0.0f;
            uint32_t rows[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) rows[h] = __shfl_sync(0xFFFFFFFFu, my_row, h);
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
            const size_t off = static_cast<size_t>(tok) * g.d + v * 8u;
            const uint4 dw = ld_na_v4(dy + off);
            float2 acc[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int h = 0; h < 16; ++h)
                if (kH || h < static_cast<int>(H)) Rows::add(acc, f[h], sc[h], gs);
            Rows::finish(acc, gs);
            const float dv[8] = {bf16_lo(dw.x), bf16_hi(dw.x), bf16_lo(dw.y), bf16_hi(dw.y),
                                 bf16_lo(dw.z), bf16_hi(dw.z), bf16_lo(dw.w), bf16_hi(dw.w)};
            const float ev[8] = {acc[0].x, acc[0].y, acc[1].x, acc[1].y,
                                 acc[2].x, acc[2].y, acc[3].x, acc[3].y};
            if (kPerToken) {
                float o[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) o[k] = __fmul_rn(dv[k], ev[k]);
                float4 *dst = reinterpret_cast<float4 *>(dg_tok + off);
                dst[0] = make_float4(o[0], o[1], o[2], o[3]);
                dst[1] = make_float4(o[4], o[5], o[6], o[7]);
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k)      // the product is exact in fp64
                    part[k] = __dadd_rn(part[k], __dmul_rn(static_cast<double>(dv[k]),
                                                           static_cast<double>(ev[k])));
            }
        }
        if (!kPerToken && active) {
            double2 *dst = reinterpret_cast<double2 *>(partial + static_cast<size_t>(ch) * g.d + v * 8u);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_double2(part[2 * k], part[2 * k + 1]);
        }
    }
}

// Shared-gate gradient from the [n_chunks][d] fp64 partials, in a fixed two-level order:
// k_gate_reduce_groups sums each group of kGateGroup consecutive chunks in order into
// group[g][d]; k_gate_reduce sums the groups in order and rounds once to fp32.  The order
// depends only on N, so the result is the same on every run.
constexpr uint32_t kGateGroup = 32;

__global__ void __launch_bounds__(256) k_gate_reduce_groups(const double *__restrict__ partial,
                                                            uint32_t n_chunks, uint32_t d,
                                                            double *__restrict__ group) {
    allow_dependents();
    grid_dependency_wait();
    const uint32_t c = blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t gi = blockIdx.y;
    if (c >= d) return;
    const uint32_t ch_end = min(n_chunks, (gi + 1u) * kGateGroup);
    double s = 0.0;
    for (uint32_t ch = gi * kGateGroup; ch < ch_end; ++ch)
        s = __dadd_rn(s, partial[static_cast<size_t>(ch) * d + c]);
    group[static_cast<size_t>(gi) * d + c] = s;
}

__global__ void __launch_bounds__(256) k_gate_reduce(const double *__restrict__ group, uint32_t n_groups,
                                                     uint32_t d, float *__restrict__ dg) {
    allow_dependents();
    grid_dependency_wait();
    const uint32_t c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= d) return;
    double s = 0.0;
    for (uint32_t gi = 0; gi < n_groups; ++gi) s = __dadd_rn(s, group[static_cast<size_t>(gi) * d + c]);
    dg[c] = __double2float_rn(s);
}

// ---------------------------------------------------------------- table gradient
// seg[u] = first position of row u in the sorted occurrence list; seg[U] = M.
__global__ void __launch_bounds__(256) k_seg_starts(const uint32_t *__restrict__ skeys, uint32_t M,
                                                    uint32_t *__restrict__ seg) {
    allow_dependents();
    grid_dependency_wait();
    for (uint32_t p = blockIdx.x * blockDim.x + threadIdx.x; p < M; p += gridDim.x * blockDim.x) {
        const uint32_t u = skeys[p];
        if (p == 0 || skeys[p - 1] != u) seg[u] = p;
        if (p == M - 1) seg[u + 1] = M;
    }
}

// One warp per (chunk of 32 consecutive distinct rows u0 .. u0+31, group of kStrips strips
// of 256 columns).  In each strip a lane owns columns 4l .. 4l+3 and 128+4l .. 128+4l+3,
// so each of its two float4 stores is part of a contiguous 512-byte warp store (whole
// sectors), and dy comes in two 8-byte loads.  Lane i loads seg[u0 + i], so the occurrence
// range of every row of the chunk is known at once; the chunk's occurrences [P0, P1) --
// each row's own in ascending order, rows one after the other -- are walked in batches of
// kBatch: the batch's loads are issued first (the tokens come from one coalesced load of
// occ_tok; a token's heads usually open consecutive rows, so L1 serves the repeats), then
// added in order, and a row's gradient is stored as soon as its last occurrence is in.
// Warps take items from an atomic counter (*next_item, zeroed before the launch): chunks
// holding the most frequent rows come first (frequent contexts appear early in a batch),
// and no warp is left with a long tail.
#ifndef NGRAM_ROWS_GRAD_STRIPS
#define NGRAM_ROWS_GRAD_STRIPS 1
#endif
// Depth per warp beats warps per SM here (B200, full prefill, ngram_backward_rows):
// 16 fragments at 2 CTAs/SM 1.077 ms; 8 at 3 CTAs 1.19 ms; 8 at 4 CTAs 1.22 ms; 12 at 3
// CTAs 1.25 ms.
#ifndef NGRAM_ROWS_GRAD_BATCH         // dy fragments in flight per lane (shared gate)
#define NGRAM_ROWS_GRAD_BATCH 16
#endif
#ifndef NGRAM_ROWS_GRAD_MIN_BLOCKS    // resident CTAs per SM the register budget targets
#define NGRAM_ROWS_GRAD_MIN_BLOCKS 2
#endif

template <bool kTokGate, int kStrips>
__global__ void __launch_bounds__(256, NGRAM_ROWS_GRAD_MIN_BLOCKS) k_rows_grad(const uint32_t *__restrict__ count,
                                                      const uint32_t *__restrict__ seg,
                                                      const uint32_t *__restrict__ occ_tok,
                                                      const uint16_t *__restrict__ dy,
                                                      const float *__restrict__ gate,
                                                      const uint16_t *__restrict__ gate_tok,
                                                      uint32_t d, float *__restrict__ grad,
                                                      uint32_t *next_item) {
    allow_dependents();
    grid_dependency_wait();
    constexpr uint32_t kBatch = (kTokGate ? NGRAM_ROWS_GRAD_BATCH / 2u : NGRAM_ROWS_GRAD_BATCH) / kStrips;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t n_strips = ((d >> 3) + 31u) >> 5;
    const uint32_t n_groups = (n_strips + kStrips - 1u) / kStrips;
    const uint32_t U = *count;
    const uint32_t n_items = ((U + 31u) >> 5) * n_groups;
    for (;;) {
        uint32_t item = 0;
        if (lane == 0) item = atomicAdd(next_item, 1u);
        item = __shfl_sync(0xFFFFFFFFu, item, 0);
        if (item >= n_items) break;
        const uint32_t ch = item / n_groups;
        const uint32_t grp = item - ch * n_groups;
        uint32_t c0[kStrips];                 // first column of the lane's first quad in each strip
        bool act[kStrips][2];                 // quad h (columns c0 + 128h ..) inside the row
#pragma unroll
        for (int k = 0; k < kStrips; ++k) {
            c0[k] = (grp * kStrips + k) * 256u + lane * 4u;
            act[k][0] = c0[k] < d;            // d % 8 == 0: a quad is wholly in or out
            act[k][1] = c0[k] + 128u < d;
        }
        const uint32_t u0 = ch * 32u;
        const uint32_t nu = min(32u, U - u0);
        const uint32_t P1 = __ldg(seg + u0 + nu);                     // end of the chunk's last row
        const uint32_t my_seg = lane < nu ? __ldg(seg + u0 + lane) : P1;
        const uint32_t P0 = __shfl_sync(0xFFFFFFFFu, my_seg, 0);
        uint32_t r = 0;                                              // current row of the chunk
        uint32_t next_end = __shfl_sync(0xFFFFFFFFu, my_seg, 1);      // first position after it
        if (nu == 1) next_end = P1;
        float acc[kStrips][8];
#pragma unroll
        for (int k = 0; k < kStrips; ++k)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[k][j] = 0.0f;
        for (uint32_t p0 = P0; p0 < P1; p0 += 32u) {
            const uint32_t nb = min(32u, P1 - p0);
            const uint32_t my_tok = lane < nb ? __ldg(occ_tok + p0 + lane) : 0u;
            for (uint32_t j0 = 0; j0 < nb; j0 += kBatch) {
                uint2 w[kBatch][kStrips][2], gw[kBatch][kStrips][2];
#pragma unroll
                for (uint32_t q = 0; q < kBatch; ++q) {
                    const uint32_t tok = __shfl_sync(0xFFFFFFFFu, my_tok, (j0 + q) & 31u);
                    if (j0 + q < nb) {
                        const uint16_t *row = dy + static_cast<size_t>(tok) * d;
                        const uint16_t *grow = gate_tok + static_cast<size_t>(tok) * d;
#pragma unroll
                        for (int k = 0; k < kStrips; ++k) {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                if (act[k][h]) {
                                    w[q][k][h] = __ldg(reinterpret_cast<const uint2 *>(row + c0[k] + h * 128u));
                                    if (kTokGate)
                                        gw[q][k][h] = __ldg(reinterpret_cast<const uint2 *>(grow + c0[k] + h * 128u));
                                }
                            }
                        }
                    }
                }
#pragma unroll
                for (uint32_t q = 0; q < kBatch; ++q) {
                    if (j0 + q >= nb) break;                          // warp-uniform
#pragma unroll
                    for (int k = 0; k < kStrips; ++k) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if (!act[k][h]) continue;
                            const uint32_t ww[2] = {w[q][k][h].x, w[q][k][h].y};
                            float *a = &acc[k][4 * h];
                            if (kTokGate) {
                                const uint32_t gg[2] = {gw[q][k][h].x, gw[q][k][h].y};
#pragma unroll
                                for (int p = 0; p < 2; ++p) {
                                    a[2 * p] = __fmaf_rn(bf16_lo(gg[p]), bf16_lo(ww[p]), a[2 * p]);
                                    a[2 * p + 1] = __fmaf_rn(bf16_hi(gg[p]), bf16_hi(ww[p]), a[2 * p + 1]);
                                }
                            } else {
#pragma unroll
                                for (int p = 0; p < 2; ++p) {
                                    a[2 * p] = __fadd_rn(a[2 * p], bf16_lo(ww[p]));
                                    a[2 * p + 1] = __fadd_rn(a[2 * p + 1], bf16_hi(ww[p]));
                                }
                            }
                        }
                    }
                    if (p0 + j0 + q + 1u == next_end) {                // row u0 + r is complete
                        float *row = grad + static_cast<size_t>(u0 + r) * d;
#pragma unroll
                        for (int k = 0; k < kStrips; ++k) {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                if (act[k][h]) {
                                    float o[4];
                                    if (kTokGate) {
#pragma unroll
                                        for (int j = 0; j < 4; ++j) o[j] = acc[k][4 * h + j];
                                    } else {
                                        const float4 gq = __ldg(reinterpret_cast<const float4 *>(gate + c0[k] + h * 128u));
                                        o[0] = __fmul_rn(gq.x, acc[k][4 * h]);
                                        o[1] = __fmul_rn(gq.y, acc[k][4 * h + 1]);
                                        o[2] = __fmul_rn(gq.z, acc[k][4 * h + 2]);
                                        o[3] = __fmul_rn(gq.w, acc[k][4 * h + 3]);
                                    }
                                    // streaming store: the gradient rows are written once,
                                    // so they should not push dy out of L2
                                    __stcs(reinterpret_cast<float4 *>(row + c0[k] + h * 128u),
                                           make_float4(o[0], o[1], o[2], o[3]));
                                }
                            }
#pragma unroll
                            for (int j = 0; j < 8; ++j) acc[k][j] = 0.0f;
                        }
                        ++r;
                        const uint32_t e = __shfl_sync(0xFFFFFFFFu, my_seg, (r + 1u) & 31u);
                        next_end = (r + 1u < nu) ? e : P1;
                    }
                }
            }
        }
    }
}

}  // namespace ngram
