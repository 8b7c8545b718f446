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
//     over fixed chunks of kGateChunk tokens (per (chunk, column) partials), then over the
//     chunks in order, rounded once to fp32 -- deterministic for any grid size.
//     Per-token gate [N][d]: dg[t] = fp32(dy[t] * e[t]).
//   * residual: dL/dresidual = dy; nothing to compute.
//
// The gate-gradient kernel recomputes e with the row-format policies of rows.cuh, which
// decode and sum exactly as the forward gathers do (same operations in the same head
// order), so e is bit-identical to the forward's.  A lane owns 8 columns here.
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

// dg[c] = fp32(sum over chunks, in order, of partial[chunk][c]).
__global__ void __launch_bounds__(256) k_gate_reduce(const double *__restrict__ partial, uint32_t n_chunks,
                                                     uint32_t d, float *__restrict__ dg) {
    const uint32_t c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= d) return;
    double s = 0.0;
    for (uint32_t ch = 0; ch < n_chunks; ++ch) s = __dadd_rn(s, partial[static_cast<size_t>(ch) * d + c]);
    dg[c] = __double2float_rn(s);
}

// ---------------------------------------------------------------- table gradient
// seg[u] = first position of row u in the sorted occurrence list; seg[U] = M.
__global__ void __launch_bounds__(256) k_seg_starts(const uint32_t *__restrict__ skeys, uint32_t M,
                                                    uint32_t *__restrict__ seg) {
    for (uint32_t p = blockIdx.x * blockDim.x + threadIdx.x; p < M; p += gridDim.x * blockDim.x) {
        const uint32_t u = skeys[p];
        if (p == 0 || skeys[p - 1] != u) seg[u] = p;
        if (p == M - 1) seg[u + 1] = M;
    }
}

// One warp per (distinct row u, strip of 256 columns); a lane owns 8 columns.  The row's
// occurrences occ_tok[seg[u] .. seg[u+1]) (token of each, ascending) are read in groups
// of 4 loads in flight and summed in order.
__global__ void __launch_bounds__(256) k_rows_grad(const uint32_t *__restrict__ count,
                                                   const uint32_t *__restrict__ seg,
                                                   const uint32_t *__restrict__ occ_tok,
                                                   const uint16_t *__restrict__ dy,
                                                   const float *__restrict__ gate,
                                                   const uint16_t *__restrict__ gate_tok,
                                                   uint32_t d, float *__restrict__ grad) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t nvec = d >> 3;
    const uint32_t n_strips = (nvec + 31u) >> 5;
    const uint32_t U = *count;
    const uint32_t n_items = U * n_strips;
    for (uint32_t item = warp; item < n_items; item += n_warps) {
        const uint32_t u = item / n_strips;
        const uint32_t v = (item - u * n_strips) * 32u + lane;
        if (v >= nvec) continue;
        const uint32_t j0 = __ldg(seg + u), j1 = __ldg(seg + u + 1);
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
        for (uint32_t j = j0; j < j1; j += 4) {
            const uint32_t nq = min(4u, j1 - j);
            uint4 w[4], gw[4];
#pragma unroll
            for (uint32_t q = 0; q < 4; ++q) {
                if (q < nq) {
                    const size_t off = static_cast<size_t>(__ldg(occ_tok + j + q)) * d + v * 8u;
                    w[q] = ld_na_v4(dy + off);
                    if (gate_tok) gw[q] = ld_na_v4(gate_tok + off);
                }
            }
#pragma unroll
            for (uint32_t q = 0; q < 4; ++q) {
                if (q < nq) {
                    const uint32_t ww[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
                    if (gate_tok) {
                        const uint32_t gg[4] = {gw[q].x, gw[q].y, gw[q].z, gw[q].w};
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            acc[2 * p] = __fmaf_rn(bf16_lo(gg[p]), bf16_lo(ww[p]), acc[2 * p]);
                            acc[2 * p + 1] = __fmaf_rn(bf16_hi(gg[p]), bf16_hi(ww[p]), acc[2 * p + 1]);
                        }
                    } else {
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            acc[2 * p] = __fadd_rn(acc[2 * p], bf16_lo(ww[p]));
                            acc[2 * p + 1] = __fadd_rn(acc[2 * p + 1], bf16_hi(ww[p]));
                        }
                    }
                }
            }
        }
        if (!gate_tok) {
            const float4 ga = __ldg(reinterpret_cast<const float4 *>(gate) + 2u * v);
            const float4 gb = __ldg(reinterpret_cast<const float4 *>(gate) + 2u * v + 1u);
            const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = __fmul_rn(gv[k], acc[k]);
        }
        float4 *dst = reinterpret_cast<float4 *>(grad + static_cast<size_t>(u) * d + v * 8u);
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

}  // namespace ngram
