// gather_staged.cuh -- the fused gather with whole rows staged in shared memory by the TMA
// engine, for any row format of rows.cuh (same operation and arithmetic, so the same bits).
//
// In the register gathers the loads in flight live in registers: 16 heads x the lane's
// fragment, about 40% of a thread's registers for the 4-bit rows, which caps the bytes in
// flight per SM.  Here the in-flight rows live in shared memory instead:
//   * Work item = one token (all d columns).  A stage holds its 16 rows (row_bytes each,
//     one cp.async.bulk per row -- 1,440 bytes for NVFP4 at d = 2560), its residual row
//     (2d bytes) and, for per-row-scaled formats, the 16 row scales.
//   * A dedicated producer warp (the last warp) issues the copies of the items S - 1
//     ahead and computes the next item's row ids while the consumers work, so neither the
//     hash nor the token loads sit on the ring's critical path.
//   * The consumer warps decode from shared memory, 8 columns per thread, with the
//     row policies (same operations in the same head order as every other gather), apply
//     gate and residual and store bf16 to global memory.
//   * The ring is CTA-synchronous: after each item every thread meets at a barrier, then
//     the producer refills the stage just read.  Every mbarrier wait gives up after 1 s
//     of %globaltimer; on expiry the CTA sets the device error word (code 2), waits
//     (bounded) for its copies still in flight, and returns.
// No multicast: every copy is global -> this CTA's shared memory.
#pragma once

#include "gather_bulk.cuh"
#include "rows.cuh"

namespace ngram {

struct StagedPlan {
    uint32_t stages;        // ring depth, 2..kBulkMaxStages
    uint32_t stage_bytes;   // 16 * row_bytes + 2d + 64 (scales), rounded up to 128
    uint32_t row_bytes;     // bytes of one table row (a multiple of 16)
    uint32_t res_off;       // offset of the residual row in a stage
    uint32_t scale_off;     // offset of the 16 row scales in a stage
};

#ifndef NGRAM_STAGED_MIN_BLOCKS       // resident CTAs per SM the register budget targets
#define NGRAM_STAGED_MIN_BLOCKS 1
#endif

template <int kH, class Rows>
__global__ void __launch_bounds__(352, NGRAM_STAGED_MIN_BLOCKS) k_gather_staged(const GatherArgs g,
                                                                                const StagedPlan plan) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127u) & ~static_cast<uintptr_t>(127u));
    __shared__ uint64_t full[kBulkMaxStages];
    __shared__ uint32_t abort_flag;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t tid = threadIdx.x;
    const uint32_t lane = tid & 31u;
    const uint32_t n_cons = blockDim.x - 32u;            // consumer threads
    const bool producer = tid >= n_cons;
    const uint32_t units = g.d >> 3;                     // 8-column units per token
    const uint8_t *__restrict__ table = static_cast<const uint8_t *>(g.table);
    const float gs = (g.row_scale != nullptr && !Rows::kRowScale) ? __ldg(g.row_scale) : 0.0f;
    const uint32_t res_bytes = g.d * 2u;

    if (tid == 0) {
        for (uint32_t s = 0; s < plan.stages; ++s) mbar_init(&full[s], 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    auto token_of = [&](uint32_t item) { return g.perm ? __ldg(g.perm + item) : item; };
    // producer lanes: the row of head `lane` of an item (0 for lanes >= H)
    auto row_of = [&](uint32_t item) { return warp_head_row(g, token_of(item), lane, H); };
    auto issue = [&](uint32_t item, uint32_t st, uint32_t row) {
        const uint32_t tok = token_of(item);
        uint8_t *base = smem + st * plan.stage_bytes;
        if (Rows::kRowScale && lane < H)
            reinterpret_cast<float *>(base + plan.scale_off)[lane] = __ldg(g.row_scale + row);
        if (lane == 0) mbar_arrive_expect_tx(&full[st], H * plan.row_bytes + res_bytes);
        __syncwarp();
        if (lane < H)
            bulk_copy_g2s(base + lane * plan.row_bytes, table + static_cast<size_t>(row) * plan.row_bytes,
                          plan.row_bytes, &full[st]);
        else if (lane == H)
            bulk_copy_g2s(base + plan.res_off, g.residual + static_cast<size_t>(tok) * g.d, res_bytes,
                          &full[st]);
    };

    uint32_t next_item = blockIdx.x + plan.stages * gridDim.x, next_row = 0;
    if (producer) {
        for (uint32_t s = 0; s < plan.stages; ++s) {
            const uint32_t item = blockIdx.x + s * gridDim.x;
            if (item < g.N) issue(item, s, row_of(item));
        }
        if (next_item < g.N) next_row = row_of(next_item);
    }

    uint32_t k = 0;
    for (uint32_t item = blockIdx.x; item < g.N; item += gridDim.x, ++k) {
        const uint32_t st = k % plan.stages;
        if (!mbar_wait_bounded(&full[st], (k / plan.stages) & 1u)) atomicExch(&abort_flag, 1u);
        __syncthreads();
        if (abort_flag) break;
        if (!producer) {
            const uint8_t *base = smem + st * plan.stage_bytes;
            const size_t tok_off = static_cast<size_t>(token_of(item)) * g.d;
            float sc[16];
#pragma unroll
            for (int h = 0; h < 16; ++h)
                sc[h] = (Rows::kRowScale && (kH || h < static_cast<int>(H)))
                            ? reinterpret_cast<const float *>(base + plan.scale_off)[h] : 0.0f;
            for (uint32_t v = tid; v < units; v += n_cons) {
                float2 acc[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[j] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int h = 0; h < 16; ++h)
                    if (kH || h < static_cast<int>(H))
                        Rows::add(acc, Rows::load_smem(base + h * plan.row_bytes, v, g.d), sc[h], gs);
                Rows::finish(acc, gs);
                const uint4 r = *reinterpret_cast<const uint4 *>(base + plan.res_off + v * 16u);
                float gv[8];
                load_gate8<false>(g, tok_off, v, gv);
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
        __syncthreads();                       // stage st fully read: refill it
        if (producer && next_item < g.N) {
            issue(next_item, st, next_row);
            next_item += gridDim.x;
            if (next_item < g.N) next_row = row_of(next_item);
        }
    }

    if (abort_flag) {
        // record the timeout, then wait (bounded) for this CTA's copies still in flight
        if (tid == 0) {
            atomicCAS(g.err, 0u, 2u);
            for (uint32_t j = 0; j < plan.stages; ++j) {     // the item that timed out, too
                const uint32_t kk = k + j;
                if (blockIdx.x + kk * gridDim.x >= g.N) break;
                mbar_wait_bounded(&full[kk % plan.stages], (kk / plan.stages) & 1u);
            }
        }
        __syncthreads();
    }
}

}  // namespace ngram
