// gather_bulk.cuh -- the bf16 gather staged through shared memory by the TMA engine.
//
// Same operation as k_gather_bf16 ("Qwen Brought Back N-Grams. All 51 Billion
// Parameters of Them.", section "N-grams, of all things": hash, gather 16 rows, sum,
// add to the residual; gate of "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with
// Heterogeneous Memory Prefetch", Key point 1), with a different memory pipeline:
//   * A work item is (token, column chunk).  Warp 0 hashes the token's heads and each
//     hashing lane issues ONE bulk copy (cp.async.bulk, global -> shared, no multicast)
//     of its row's chunk; one more lane copies the residual chunk.  All copies of an
//     item complete on one mbarrier (expect_tx = bytes of the item).
//   * A ring of S stages keeps S-1 items in flight per CTA while the CTA sums the
//     current one out of shared memory (fp32, head order), applies gate and residual
//     and stores bf16 to global memory.
//   * Every wait is bounded by a 1 s deadline on %globaltimer; on expiry the CTA sets
//     the device error word (code 2), waits (bounded) for its other copies and returns.
#pragma once

#include "device_common.cuh"
#include "gather.cuh"

namespace ngram {

constexpr uint32_t kBulkMaxStages = 16;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for phase `parity` of bar, giving up after the deadline.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t deadline = global_ns() + limit_ns;
    while (!mbar_try_wait(bar, parity))
        if (global_ns() > deadline) return false;
    return true;
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from global
// memory of this GPU into this CTA's shared memory, completing on bar.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// The error path of the bounded waits, on demand: one mbarrier that expects one arrival
// which never comes, waited on with mbar_wait_bounded.  The wait must give up after
// limit_ns, set the device error word (code 2) and return; nothing else runs.
__global__ void __launch_bounds__(32) k_selftest_wait(uint32_t *err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit_ns)) atomicCAS(err, 0u, 2u);
}

struct BulkPlan {
    uint32_t chunk_cols;    // columns per item (multiple of 8)
    uint32_t n_chunks;      // ceil(d / chunk_cols)
    uint32_t stages;        // ring depth, 2..16
    uint32_t stage_bytes;   // (H + 1) * chunk_cols * 2, rounded up to 128
};

template <int kH>
__global__ void __launch_bounds__(512, 1) k_gather_bf16_bulk(const GatherArgs g, const BulkPlan plan) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // stage ring base rounded up to 128 bytes (the launch adds 128 spare bytes)
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127u) & ~static_cast<uintptr_t>(127u));
    __shared__ uint64_t full[kBulkMaxStages];
    __shared__ uint32_t abort_flag;
    const uint32_t H = kH ? static_cast<uint32_t>(kH) : g.h.n_heads;
    const uint32_t tid = threadIdx.x;
    const uint32_t lane = tid & 31u;
    const bool producer_warp = (tid >> 5) == 0;
    const uint32_t slot_bytes = plan.chunk_cols * 2u;          // one row chunk in the stage
    const uint32_t n_items = g.N * plan.n_chunks;
    const uint16_t *__restrict__ table = static_cast<const uint16_t *>(g.table);

    if (tid == 0) {
        for (uint32_t s = 0; s < plan.stages; ++s) mbar_init(&full[s], 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // warp 0: hash the item's token and launch its H + 1 bulk copies into stage st
    auto issue = [&](uint32_t item, uint32_t st) {
        const uint32_t tok = item / plan.n_chunks;
        const uint32_t col0 = (item - tok * plan.n_chunks) * plan.chunk_cols;
        const uint32_t bytes = min(plan.chunk_cols, g.d - col0) * 2u;
        const uint32_t row = warp_head_row(g, tok, lane, H);
        uint8_t *base = smem + st * plan.stage_bytes;
        if (lane == 0) mbar_arrive_expect_tx(&full[st], (H + 1u) * bytes);
        __syncwarp();
        if (lane < H)
            bulk_copy_g2s(base + lane * slot_bytes, table + static_cast<size_t>(row) * g.d + col0,
                          bytes, &full[st]);
        else if (lane == H)
            bulk_copy_g2s(base + H * slot_bytes, g.residual + static_cast<size_t>(tok) * g.d + col0,
                          bytes, &full[st]);
    };

    // prologue: fill the ring
    if (producer_warp)
        for (uint32_t s = 0; s < plan.stages; ++s) {
            const uint32_t item = blockIdx.x + s * gridDim.x;
            if (item < n_items) issue(item, s);
        }

    uint32_t k = 0;
    for (uint32_t item = blockIdx.x; item < n_items; item += gridDim.x, ++k) {
        const uint32_t st = k % plan.stages;
        const uint32_t parity = (k / plan.stages) & 1u;
        if (!mbar_wait_bounded(&full[st], parity)) atomicExch(&abort_flag, 1u);
        __syncthreads();
        if (abort_flag) break;

        const uint32_t tok = item / plan.n_chunks;
        const uint32_t col0 = (item - tok * plan.n_chunks) * plan.chunk_cols;
        const uint32_t nv = min(plan.chunk_cols, g.d - col0) >> 3;
        const uint8_t *base = smem + st * plan.stage_bytes;
        const size_t out_off = static_cast<size_t>(tok) * g.d + col0;
        for (uint32_t v = tid; v < nv; v += blockDim.x) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                if (kH || h < static_cast<int>(H)) {
                    const uint4 e = *reinterpret_cast<const uint4 *>(base + h * slot_bytes + v * 16u);
                    acc[0] = __fadd_rn(acc[0], bf16_lo(e.x));
                    acc[1] = __fadd_rn(acc[1], bf16_hi(e.x));
                    acc[2] = __fadd_rn(acc[2], bf16_lo(e.y));
                    acc[3] = __fadd_rn(acc[3], bf16_hi(e.y));
                    acc[4] = __fadd_rn(acc[4], bf16_lo(e.z));
                    acc[5] = __fadd_rn(acc[5], bf16_hi(e.z));
                    acc[6] = __fadd_rn(acc[6], bf16_lo(e.w));
                    acc[7] = __fadd_rn(acc[7], bf16_hi(e.w));
                }
            }
            const uint4 r = *reinterpret_cast<const uint4 *>(base + H * slot_bytes + v * 16u);
            const float4 *gp = reinterpret_cast<const float4 *>(g.gate + col0) + 2u * v;
            const float4 ga = __ldg(gp), gb = __ldg(gp + 1);
            const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
            uint32_t o[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float y0 = __fadd_rn(bf16_lo(rw[p]), __fmul_rn(gv[2 * p], acc[2 * p]));
                const float y1 = __fadd_rn(bf16_hi(rw[p]), __fmul_rn(gv[2 * p + 1], acc[2 * p + 1]));
                o[p] = pack_bf16x2(y0, y1);
            }
            *reinterpret_cast<uint4 *>(g.out + out_off + v * 8u) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncthreads();                       // stage st fully read: refill it
        if (producer_warp) {
            const uint32_t next = item + plan.stages * gridDim.x;
            if (next < n_items) issue(next, st);
        }
    }

    if (abort_flag) {
        // record the timeout, then wait (bounded) for this CTA's other copies in flight
        if (tid == 0) {
            atomicCAS(g.err, 0u, 2u);
            for (uint32_t j = 1; j < plan.stages; ++j) {
                const uint32_t kk = k + j;
                const uint32_t it = blockIdx.x + kk * gridDim.x;
                if (it >= n_items) break;
                mbar_wait_bounded(&full[kk % plan.stages], (kk / plan.stages) & 1u);
            }
        }
        __syncthreads();
    }
}

}  // namespace ngram
