// mma_peak.cuh -- the ceiling that the INT4 and INT8 linear layers are
// measured against: the rate of dense tcgen05.mma.kind::i8 instructions of the
// shape those kernels use (CTA pairs, M 256, N 256, K 32, int32 accumulation
// in tensor memory), with both operands resident in shared memory, so nothing
// but the tensor pipe is timed.  No copies, no epilogue: the leader thread of
// every CTA pair issues `steps` groups of four MMAs (one 128-byte K block)
// into one accumulator and waits for them at the end; the results are never
// read.  One CTA per SM (the shared-memory request keeps a second one off).
#pragma once

#include "int4_gemm.cuh"

namespace quarot {

struct MmaPeakShape {
    static constexpr int kTile = 128 * kGemmBK;                 // 16 KB: 128 rows x 128 bytes
    static constexpr int kThreads = 128;
    static constexpr int kTmemCols = 256;
    static constexpr int kBarOffset = 2 * kTile;
    static constexpr int kMiscOffset = kBarOffset + 16;
    // more than half of the SM's shared memory: one CTA per SM
    static constexpr int kSmemBytes = 120 * 1024;
    static_assert(kMiscOffset + 16 + 1024 <= kSmemBytes, "layout fits");
};

__global__ void __launch_bounds__(MmaPeakShape::kThreads, 1)
mma_peak_i8_kernel(int64_t steps)
{
    using S = MmaPeakShape;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_done = sbase + S::kBarOffset;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOffset);
    const int warp = threadIdx.x >> 5;
    const bool leader = cluster_ctarank() == 0;

    // operands: any bytes will do; zeros keep the accumulator exact
    for (int i = threadIdx.x; i < 2 * S::kTile / 16; i += S::kThreads)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(bar_done, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_u32(tmem_slot), S::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (leader && threadIdx.x == 0) {
        constexpr uint32_t idesc = idesc_i8(256, 256);
        const uint32_t as = sbase, bs = sbase + S::kTile;
        for (int64_t s = 0; s < steps; ++s) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                umma_i8_ss_pair(tmem_base, desc_kmajor_sw128(as + 32 * j), desc_kmajor_sw128(bs + 32 * j), idesc,
                                (s > 0 || j > 0) ? 1u : 0u);
        }
        umma_commit_pair(bar_done, 0x1);
        gemm_wait_drain(bar_done, 0);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // the pair's MMAs are complete before the memory is released
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, S::kTmemCols);
    }
}

}  // namespace quarot
