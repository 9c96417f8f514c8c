// mma_peak.cuh -- the ceiling that the INT4 and INT8 linear layers are
// measured against: the rate of dense tcgen05.mma.kind::i8 instructions of the
// shape those kernels use (CTA pairs, M 256, N 256, K 32, int32 accumulation
// in tensor memory), with both operands resident in shared memory, so nothing
// but the tensor pipe is timed.  No copies, no epilogue: the leader thread of
// every CTA pair issues `steps` groups of four MMAs (one 128-byte K block)
// into one accumulator and waits for them at the end; the results are never
// read.  One CTA per SM (the shared-memory request keeps a second one off).
//
// The operands are all zero, pseudo-random bytes, or pseudo-random 4-bit
// codes held in the high nibble of each byte (the form in which the INT4
// GEMMs hand their codes to the tensor core).  The work per clock is the same
// for all three, but the power drawn is not: nonzero operands toggle the
// multipliers as real data does, and under the board's power limit the SM
// clock, and with it the rate per second, settles lower than with zeros.
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

// MurmurHash3's 32-bit finalizer (Appleby): a bijective mix of a counter
// into well-spread bits, here only a source of operand bytes.
__device__ __forceinline__ uint32_t fmix32(uint32_t h)
{
    h ^= h >> 16;
    h *= 0x85ebca6bu;
    h ^= h >> 13;
    h *= 0xc2b2ae35u;
    h ^= h >> 16;
    return h;
}

__global__ void __launch_bounds__(MmaPeakShape::kThreads, 1)
mma_peak_i8_kernel(int64_t steps, int operands)
{
    using S = MmaPeakShape;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_done = sbase + S::kBarOffset;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOffset);
    const int warp = threadIdx.x >> 5;
    const bool leader = cluster_ctarank() == 0;

    // operands: zeros, or bytes mixed from (CTA, word index), optionally with
    // the low nibbles cleared; the int32 accumulation of random products
    // wraps, which nothing reads
    const uint32_t keep = operands == 2 ? 0xf0f0f0f0u : 0xffffffffu;
    for (int i = threadIdx.x; i < 2 * S::kTile / 16; i += S::kThreads) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (operands != 0) {
            const uint32_t c = (blockIdx.x * (2u * S::kTile / 16u) + (uint32_t)i) * 4u;
            v = make_uint4(fmix32(c + 1u) & keep, fmix32(c + 2u) & keep, fmix32(c + 3u) & keep,
                           fmix32(c + 4u) & keep);
        }
        reinterpret_cast<uint4 *>(smem)[i] = v;
    }
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
