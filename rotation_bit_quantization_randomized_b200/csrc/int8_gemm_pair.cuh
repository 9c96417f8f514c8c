// int8_gemm_pair.cuh -- the 8-bit variant of the linear layer: INT8 x INT8
// codes (one signed byte each), int32 accumulation on the tensor cores and the
// same dequantizing epilogue (QuaRot abstract: higher code widths of the same
// round-to-nearest recipe; QuaRot summary: products in integers).
//
//   acc[m, n] = sum_k qa[m, k] qw[n, k]            (|acc| <= 2^14 K < 2^31)
//   out[m, n] = fp16(acc * s_a[m] * s_w[n])
//
// The codes are already bytes, so no thread touches the operands: this is a
// pure copy-engine -> tensor-core pipeline on CTA pairs.
//  * Tiles of 256 x 256 outputs per CTA pair (tcgen05.mma.cta_group::2,
//    kind::i8, M 256, N 256, K 32); each CTA holds 128 rows of A and its 128
//    rows (half of the N tile) of B, K step 128.
//  * One TMA thread per CTA copies its A and B boxes (128 rows x 128 bytes,
//    128-byte swizzle: exactly the K-major layout the MMA reads) into a ring
//    of stages.  Both CTAs' copies complete their bytes on the LEADER's
//    "stage full" barrier (the copies carry the cta_group::2 qualifier so
//    that the barrier may sit in the peer CTA); only the leader's producer
//    arrives on it, declaring the bytes of both CTAs.  No copy is multicast.
//  * The leader's MMA thread waits for a full stage, issues four MMAs and
//    commits with a multicast to both CTAs' "stage empty" barriers, and at
//    the end of a tile to their "accumulator full" barriers.  Two 256-column
//    accumulators in tensor memory let the epilogue of one tile overlap the
//    next tile.
//  * Each CTA's four epilogue warps read their 128 accumulator rows, scale
//    and store fp16 (or store the int32 sums), and arrive on the leader's
//    "accumulator empty" barrier.
//  * Every wait is bounded in time, as in the INT4 kernels.
#pragma once

#include "int4_gemm.cuh"

namespace quarot {

constexpr int kI8PairBM = 256;
constexpr int kI8PairBN = 256;

struct I8PairShape {
    static constexpr int kRows = 128;                            // A rows and B rows per CTA
    static constexpr int kTileBytes = kRows * kGemmBK;           // 16 KB, one operand box
    static constexpr int kStageBytes = 2 * kTileBytes;           // A then B
    static constexpr int kStages = 6;
    static constexpr int kEpiWarps = 4;
    static constexpr int kMmaWarp = 4;
    static constexpr int kTmaWarp = 5;
    static constexpr int kThreads = 32 * 6;
    static constexpr int kTmemCols = 2 * kI8PairBN;
    static constexpr int kBarOffset = kStages * kStageBytes;
    static constexpr int kNumBars = 2 * kStages + 5;
    static constexpr int kMiscOffset = kBarOffset + 8 * kNumBars;
    static constexpr int kSmemBytes = kMiscOffset + 16 + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kStageBytes % 1024 == 0, "1024-byte aligned stages for the 128-byte swizzle");
};

// Tiled 2-D copy into this CTA's shared memory whose transaction bytes are
// counted on the mbarrier at shared::cluster address `bar_cluster` (this
// CTA's or its pair peer's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void *tmap, int x, int y, uint32_t bar_cluster)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}

template <int EPI>
__global__ void __launch_bounds__(I8PairShape::kThreads, 1)
int8_gemm_pair_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tma_a,
                      const __grid_constant__ CUtensorMap tma_b)
{
    using S = I8PairShape;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + S::kBarOffset;              // used in the leader
    const uint32_t bar_empty = bar_full + 8 * S::kStages;
    const uint32_t bar_accf = bar_empty + 8 * S::kStages;
    const uint32_t bar_acce = bar_accf + 16;                      // used in the leader
    const uint32_t bar_drain = bar_acce + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + S::kMiscOffset + 4);
    int *peer_steps = reinterpret_cast<int *>(smem + S::kMiscOffset + 8);   // leader: steps the peer issued

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1;
    const int nclusters = gridDim.x >> 1;
    const int num_tiles = a.tiles_m * a.tiles_n;
    const int KB = a.kblocks;
    const int my_tiles = cluster < num_tiles ? (num_tiles - 1 - cluster) / nclusters + 1 : 0;
    const int total = my_tiles * KB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S::kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);                        // the leader's producer only
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_accf + 8 * b, 1);
            mbar_init(bar_acce + 8 * b, 2 * S::kEpiWarps);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        *peer_steps = -1;
        mbar_fence_init();
    }
    if (warp == S::kMmaWarp) {
        tmem_alloc_pair(smem_u32(tmem_slot), S::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // both CTAs' barriers exist before any remote signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == S::kTmaWarp) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&tma_a);
            tma_prefetch_desc(&tma_b);
            int lt = 0, kb = 0, mb = 0, nb = 0;
            if (total > 0)
                gemm_tile_coords(cluster, a.tiles_m, a.tiles_n, mb, nb);
            int step = 0;
            for (; step < total; ++step) {
                const int s = step % S::kStages;
                const uint32_t use = (uint32_t)(step / S::kStages);
                if (!gemm_wait(bar_empty + 8 * s, (use & 1) ^ 1, abort_flag))
                    break;
                const uint32_t full_leader = mapa_shared(bar_full + 8 * s, 0);
                if (leader)
                    mbar_arrive_expect_tx(bar_full + 8 * s, 2 * S::kStageBytes);
                const uint32_t dst = sbase + s * S::kStageBytes;
                tma_load_2d_pair(dst, &tma_a, kb * kGemmBK, mb * kI8PairBM + S::kRows * rank, full_leader);
                tma_load_2d_pair(dst + S::kTileBytes, &tma_b, kb * kGemmBK, nb * kI8PairBN + S::kRows * rank,
                                 full_leader);
                if (++kb == KB) {
                    kb = 0;
                    if (++lt < my_tiles)
                        gemm_tile_coords(cluster + lt * nclusters, a.tiles_m, a.tiles_n, mb, nb);
                }
            }
            // Every copy either CTA issued lands before the pair passes the
            // final cluster barrier.  All of them count on the leader's stage
            // barriers, so the peer reports how many steps it issued and the
            // leader waits for the last kStages steps of either CTA (earlier
            // ones were consumed before their stages were refilled).  In a
            // normal run both issued every step and those phases are complete.
            // After an abort the two counts may differ: a step only the peer
            // issued gets the leader's missing arrival (declaring the peer's
            // bytes), a step only the leader issued gets the peer's declared
            // bytes completed without a copy, so each phase completes once the
            // copies actually issued have landed.
            if (!leader) {
                st_release_cluster_u32(mapa_shared(smem_u32(peer_steps), 0), (uint32_t)step);
            } else {
                int peer = -1;
                const uint64_t t0 = globaltimer_ns();
                while ((peer = (int)ld_acquire_cluster_u32(smem_u32(peer_steps))) < 0) {
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        record_timeout();
                        break;
                    }
                }
                if (peer >= 0) {
                    const int hi = max(step, peer);
                    for (int j = max(0, hi - S::kStages); j < hi; ++j) {
                        const uint32_t fb = bar_full + 8 * (j % S::kStages);
                        if (j >= step)
                            mbar_arrive_expect_tx(fb, S::kStageBytes);
                        else if (j >= peer)
                            mbar_complete_tx(fb, S::kStageBytes);
                        gemm_wait_drain(fb, (uint32_t)(j / S::kStages) & 1);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == S::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kI8PairBM, kI8PairBN);
            bool ok = true;
            int step = 0;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                const int ab = lt & 1;
                if (!gemm_wait(bar_acce + 8 * ab, ((uint32_t)(lt >> 1) & 1) ^ 1, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + ab * kI8PairBN;
                for (int kb = 0; kb < KB; ++kb, ++step) {
                    const int s = step % S::kStages;
                    if (!gemm_wait(bar_full + 8 * s, (uint32_t)(step / S::kStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t as = sbase + s * S::kStageBytes;
                    const uint32_t bs = as + S::kTileBytes;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_i8_ss_pair(d, desc_kmajor_sw128(as + 32 * j), desc_kmajor_sw128(bs + 32 * j), idesc,
                                        (kb > 0 || j > 0) ? 1u : 0u);
                    umma_commit_pair(bar_empty + 8 * s, 0x3);
                    if (kb == KB - 1)
                        umma_commit_pair(bar_accf + 8 * ab, 0x3);
                }
            }
            umma_commit_pair(bar_drain, 0x1);
            gemm_wait_drain(bar_drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int wq = warp & 3;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * wq) << 16);
        for (int lt = 0; lt < my_tiles; ++lt) {
            int mb, nb;
            gemm_tile_coords(cluster + lt * nclusters, a.tiles_m, a.tiles_n, mb, nb);
            const int64_t m = (int64_t)mb * kI8PairBM + S::kRows * rank + 32 * wq + lane;
            const int64_t n0 = (int64_t)nb * kI8PairBN;
            const bool mrow = m < a.M;
            const int ab = lt & 1;
            if (!gemm_wait_warp(bar_accf + 8 * ab, (uint32_t)(lt >> 1) & 1, abort_flag))
                break;
            tc_fence_after();
            float sam = 0.f;
            if (EPI == kEpiScaledF16 && mrow)
                sam = reinterpret_cast<const float *>(a.sa)[m];
#pragma unroll 1
            for (int c = 0; c < kI8PairBN / 32; ++c) {
                uint32_t r[32];
                __syncwarp();
                tmem_ld32(lane_addr + ab * kI8PairBN + 32 * c, r);
                tmem_wait_ld(r);
                if (c == kI8PairBN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive_remote(mapa_shared(bar_acce + 8 * ab, 0));
                }
                if (mrow && EPI == kEpiScaledF16) {
                    __half *orow = reinterpret_cast<__half *>(a.out) + m * a.N;
                    const float *swp = reinterpret_cast<const float *>(a.sw);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int64_t n = n0 + 32 * c + 8 * v;
                        if (n < a.N) {
                            const float4 w0 = __ldg(reinterpret_cast<const float4 *>(swp + n));
                            const float4 w1 = __ldg(reinterpret_cast<const float4 *>(swp + n + 4));
                            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                            uint32_t h[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float f0 = __int2float_rn((int)r[8 * v + 2 * i]) * sam * wv[2 * i];
                                const float f1 = __int2float_rn((int)r[8 * v + 2 * i + 1]) * sam * wv[2 * i + 1];
                                h[i] = h2_as_u32(__floats2half2_rn(f0, f1));
                            }
                            if (QUAROT_IN_RANGE(orow + n, 16, a.out, a.M * a.N * 2))
                                *reinterpret_cast<uint4 *>(orow + n) = make_uint4(h[0], h[1], h[2], h[3]);
                        }
                    }
                } else if (mrow) {
                    int32_t *orow = reinterpret_cast<int32_t *>(a.out) + m * a.N;
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const int64_t n = n0 + 32 * c + 4 * v;
                        if (n < a.N && QUAROT_IN_RANGE(orow + n, 16, a.out, a.M * a.N * 4))
                            *reinterpret_cast<int4 *>(orow + n) =
                                make_int4((int)r[4 * v], (int)r[4 * v + 1], (int)r[4 * v + 2], (int)r[4 * v + 3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // the peer no longer reads this CTA's memory or signals it
    if (warp == S::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, S::kTmemCols);
    }
}

}  // namespace quarot
