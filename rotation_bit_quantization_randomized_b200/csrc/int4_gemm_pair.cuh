// int4_gemm_pair.cuh -- the per-token / per-channel INT4 linear layer on CTA
// pairs: tcgen05.mma.cta_group::2 computes 256 x 256 output tiles, each CTA of
// the pair holding 128 rows of A and 128 rows (its half of the N tile) of B.
//
// Same method and data flow as int4_gemm.cuh (TMA of packed tiles, nibble
// widening by unpack warps, int8 tensor-core MMA into tensor memory, fused
// dequantizing epilogue); what changes is that each SM now stages and widens
// half of the B tile instead of all of it, which cuts the shared-memory
// traffic per multiply-add by a third -- the kernel's bound.
//
// Pair protocol (CTA rank 0 = leader):
//  * each CTA's TMA producer fills its own packed ring; its unpack warps fill
//    its own int8 ring and, after a proxy fence, every unpack thread of both
//    CTAs arrives on the LEADER's "int8 stage full" barrier;
//  * the leader's MMA thread issues the pair MMAs and commits with a
//    multicast to the "stage empty" / "accumulator full" barriers of both
//    CTAs;
//  * each CTA's epilogue reads its own 128 accumulator rows and arrives on
//    the leader's "accumulator empty" barrier;
//  * a cluster barrier precedes the release of tensor memory, so neither CTA
//    leaves while its peer may still read its shared memory or signal it.
// All waits are bounded in time, as in the single-CTA kernel.
#pragma once

#include "int4_gemm.cuh"

namespace quarot {

constexpr int kPairBM = 256;       // output rows per CTA pair
constexpr int kPairBN = 256;       // output columns per CTA pair

template <int EPI>
struct PairShape {
    static constexpr int kRows = 128;                                 // A rows and B rows per CTA
    static constexpr int kPackedA = kRows * kGemmBK / 2;
    static constexpr int kPackedStage = 2 * kPackedA;
    static constexpr int kABytes = kRows * kGemmBK;
    static constexpr int kStageBytes = 2 * kABytes;
    static constexpr int kPStages = 4;
    static constexpr int kIStages = 4;
    static constexpr int kGroupsPerWarp = 8;
    static constexpr int kUnpackWarps = 2 * kRows / (8 * kGroupsPerWarp);   // 4
    static constexpr int kUnpackThreads = 32 * kUnpackWarps;
    static constexpr int kEpiWarps = 4;
    static constexpr int kMmaWarp = 4;
    static constexpr int kTmaWarp = 5;
    static constexpr int kUnpackWarp0 = 6;
    static constexpr int kThreads = 32 * (kUnpackWarp0 + kUnpackWarps);
    static constexpr int kTmemCols = 2 * kPairBN;                     // two accumulator buffers
    static constexpr int kIntOffset = kPStages * kPackedStage;
    static constexpr int kBarOffset = kIntOffset + kIStages * kStageBytes;
    static constexpr int kNumBars = 2 * kPStages + 2 * kIStages + 5;
    static constexpr int kMiscOffset = kBarOffset + 8 * kNumBars;
    static constexpr int kSmemBytes = kMiscOffset + 16 + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kStageBytes % 1024 == 0 && kIntOffset % 1024 == 0, "1024-byte aligned int8 stages");
};

template <int EPI>
__global__ void __launch_bounds__(PairShape<EPI>::kThreads, 1)
int4_gemm_pair_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tma_a,
                      const __grid_constant__ CUtensorMap tma_b)
{
    using S = PairShape<EPI>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_pfull = sbase + S::kBarOffset;
    const uint32_t bar_pempty = bar_pfull + 8 * S::kPStages;
    const uint32_t bar_ifull = bar_pempty + 8 * S::kPStages;       // used in the leader
    const uint32_t bar_iempty = bar_ifull + 8 * S::kIStages;
    const uint32_t bar_accf = bar_iempty + 8 * S::kIStages;
    const uint32_t bar_acce = bar_accf + 16;                       // used in the leader
    const uint32_t bar_drain = bar_acce + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + S::kMiscOffset + 4);

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
        for (int s = 0; s < S::kPStages; ++s) {
            mbar_init(bar_pfull + 8 * s, 1);
            mbar_init(bar_pempty + 8 * s, S::kUnpackThreads);
        }
        for (int s = 0; s < S::kIStages; ++s) {
            mbar_init(bar_ifull + 8 * s, 2 * S::kUnpackThreads);    // leader's: both CTAs' unpackers
            mbar_init(bar_iempty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_accf + 8 * b, 1);
            mbar_init(bar_acce + 8 * b, 2 * S::kEpiWarps);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == S::kMmaWarp) {
        tmem_alloc_pair(smem_u32(tmem_slot), S::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == S::kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tma_a);
            tma_prefetch_desc(&tma_b);
            int lt = 0, kb = 0, mb = 0, nb = 0;
            if (total > 0)
                gemm_tile_coords(cluster, a.tiles_m, a.tiles_n, mb, nb);
            int step = 0;
            for (; step < total; ++step) {
                const int ps = step % S::kPStages;
                const uint32_t use = (uint32_t)(step / S::kPStages);
                if (!gemm_wait(bar_pempty + 8 * ps, (use & 1) ^ 1, abort_flag))
                    break;
                const uint32_t dst = sbase + ps * S::kPackedStage;
                mbar_arrive_expect_tx(bar_pfull + 8 * ps, S::kPackedStage);
                tma_load_2d(dst, &tma_a, kb * (kGemmBK / 2), mb * kPairBM + S::kRows * rank, bar_pfull + 8 * ps);
                tma_load_2d(dst + S::kPackedA, &tma_b, kb * (kGemmBK / 2), nb * kPairBN + S::kRows * rank,
                            bar_pfull + 8 * ps);
                if (++kb == KB) {
                    kb = 0;
                    if (++lt < my_tiles)
                        gemm_tile_coords(cluster + lt * nclusters, a.tiles_m, a.tiles_n, mb, nb);
                }
            }
            for (int s = step - S::kPStages; s < step; ++s)
                if (s >= 0)
                    gemm_wait_drain(bar_pfull + 8 * (s % S::kPStages), (uint32_t)(s / S::kPStages) & 1);
        }
        __syncwarp();
    } else if (warp >= S::kUnpackWarp0) {
        // ------------------------------------------------------------ unpackers
        // warps 0-1 of this role widen the 128 A rows, warps 2-3 the 128 B rows;
        // lane (r, c) = (lane / 4, lane % 4) handles 16 packed bytes of row 8 g + r
        const int uw = warp - S::kUnpackWarp0;
        const int rsub = lane >> 2;
        const int csub = lane & 3;
        const int row0 = 8 * S::kGroupsPerWarp * uw;           // 0, 64 (A) or 128, 192 (B)
        const bool isA = row0 < S::kRows;
        const int tile_row0 = isA ? row0 : row0 - S::kRows;
        const uint32_t p_off = isA ? 0u : (uint32_t)S::kPackedA;
        const uint32_t i_off = isA ? 0u : (uint32_t)S::kABytes;
        for (int step = 0; step < total; ++step) {
            const int ps = step % S::kPStages;
            const int is = step % S::kIStages;
            if (!gemm_wait(bar_pfull + 8 * ps, (uint32_t)(step / S::kPStages) & 1, abort_flag))
                break;
            uint4 w[S::kGroupsPerWarp];
            const uint8_t *src = smem + ps * S::kPackedStage + p_off;
#pragma unroll
            for (int j = 0; j < S::kGroupsPerWarp; ++j) {
                const int r = tile_row0 + 8 * j + rsub;
                w[j] = *reinterpret_cast<const uint4 *>(src + r * (kGemmBK / 2) + csub * 16);
            }
            if (!gemm_wait(bar_iempty + 8 * is, ((uint32_t)(step / S::kIStages) & 1) ^ 1, abort_flag))
                break;
            uint8_t *st_base = smem + S::kIntOffset + is * S::kStageBytes + i_off;
#pragma unroll
            for (int j = 0; j < S::kGroupsPerWarp; ++j) {
                const int r = tile_row0 + 8 * j + rsub;
                uint8_t *dst = st_base + (r >> 3) * 1024 + (r & 7) * 128;
                const int sw = r & 7;
                const uint4 v = w[j];
                const uint4 lo = make_uint4((v.x << 4) & 0xF0F0F0F0u, (v.y << 4) & 0xF0F0F0F0u,
                                            (v.z << 4) & 0xF0F0F0F0u, (v.w << 4) & 0xF0F0F0F0u);
                const uint4 hi = make_uint4(v.x & 0xF0F0F0F0u, v.y & 0xF0F0F0F0u,
                                            v.z & 0xF0F0F0F0u, v.w & 0xF0F0F0F0u);
                *reinterpret_cast<uint4 *>(dst + (((2 * csub) ^ sw) << 4)) = lo;
                *reinterpret_cast<uint4 *>(dst + (((2 * csub + 1) ^ sw) << 4)) = hi;
            }
            // the int8 stage is complete and visible to the tensor core; the
            // packed stage's reads are complete (their values were stored)
            fence_proxy_async_smem();
            mbar_arrive_remote(mapa_shared(bar_ifull + 8 * is, 0));
            mbar_arrive(bar_pempty + 8 * ps);
        }
    } else if (warp == S::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kPairBM, kPairBN);
            bool ok = true;
            int step = 0;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                const int ab = lt & 1;
                if (!gemm_wait(bar_acce + 8 * ab, ((uint32_t)(lt >> 1) & 1) ^ 1, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + ab * kPairBN;
                for (int kb = 0; kb < KB; ++kb, ++step) {
                    const int is = step % S::kIStages;
                    if (!gemm_wait(bar_ifull + 8 * is, (uint32_t)(step / S::kIStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t as = sbase + S::kIntOffset + is * S::kStageBytes;
                    const uint32_t bs = as + S::kABytes;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_i8_ss_pair(d, desc_kmajor_sw128(as + 32 * j), desc_kmajor_sw128(bs + 32 * j), idesc,
                                        (kb > 0 || j > 0) ? 1u : 0u);
                    umma_commit_pair(bar_iempty + 8 * is, 0x3);
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
            const int64_t m = (int64_t)mb * kPairBM + S::kRows * rank + 32 * wq + lane;
            const int64_t n0 = (int64_t)nb * kPairBN;
            const bool mrow = m < a.M;
            const int ab = lt & 1;
            if (!gemm_wait(bar_accf + 8 * ab, (uint32_t)(lt >> 1) & 1, abort_flag))
                break;
            tc_fence_after();
            float sam = 0.f;
            if (EPI == kEpiScaledF16 && mrow)
                sam = reinterpret_cast<const float *>(a.sa)[m] * (1.0f / 256.0f);
#pragma unroll 1
            for (int c = 0; c < kPairBN / 32; ++c) {
                uint32_t r[32];
                __syncwarp();
                tmem_ld32(lane_addr + ab * kPairBN + 32 * c, r);
                tmem_wait_ld(r);
                if (c == kPairBN / 32 - 1) {
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
                            *reinterpret_cast<uint4 *>(orow + n) = make_uint4(h[0], h[1], h[2], h[3]);
                        }
                    }
                } else if (mrow) {
                    int32_t *orow = reinterpret_cast<int32_t *>(a.out) + m * a.N;
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const int64_t n = n0 + 32 * c + 4 * v;
                        if (n < a.N)
                            *reinterpret_cast<int4 *>(orow + n) =
                                make_int4((int)r[4 * v] >> 8, (int)r[4 * v + 1] >> 8, (int)r[4 * v + 2] >> 8,
                                          (int)r[4 * v + 3] >> 8);
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
