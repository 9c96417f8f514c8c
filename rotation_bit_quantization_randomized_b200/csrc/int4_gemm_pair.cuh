// int4_gemm_pair.cuh -- the per-token / per-channel INT4 linear layer on CTA
// pairs: tcgen05.mma.cta_group::2 computes 256 x BN output tiles; each CTA of
// the pair holds 128 rows of A and BN/2 rows (its half of the N tile) of B.
//
// Same method as int4_gemm.cuh (TMA of packed tiles, nibble widening, int8
// tensor-core MMA with int32 accumulation in tensor memory, fused
// dequantizing epilogue).  The kernel is bound by shared-memory bandwidth, so
// the operands take different routes:
//  * A (activations): each unpack thread owns one A row; it reads the row's
//    64 packed bytes (the TMA writes them with the 64-byte swizzle, so the
//    per-row reads of a warp hit distinct banks), widens them in registers
//    and writes the 128 int8 values straight into tensor memory with
//    tcgen05.st (lane = row).  The MMA reads A from tensor memory: A never
//    passes through shared memory in widened form.
//  * B (weights): widened into the 128-byte-swizzled K-major shared-memory
//    stage the MMA reads, as in the single-CTA kernel, but only the CTA's
//    half of the N tile.
//
// Tensor memory (512 columns per CTA): two accumulator buffers of BN columns
// at 0 and BN, then the int8 A stages of 32 columns (128 K values) each; the
// number of stages is what the remaining columns hold.
//
// Stages: a ring of 8 packed stages (TMA -> unpackers), 4 int8 B stages in
// shared memory and kAStages = (512 - 2 BN) / 32 int8 A stages in tensor
// memory.  Two groups of four unpack warps take alternate K steps.  A group
// reads and widens step s, stores its B half as soon as the MMAs of step
// s - 4 are done, and only then waits for the MMAs of step s - kAStages to
// free its A stage: after that wait comes nothing but the tensor-memory store
// and the arrival, so the stage hand-off the tensor core waits on is short.
//
// Pair protocol (CTA rank 0 = leader):
//  * each CTA's TMA producer fills its own packed ring; its unpack warps fill
//    its own A stage (tensor memory) and B stage (shared memory) and, after
//    the store waits, fences and a warp barrier, lane 0 of every unpack warp
//    of both CTAs arrives on the LEADER's "int8 stage full" barrier;
//  * the leader's MMA thread issues the pair MMAs and commits with a
//    multicast to the "step done" / "accumulator full" barriers of both
//    CTAs (MMAs complete in order, so "step s done" also frees the stages of
//    every earlier step);
//  * each CTA's epilogue reads its own 128 accumulator rows and arrives on
//    the leader's "accumulator empty" barrier;
//  * a cluster barrier precedes the release of tensor memory, so neither CTA
//    leaves while its peer may still read its memory or signal it.
// All waits are bounded in time, as in the single-CTA kernel; waits in front
// of warp-collective tcgen05 instructions are warp-uniform.
//
// Grouped scales (EPI == kEpiGroupF16, 128-wide K groups, N tile 128 per
// pair): every K step is its own int32 accumulation, into one of three
// 128-column accumulators that rotate step by step (four A stages fill the
// rest of tensor memory); eight epilogue warps per CTA (two per lane
// quarter, 64 columns each) read each step's partial sums, convert them
// exactly, scale them by the step's row and column scales (staged in shared
// memory eight groups at a time) and accumulate in fp32 registers; the MMA
// thread waits for an accumulator's previous partial sums to be read before
// it starts the next step in it.
#pragma once

#include "int4_gemm.cuh"

namespace quarot {

constexpr int kPairBM = 256;       // output rows per CTA pair

template <int BN, int EPI>
struct PairShape {
    static constexpr bool kGrouped = EPI == kEpiGroupF16;
    static constexpr int kRowsA = kPairBM / 2;                        // A rows per CTA
    static constexpr int kRowsB = BN / 2;                             // B rows per CTA
    static constexpr int kPackedA = kRowsA * kGemmBK / 2;             // 8 KB, 64-byte swizzled
    static constexpr int kPackedB = kRowsB * kGemmBK / 2;
    static constexpr int kPackedStage = kPackedA + kPackedB;
    static constexpr int kBBytes = kRowsB * kGemmBK;                  // widened B stage
    static constexpr int kTmemCols = 512;
    static constexpr int kAccBufs = kGrouped ? 3 : 2;                // accumulators of BN columns
    static constexpr int kAStages = (kTmemCols - kAccBufs * BN) / 32; // int8 A stages in tensor memory
    static constexpr int kBStages = 4;                                // int8 B stages in shared memory
    static constexpr int kPStages = 8;
    static constexpr int kBGroups = kRowsB / 8;                       // groups of 8 B rows
    static constexpr int kUnpackWarps = 4;                            // per group: one per TMEM lane quarter
    // groups take alternate K steps; the grouped kernel keeps one, because its
    // eight epilogue warps hold 64 fp32 sums each and 18 warps would leave
    // them too few registers (measured: 2.40 ms with one group against 2.79
    // ms with two, which spill, at 4096 x 28672 x 8192)
    static constexpr int kUnpackGroups = kGrouped ? 1 : 2;
    static constexpr int kBGroupsPerWarp = (kBGroups + kUnpackWarps - 1) / kUnpackWarps;
    static constexpr int kUnpackArrivals = kUnpackWarps;              // one arrival per warp and stage
    static constexpr int kEpiWarps = kGrouped ? 8 : 4;
    static constexpr int kEpiThreads = 32 * kEpiWarps;
    static constexpr int kMmaWarp = kEpiWarps;
    static constexpr int kTmaWarp = kEpiWarps + 1;
    static constexpr int kUnpackWarp0 = kEpiWarps + 2;
    static constexpr int kThreads = 32 * (kUnpackWarp0 + kUnpackGroups * kUnpackWarps);
    static constexpr int kACol0 = kAccBufs * BN;                      // A stage s at kACol0 + 32 s
    static constexpr int kIntOffset = kPStages * kPackedStage;
    static constexpr int kBarOffset = kIntOffset + kBStages * kBBytes;
    static constexpr int kNumBars = 2 * kPStages + 2 * kBStages + 2 * kAccBufs + 1;
    static constexpr int kMiscOffset = kBarOffset + 8 * kNumBars;
    static constexpr int kGroupChunk = 8;                             // K groups per staged scale chunk
    static constexpr int kSwOffset = kMiscOffset + 16;                // grouped: [2][8][128] row, [2][8][BN] column scales
    static constexpr int kSmemBytes = kSwOffset + (kGrouped ? 2 * kGroupChunk * (kRowsA + BN) * 4 : 0) + 1024;
    static_assert(!kGrouped || (BN == 128 && kEpiThreads == kRowsA + BN),
                  "grouped: N tile 128, one scale-staging thread per tile row and column");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kPackedStage % 1024 == 0 && kBBytes % 1024 == 0, "1024-byte aligned stages");
    static_assert(kRowsB % 8 == 0 && BN % 32 == 0 && BN <= 256, "B rows in groups of 8; N tile of whole column chunks");
    static_assert(kAStages >= kUnpackGroups && kACol0 + 32 * kAStages <= kTmemCols, "tensor-memory plan");
    static_assert(kBStages >= kAStages && kBStages % kAStages == 0, "an A stage is free once its B stage is");
    static_assert(kPStages % kUnpackGroups == 0 && kBStages % kUnpackGroups == 0,
                  "each stage barrier is used by one unpack group");
};

// UNS: the codes are unsigned nibbles (asymmetric quantization): they are
// widened to the byte values 0..15 and multiplied as unsigned 8-bit.
template <int BN, int EPI, bool UNS = false>
__global__ void __launch_bounds__(PairShape<BN, EPI>::kThreads, 1)
int4_gemm_pair_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tma_a,
                      const __grid_constant__ CUtensorMap tma_b)
{
    using S = PairShape<BN, EPI>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_pfull = sbase + S::kBarOffset;
    const uint32_t bar_pempty = bar_pfull + 8 * S::kPStages;
    const uint32_t bar_ifull = bar_pempty + 8 * S::kPStages;       // used in the leader
    const uint32_t bar_sdone = bar_ifull + 8 * S::kBStages;        // MMAs of step s done (slot s % kBStages)
    const uint32_t bar_accf = bar_sdone + 8 * S::kBStages;
    const uint32_t bar_acce = bar_accf + 8 * S::kAccBufs;          // used in the leader
    const uint32_t bar_drain = bar_acce + 8 * S::kAccBufs;
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
            mbar_init(bar_pempty + 8 * s, S::kUnpackArrivals);
        }
        for (int s = 0; s < S::kBStages; ++s) {
            mbar_init(bar_ifull + 8 * s, 2 * S::kUnpackArrivals);   // leader's: both CTAs' unpackers
            mbar_init(bar_sdone + 8 * s, 1);
        }
        for (int b = 0; b < S::kAccBufs; ++b) {
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
                tma_load_2d(dst, &tma_a, kb * (kGemmBK / 2), mb * kPairBM + S::kRowsA * rank, bar_pfull + 8 * ps);
                tma_load_2d(dst + S::kPackedA, &tma_b, kb * (kGemmBK / 2), nb * BN + S::kRowsB * rank,
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
        // Group h takes the K steps h, h + kUnpackGroups, ...  Within a group,
        // A: thread = A row 32 q + lane of TMEM lane quarter q = warp % 4;
        // B: warp u widens the 8-row groups u, u + 4, ...; lane (r, c) =
        // (lane / 4, lane % 4) handles 16 packed bytes of row 8 g + r.
        const int uw = (warp - S::kUnpackWarp0) % S::kUnpackWarps;
        const int ugroup = (warp - S::kUnpackWarp0) / S::kUnpackWarps;
        const int q = warp & 3;
        const int ra = 32 * q + lane;
        const int aswz = (ra >> 1) & 3;                    // 64-byte swizzle of packed row ra
        const int rsub = lane >> 2;
        const int csub = lane & 3;
        const uint32_t a_lane = tmem_base + ((uint32_t)(32 * q) << 16) + S::kACol0;
        for (int step = ugroup; step < total; step += S::kUnpackGroups) {
            const int ps = step % S::kPStages;
            const int bs = step % S::kBStages;
            const int as = step % S::kAStages;
            if (!gemm_wait_warp(bar_pfull + 8 * ps, (uint32_t)(step / S::kPStages) & 1, abort_flag))
                break;
            const uint8_t *src = smem + ps * S::kPackedStage;
            uint4 wa[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                wa[c] = *reinterpret_cast<const uint4 *>(src + ra * (kGemmBK / 2) + ((c ^ aswz) << 4));
            uint4 wb[S::kBGroupsPerWarp];
#pragma unroll
            for (int j = 0; j < S::kBGroupsPerWarp; ++j) {
                const int g = uw + S::kUnpackWarps * j;
                if (g < S::kBGroups)
                    wb[j] = *reinterpret_cast<const uint4 *>(src + S::kPackedA + (8 * g + rsub) * (kGemmBK / 2) +
                                                             csub * 16);
            }
            // A row: packed word i of chunk c holds codes 32 c + [8 i, 8 i + 8);
            // column 8 c + i gets their low nibbles, column 8 c + 4 + i the high
            // ones -- the order the B stage uses within each 32-wide K chunk
            uint32_t av[32];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t w4[4] = {wa[c].x, wa[c].y, wa[c].z, wa[c].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    av[8 * c + i] = UNS ? (w4[i] & 0x0F0F0F0Fu) : ((w4[i] << 4) & 0xF0F0F0F0u);
                    av[8 * c + 4 + i] = UNS ? ((w4[i] >> 4) & 0x0F0F0F0Fu) : (w4[i] & 0xF0F0F0F0u);
                }
            }
            // B stage bs is free once the MMAs of step - kBStages are done
            if (!gemm_wait_warp(bar_sdone + 8 * bs, ((uint32_t)(step / S::kBStages) & 1) ^ 1, abort_flag))
                break;
            uint8_t *st_base = smem + S::kIntOffset + bs * S::kBBytes;
#pragma unroll
            for (int j = 0; j < S::kBGroupsPerWarp; ++j) {
                const int g = uw + S::kUnpackWarps * j;
                if (g < S::kBGroups) {
                    const int r = 8 * g + rsub;
                    uint8_t *dst = st_base + g * 1024 + rsub * 128;
                    const uint4 v = wb[j];
                    const uint4 lo = UNS ? make_uint4(v.x & 0x0F0F0F0Fu, v.y & 0x0F0F0F0Fu, v.z & 0x0F0F0F0Fu,
                                                      v.w & 0x0F0F0F0Fu)
                                         : make_uint4((v.x << 4) & 0xF0F0F0F0u, (v.y << 4) & 0xF0F0F0F0u,
                                                      (v.z << 4) & 0xF0F0F0F0u, (v.w << 4) & 0xF0F0F0F0u);
                    const uint4 hi = UNS ? make_uint4((v.x >> 4) & 0x0F0F0F0Fu, (v.y >> 4) & 0x0F0F0F0Fu,
                                                      (v.z >> 4) & 0x0F0F0F0Fu, (v.w >> 4) & 0x0F0F0F0Fu)
                                         : make_uint4(v.x & 0xF0F0F0F0u, v.y & 0xF0F0F0F0u, v.z & 0xF0F0F0F0u,
                                                      v.w & 0xF0F0F0F0u);
                    *reinterpret_cast<uint4 *>(dst + (((2 * csub) ^ (r & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4 *>(dst + (((2 * csub + 1) ^ (r & 7)) << 4)) = hi;
                }
            }
            fence_proxy_async_smem();
            // A stage as is free once the MMAs of step - kAStages are done (MMAs
            // complete in order, so that step's "done" barrier says so); this
            // wait is the only one on the tensor core's critical path, and only
            // the tensor-memory store follows it
            if (step >= S::kAStages) {
                const int prev = step - S::kAStages;
                if (!gemm_wait_warp(bar_sdone + 8 * (prev % S::kBStages), (uint32_t)(prev / S::kBStages) & 1,
                                    abort_flag))
                    break;
            }
            tc_fence_after();
            tmem_st32(a_lane + (uint32_t)(32 * as), av);
            // every lane's part of the int8 stage is complete and visible to the
            // tensor core, and every value read from the packed stage has been
            // consumed by a store; the warp barrier orders all lanes' writes
            // before lane 0's arrivals
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_remote(mapa_shared(bar_ifull + 8 * bs, 0));
                mbar_arrive(bar_pempty + 8 * ps);
            }
        }
    } else if (warp == S::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kPairBM, BN, UNS);
            bool ok = true;
            int step = 0;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                const int ab = lt & 1;
                if (!S::kGrouped && !gemm_wait(bar_acce + 8 * ab, ((uint32_t)(lt >> 1) & 1) ^ 1, abort_flag))
                    break;
                tc_fence_after();
                uint32_t d = tmem_base + ab * BN;
                for (int kb = 0; kb < KB; ++kb, ++step) {
                    if (S::kGrouped) {
                        // step's own accumulator: free once the epilogue has read
                        // the partial sums of step - kAccBufs
                        const int gb = step % S::kAccBufs;
                        if (!gemm_wait(bar_acce + 8 * gb, ((uint32_t)(step / S::kAccBufs) & 1) ^ 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        d = tmem_base + gb * BN;
                    }
                    const int bsi = step % S::kBStages;
                    if (!gemm_wait(bar_ifull + 8 * bsi, (uint32_t)(step / S::kBStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t at = tmem_base + S::kACol0 + 32 * (step % S::kAStages);
                    const uint32_t bs = sbase + S::kIntOffset + bsi * S::kBBytes;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        umma_i8_ts_pair(d, at + 8 * j, desc_kmajor_sw128(bs + 32 * j), idesc,
                                        ((!S::kGrouped && kb > 0) || j > 0) ? 1u : 0u);
                    umma_commit_pair(bar_sdone + 8 * bsi, 0x3);
                    if (S::kGrouped)
                        umma_commit_pair(bar_accf + 8 * (step % S::kAccBufs), 0x3);
                    else if (kb == KB - 1)
                        umma_commit_pair(bar_accf + 8 * ab, 0x3);
                }
            }
            umma_commit_pair(bar_drain, 0x1);
            gemm_wait_drain(bar_drain, 0);
        }
        __syncwarp();
    } else if constexpr (S::kGrouped) {
        // ------------------------------------------------------------ grouped epilogue (both CTAs)
        // Warps w and w + 4 share TMEM lane quarter w % 4 and split the 128
        // columns.  The row and column scales of 8 K groups at a time are
        // staged in shared memory one chunk ahead (threads 0-127: this CTA's
        // 128 rows, 128-255: the tile's 128 columns); a named barrier of the
        // epilogue warps hands each chunk over and makes every thread's
        // decision to go on (or to give up after a timeout) the same.
        constexpr int kCh = S::kGroupChunk;
        constexpr int HALF = BN / 2;
        const int wq = warp & 3;
        const int col0 = (warp >> 2) * HALF;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * wq) << 16);
        const int et = threadIdx.x;                         // 0 .. kEpiThreads - 1
        const int G = KB;
        float *sac = reinterpret_cast<float *>(smem + S::kSwOffset);       // [2][kCh][kRowsA]
        float *swc = sac + 2 * kCh * S::kRowsA;                            // [2][kCh][BN]
        const bool is_row = et < S::kRowsA;
        const float smul = is_row ? (1.0f / 256.0f) : 1.0f;                // both operands are 16 x code
        bool ok = true;
        int step = 0;
        for (int lt = 0; lt < my_tiles && ok; ++lt) {
            int mb, nb;
            gemm_tile_coords(cluster + lt * nclusters, a.tiles_m, a.tiles_n, mb, nb);
            const int64_t mrow0 = (int64_t)mb * kPairBM + S::kRowsA * rank;
            const int64_t m = mrow0 + 32 * wq + lane;
            const int64_t n0 = (int64_t)nb * BN;
            const bool mrow = m < a.M;
            const int64_t srow = is_row ? mrow0 + et : n0 + (et - S::kRowsA);
            const bool sval = is_row ? srow < a.M : srow < a.N;
            const __half *sptr = reinterpret_cast<const __half *>(is_row ? a.sa : a.sw) + (sval ? srow : 0) * G;
            auto load_chunk = [&](int kb0, float (&d)[kCh]) {
                if (sval && G % kCh == 0) {
                    const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(sptr + kb0));
                    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 f = half2_bits_to_float2(w4[i]);
                        d[2 * i] = f.x * smul;
                        d[2 * i + 1] = f.y * smul;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < kCh; ++i)
                        d[i] = (sval && kb0 + i < G) ? __half2float(sptr[kb0 + i]) * smul : 0.f;
                }
            };
            auto store_chunk = [&](int cb, const float (&d)[kCh]) {
#pragma unroll
                for (int i = 0; i < kCh; ++i) {
                    if (is_row)
                        sac[(cb * kCh + i) * S::kRowsA + et] = d[i];
                    else
                        swc[(cb * kCh + i) * BN + (et - S::kRowsA)] = d[i];
                }
            };
            float accv[HALF];
#pragma unroll
            for (int i = 0; i < HALF; ++i)
                accv[i] = 0.f;
            {
                float d[kCh];
                load_chunk(0, d);
                store_chunk(0, d);
            }
            for (int kb0 = 0; kb0 < KB; kb0 += kCh) {
                const int cb = (kb0 / kCh) & 1;
                ok = epi_barrier_and(S::kEpiThreads, ok);
                if (!ok)
                    break;
                float nxt[kCh];
                if (kb0 + kCh < KB)
                    load_chunk(kb0 + kCh, nxt);
                const int nu = min(kCh, KB - kb0);
                for (int u = 0; u < nu; ++u, ++step) {
                    const int gb = step % S::kAccBufs;
                    if (!gemm_wait_warp(bar_accf + 8 * gb, (uint32_t)(step / S::kAccBufs) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const float sag = sac[(cb * kCh + u) * S::kRowsA + 32 * wq + lane];
                    const float *sws = swc + (cb * kCh + u) * BN;
#pragma unroll
                    for (int c = 0; c < HALF / 16; ++c) {
                        uint32_t r[16];
                        __syncwarp();
                        tmem_ld16(lane_addr + gb * BN + col0 + 16 * c, r);
                        tmem_wait_ld16(r);
                        if (c == HALF / 16 - 1) {
                            // both CTAs' 8 warps arrive on the leader's barrier
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0)
                                mbar_arrive_remote(mapa_shared(bar_acce + 8 * gb, 0));
                        }
                        // two partial sums at a time: exact int -> float with one
                        // packed subtract (|acc| < 2^22), times the column scales,
                        // then accumulated with the row scale by one packed FMA
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            float f0, f1;
                            sub_x2(__uint_as_float(r[i] + 0x4B400000u), __uint_as_float(r[i + 1] + 0x4B400000u),
                                   12582912.0f, f0, f1);
                            const float2 w = *reinterpret_cast<const float2 *>(sws + col0 + 16 * c + i);
                            mul_x2(f0, f1, w.x, w.y, f0, f1);
                            fma_x2_acc(f0, f1, sag, accv[16 * c + i], accv[16 * c + i + 1]);
                        }
                    }
                }
                if (kb0 + kCh < KB)
                    store_chunk(cb ^ 1, nxt);
            }
            ok = epi_barrier_and(S::kEpiThreads, ok);
            if (!ok)
                break;
            if (mrow) {
                __half *orow = reinterpret_cast<__half *>(a.out) + m * a.N;
#pragma unroll
                for (int v = 0; v < HALF / 8; ++v) {
                    const int64_t n = n0 + col0 + 8 * v;
                    if (n < a.N) {
                        uint32_t h[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            h[i] = h2_as_u32(__floats2half2_rn(accv[8 * v + 2 * i], accv[8 * v + 2 * i + 1]));
                        if (QUAROT_IN_RANGE(orow + n, 16, a.out, a.M * a.N * 2))
                            *reinterpret_cast<uint4 *>(orow + n) = make_uint4(h[0], h[1], h[2], h[3]);
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int wq = warp & 3;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * wq) << 16);
        for (int lt = 0; lt < my_tiles; ++lt) {
            int mb, nb;
            gemm_tile_coords(cluster + lt * nclusters, a.tiles_m, a.tiles_n, mb, nb);
            const int64_t m = (int64_t)mb * kPairBM + S::kRowsA * rank + 32 * wq + lane;
            const int64_t n0 = (int64_t)nb * BN;
            const bool mrow = m < a.M;
            const int ab = lt & 1;
            if (!gemm_wait_warp(bar_accf + 8 * ab, (uint32_t)(lt >> 1) & 1, abort_flag))
                break;
            tc_fence_after();
            float sam = 0.f;
            int32_t zam = 0, ram = 0;
            if (EPI == kEpiScaledF16 && mrow)
                sam = reinterpret_cast<const float *>(a.sa)[m] * (1.0f / 256.0f);
            if (EPI == kEpiAsymF16 && mrow) {
                sam = reinterpret_cast<const float *>(a.sa)[m];
                zam = a.za[m];
                ram = a.ra[m];
            }
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                __syncwarp();
                tmem_ld32(lane_addr + ab * BN + 32 * c, r);
                tmem_wait_ld(r);
                if (c == BN / 32 - 1) {
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
                } else if (mrow && EPI == kEpiAsymF16) {
                    // y = da dw (acc - zw ra - za rw + K za zw): the bracket is formed
                    // exactly in 64-bit integers (zero points are not bounded by the
                    // code width), then converted and scaled
                    __half *orow = reinterpret_cast<__half *>(a.out) + m * a.N;
                    const float *swp = reinterpret_cast<const float *>(a.sw);
                    const int64_t kz = a.K * (int64_t)zam;
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int64_t n = n0 + 32 * c + 8 * v;
                        if (n < a.N) {
                            const float4 w0 = __ldg(reinterpret_cast<const float4 *>(swp + n));
                            const float4 w1 = __ldg(reinterpret_cast<const float4 *>(swp + n + 4));
                            const int4 z0 = __ldg(reinterpret_cast<const int4 *>(a.zw + n));
                            const int4 z1 = __ldg(reinterpret_cast<const int4 *>(a.zw + n + 4));
                            const int4 s0 = __ldg(reinterpret_cast<const int4 *>(a.rw + n));
                            const int4 s1 = __ldg(reinterpret_cast<const int4 *>(a.rw + n + 4));
                            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                            const int32_t zv[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
                            const int32_t sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
                            uint32_t h[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                float f[2];
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const int k = 2 * i + e;
                                    const int64_t br = (int64_t)(int32_t)r[8 * v + k] - (int64_t)zv[k] * ram -
                                                       (int64_t)zam * sv[k] + kz * zv[k];
                                    f[e] = __ll2float_rn(br) * sam * wv[k];
                                }
                                h[i] = h2_as_u32(__floats2half2_rn(f[0], f[1]));
                            }
                            if (QUAROT_IN_RANGE(orow + n, 16, a.out, a.M * a.N * 2))
                                *reinterpret_cast<uint4 *>(orow + n) = make_uint4(h[0], h[1], h[2], h[3]);
                        }
                    }
                } else if (mrow) {
                    int32_t *orow = reinterpret_cast<int32_t *>(a.out) + m * a.N;
                    constexpr int sh = UNS ? 0 : 8;           // signed codes are widened x16 each
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const int64_t n = n0 + 32 * c + 4 * v;
                        if (n < a.N && QUAROT_IN_RANGE(orow + n, 16, a.out, a.M * a.N * 4))
                            *reinterpret_cast<int4 *>(orow + n) =
                                make_int4((int)r[4 * v] >> sh, (int)r[4 * v + 1] >> sh, (int)r[4 * v + 2] >> sh,
                                          (int)r[4 * v + 3] >> sh);
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
