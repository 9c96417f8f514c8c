// int4_gemm.cuh -- INT4 x INT4 linear layer on the sm_100a tensor cores.
//
// QuaRot abstract (ISTA record): all matrix multiplications run in 4 bits;
// QuaRot summary: products in integers.  The tensor cores have no 4-bit
// integer kind, so packed nibbles are widened to 8-bit and multiplied with
// tcgen05.mma.kind::i8 (int32 accumulation in tensor memory); |code| <= 8, so
// the int32 sums are exact.
//
//   acc[m, n]  = sum_k qa[m, k] qw[n, k]
//   out[m, n]  = fp16(acc * s_a[m] * s_w[n])                       (per token / channel)
//   out[m, n]  = fp16(sum_g acc_g[m, n] * s_a[m, g] * s_w[n, g])   (groups of 128)
//
// Kernel structure (persistent, one CTA per SM, warp-specialized):
//  * TMA producer (one thread): per 128-wide K block, two tiled bulk-tensor
//    copies bring the packed A tile (128 rows x 64 B) and B tile (BN rows x
//    64 B) into a ring of packed stages; rows past M or N arrive as zeros.
//    The copy engine keeps many blocks in flight without the per-SM limits
//    of ordinary loads.
//  * unpack warps: read a packed stage (16 B per lane, 8 rows x 64 B per warp
//    instruction), widen each nibble to an int8 equal to 16 * code (the
//    nibble lands in the top half of its byte, so the sign comes for free),
//    store the ring of int8 stages, and only then release the packed stage
//    to the copy engine (its reads are complete once their values have been
//    stored).  The int8 stages use the 128-byte-swizzled K-major layout the
//    tensor core reads.  Inside each
//    32-wide K chunk the widened order is [low nibbles, high nibbles]; A and B
//    use the same order, so every dot product is unchanged.  Both operands
//    are scaled by 16, so the accumulator holds 256 * acc, removed exactly in
//    the epilogue (|256 acc| <= 2^14 K < 2^31 for K <= 65536).
//  * one MMA thread: waits for a full int8 stage, issues four 128 x BN x 32
//    tcgen05.mma and commits to the stage's "empty" barrier; at the end of a
//    tile it commits to the accumulator's "full" barrier.  Two accumulator
//    buffers in tensor memory let the epilogue of tile i overlap the
//    mainloop of tile i+1.
//  * epilogue warps: tcgen05.ld the accumulator (warp w reads TMEM lanes
//    32(w%4)..+31 = tile rows), scale, convert, store.
//  * every wait is bounded in time; on expiry the CTA records a timeout in
//    the device status word, drains its issued copies and MMAs and frees
//    tensor memory.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace quarot {

enum : int { kEpiScaledF16 = 0, kEpiS32 = 1, kEpiGroupF16 = 2, kEpiAsymF16 = 3 };

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 128;            // int8 elements of K per stage (one 128-byte row)
constexpr int kGemmGroupM = 16;         // tiles along M that share a band of N tiles
constexpr uint64_t kWaitLimitNs = 2000000000ull;

template <int BN, int EPI>
struct GemmShape {
    static constexpr int kPackedA = kGemmBM * kGemmBK / 2;       // bytes of a packed A block
    static constexpr int kPackedB = BN * kGemmBK / 2;
    static constexpr int kPackedStage = kPackedA + kPackedB;
    static constexpr int kABytes = kGemmBM * kGemmBK;            // widened int8 A block
    static constexpr int kBBytes = BN * kGemmBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kPStages = BN == 256 ? 3 : 4;           // packed ring
    static constexpr int kIStages = BN == 256 ? 3 : 4;           // int8 ring
    static constexpr int kLoadRows = kGemmBM + BN;               // A rows then B rows of a tile
    static constexpr int kGroupsPerWarp = 8;                     // 8 rows per warp instruction
    static constexpr int kUnpackWarps = kLoadRows / (8 * kGroupsPerWarp);
    static constexpr int kUnpackThreads = 32 * kUnpackWarps;
    static constexpr int kEpiWarps = EPI == kEpiGroupF16 ? 8 : 4;
    static constexpr int kEpiThreads = 32 * kEpiWarps;
    static constexpr int kMmaWarp = kEpiWarps;
    static constexpr int kTmaWarp = kEpiWarps + 1;
    static constexpr int kUnpackWarp0 = kEpiWarps + 2;
    static constexpr int kThreads = 32 * (kUnpackWarp0 + kUnpackWarps);
    // accumulators in tensor memory: two per-tile buffers, or (grouped) four
    // per-K-block buffers so that the MMA runs ahead of the rescale
    static constexpr int kAccBufs = EPI == kEpiGroupF16 ? 4 : 2;
    static constexpr int kTmemCols = kAccBufs * BN;
    static constexpr int kIntOffset = kPStages * kPackedStage;  // int8 ring after the packed ring
    static constexpr int kBarOffset = kIntOffset + kIStages * kStageBytes;
    static constexpr int kNumBars = 2 * kPStages + 2 * kIStages + 2 * kAccBufs + 1;
    static constexpr int kMiscOffset = kBarOffset + 8 * kNumBars;
    static constexpr int kSwOffset = kMiscOffset + 16;
    static constexpr int kSmemBytes = kSwOffset + 2 * 8 * (kGemmBM + BN) * 4 + 1024;   // grouped scale chunks
    static_assert(kStageBytes % 1024 == 0 && kIntOffset % 1024 == 0, "int8 stages keep 1024-byte alignment");
    static_assert(kPackedStage % 1024 == 0, "packed stages keep 1024-byte alignment");
    static_assert(kGemmBM % (8 * kGroupsPerWarp) == 0, "an unpack warp handles only A or only B rows");
    static_assert(kTmemCols == 256 || kTmemCols == 512, "TMEM allocation is a power of two");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct GemmArgs {
    const uint8_t *qa;      // [M, K/2]
    const void *sa;         // fp32 [M] or fp16 [M, K/128]
    const uint8_t *qw;      // [N, K/2]
    const void *sw;         // fp32 [N] or fp16 [N, K/128]
    void *out;              // fp16 or int32 [M, N]
    const int32_t *za, *ra; // asymmetric: activation zero points and code row sums [M]
    const int32_t *zw, *rw; // asymmetric: weight zero points and code row sums [N]
    int64_t M, N, K;
    int tiles_m, tiles_n, kblocks;
};

// Grouped raster: consecutive tile indices walk down kGemmGroupM M-tiles
// before moving to the next N-tile, so the CTAs working at one time share a
// small band of A and of W in L2.
__device__ __forceinline__ void gemm_tile_coords(int t, int tiles_m, int tiles_n, int &mb, int &nb)
{
    const int group = kGemmGroupM * tiles_n;
    const int g = t / group;
    const int first = g * kGemmGroupM;
    const int gm = min(kGemmGroupM, tiles_m - first);
    const int r = t - g * group;
    mb = first + r % gm;
    nb = r / gm;
}

// Bounded wait: true when the phase completed; false when another role gave
// up (abort flag) or the time limit expired (then this thread sets both).
__device__ __forceinline__ bool gemm_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (*abort_flag)
            return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            record_timeout();
            return false;
        }
    }
}

// Warp-uniform bounded wait: the warp goes on only if every lane saw the
// phase complete, so after a timeout no lane reaches a warp-collective
// tcgen05 instruction without the others.
__device__ __forceinline__ bool gemm_wait_warp(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
    return __all_sync(0xffffffffu, gemm_wait(bar, parity, abort_flag));
}

// Bounded wait that ignores the abort flag (used to drain issued work).
__device__ __forceinline__ bool gemm_wait_drain(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_timeout();
            return false;
        }
    }
    return true;
}

// Named barrier 1 among the first `nthreads` threads (the epilogue warps)
// that also returns the AND of every participant's `p`.
__device__ __forceinline__ bool epi_barrier_and(int nthreads, bool p)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, 1, %2, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

template <int BN, int EPI>
__global__ void __launch_bounds__(GemmShape<BN, EPI>::kThreads, 1)
int4_gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tma_a,
                 const __grid_constant__ CUtensorMap tma_b)
{
    using S = GemmShape<BN, EPI>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_pfull = sbase + S::kBarOffset;
    const uint32_t bar_pempty = bar_pfull + 8 * S::kPStages;
    const uint32_t bar_ifull = bar_pempty + 8 * S::kPStages;
    const uint32_t bar_iempty = bar_ifull + 8 * S::kIStages;
    const uint32_t bar_accf = bar_iempty + 8 * S::kIStages;
    const uint32_t bar_acce = bar_accf + 8 * S::kAccBufs;
    const uint32_t bar_drain = bar_acce + 8 * S::kAccBufs;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + S::kMiscOffset + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = a.tiles_m * a.tiles_n;
    const int KB = a.kblocks;
    const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int total = my_tiles * KB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S::kPStages; ++s) {
            mbar_init(bar_pfull + 8 * s, 1);
            mbar_init(bar_pempty + 8 * s, S::kUnpackThreads);
        }
        for (int s = 0; s < S::kIStages; ++s) {
            mbar_init(bar_ifull + 8 * s, S::kUnpackThreads);
            mbar_init(bar_iempty + 8 * s, 1);
        }
        for (int b = 0; b < S::kAccBufs; ++b) {
            mbar_init(bar_accf + 8 * b, 1);
            mbar_init(bar_acce + 8 * b, S::kEpiThreads);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == S::kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // inputs may come from the kernel launched just before (programmatic
    // dependent launch); everything above overlapped its tail
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == S::kTmaWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tma_a);
            tma_prefetch_desc(&tma_b);
            int lt = 0, kb = 0, mb = 0, nb = 0;
            if (total > 0)
                gemm_tile_coords(blockIdx.x, a.tiles_m, a.tiles_n, mb, nb);
            int step = 0;
            for (; step < total; ++step) {
                const int ps = step % S::kPStages;
                const uint32_t use = (uint32_t)(step / S::kPStages);
                if (!gemm_wait(bar_pempty + 8 * ps, (use & 1) ^ 1, abort_flag))
                    break;
                const uint32_t dst = sbase + ps * S::kPackedStage;
                mbar_arrive_expect_tx(bar_pfull + 8 * ps, S::kPackedStage);
                tma_load_2d(dst, &tma_a, kb * (kGemmBK / 2), mb * kGemmBM, bar_pfull + 8 * ps);
                tma_load_2d(dst + S::kPackedA, &tma_b, kb * (kGemmBK / 2), nb * BN, bar_pfull + 8 * ps);
                if (++kb == KB) {
                    kb = 0;
                    if (++lt < my_tiles)
                        gemm_tile_coords(blockIdx.x + lt * gridDim.x, a.tiles_m, a.tiles_n, mb, nb);
                }
            }
            // copies into stages the unpackers never consumed (abort only) land
            // before the CTA exits
            for (int s = step - S::kPStages; s < step; ++s)
                if (s >= 0)
                    gemm_wait_drain(bar_pfull + 8 * (s % S::kPStages), (uint32_t)(s / S::kPStages) & 1);
        }
        __syncwarp();
    } else if (warp >= S::kUnpackWarp0) {
        // ------------------------------------------------------------ unpackers
        // Unpack warp uw owns row groups 8 uw .. 8 uw + 7 of the combined
        // [A rows 0..127 | B rows 0..BN-1] index space; in each group lane
        // (r, c) = (lane / 4, lane % 4) handles 16 packed bytes (32 codes) of
        // row 8 g + r, which become the row's 16-byte int8 chunks 2c (low
        // nibbles) and 2c + 1 (high nibbles).
        const int uw = warp - S::kUnpackWarp0;
        const int rsub = lane >> 2;
        const int csub = lane & 3;
        const int row0 = 8 * S::kGroupsPerWarp * uw;
        const bool isA = row0 < kGemmBM;                          // warp-uniform
        const int tile_row0 = isA ? row0 : row0 - kGemmBM;        // row inside the A or B tile
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
            // The packed stage is released only now: its values have been
            // consumed by the stores above, so the shared-memory reads are
            // complete, and the proxy fence orders them before the copy
            // engine's next write into the stage.
            fence_proxy_async_smem();
            mbar_arrive(bar_ifull + 8 * is);
            mbar_arrive(bar_pempty + 8 * ps);
        }
    } else if (warp == S::kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kGemmBM, BN);
            bool ok = true;
            int step = 0;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                for (int kb = 0; kb < KB && ok; ++kb, ++step) {
                    const int ab = EPI == kEpiGroupF16 ? (step % S::kAccBufs) : (lt & 1);
                    const uint32_t ause = EPI == kEpiGroupF16 ? (uint32_t)(step / S::kAccBufs) : (uint32_t)(lt >> 1);
                    if (EPI == kEpiGroupF16 || kb == 0) {
                        if (!gemm_wait(bar_acce + 8 * ab, (ause & 1) ^ 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    const int is = step % S::kIStages;
                    if (!gemm_wait(bar_ifull + 8 * is, (uint32_t)(step / S::kIStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t as = sbase + S::kIntOffset + is * S::kStageBytes;
                    const uint32_t bs = as + S::kABytes;
                    const uint32_t d = tmem_base + ab * BN;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t acc = (EPI == kEpiGroupF16) ? (j > 0) : (kb > 0 || j > 0);
                        umma_i8_ss(d, desc_kmajor_sw128(as + 32 * j), desc_kmajor_sw128(bs + 32 * j), idesc, acc);
                    }
                    umma_commit(bar_iempty + 8 * is);
                    if (EPI == kEpiGroupF16 || kb == KB - 1)
                        umma_commit(bar_accf + 8 * ab);
                }
            }
            umma_commit(bar_drain);
            gemm_wait_drain(bar_drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int wq = warp & 3;                 // TMEM lane quarter of this warp
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * wq) << 16);
        bool ok = true;
        int step = 0;
        for (int lt = 0; lt < my_tiles && ok; ++lt) {
            int mb, nb;
            gemm_tile_coords(blockIdx.x + lt * gridDim.x, a.tiles_m, a.tiles_n, mb, nb);
            const int64_t m = (int64_t)mb * kGemmBM + 32 * wq + lane;
            const int64_t n0 = (int64_t)nb * BN;
            const bool mrow = m < a.M;

            if (EPI != kEpiGroupF16) {
                const int ab = lt & 1;
                if (!gemm_wait(bar_accf + 8 * ab, (uint32_t)(lt >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float sam = 0.f;
                if (EPI == kEpiScaledF16 && mrow)
                    sam = reinterpret_cast<const float *>(a.sa)[m] * (1.0f / 256.0f);
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    __syncwarp();
                    tmem_ld32(lane_addr + ab * BN + 32 * c, r);
                    tmem_wait_ld(r);
                    if (c == BN / 32 - 1) {
                        tc_fence_before();
                        mbar_arrive(bar_acce + 8 * ab);
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
                                    make_int4((int)r[4 * v] >> 8, (int)r[4 * v + 1] >> 8,
                                              (int)r[4 * v + 2] >> 8, (int)r[4 * v + 3] >> 8);
                        }
                    }
                }
            } else {
                // grouped: warps w and w+4 share TMEM lanes and split the columns.
                // The scales of 8 K groups at a time are staged in shared memory
                // one chunk ahead (threads 0-127 the tile's row scales, 128-255
                // its column scales), so no step waits on a global load; a
                // named barrier of the epilogue warps hands each chunk over.
                constexpr int HALF = BN / 2;
                constexpr int kCh = 8;                           // K groups per staged chunk
                static_assert(S::kEpiThreads == kGemmBM + BN, "one staging thread per tile row and column");
                const int col0 = (warp >> 2) * HALF;
                const int et = threadIdx.x;                      // 0 .. kEpiThreads-1
                const int G = KB;
                float *sac = reinterpret_cast<float *>(smem + S::kSwOffset);       // [2][kCh][kGemmBM]
                float *swc = sac + 2 * kCh * kGemmBM;                              // [2][kCh][BN]
                const bool is_row = et < kGemmBM;
                const int64_t srow = is_row ? (int64_t)mb * kGemmBM + et : n0 + (et - kGemmBM);
                const bool sval = is_row ? srow < a.M : srow < a.N;
                const __half *sptr = reinterpret_cast<const __half *>(is_row ? a.sa : a.sw) + (sval ? srow : 0) * G;
                const float smul = is_row ? (1.0f / 256.0f) : 1.0f;
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
                            sac[(cb * kCh + i) * kGemmBM + et] = d[i];
                        else
                            swc[(cb * kCh + i) * BN + (et - kGemmBM)] = d[i];
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
                    // chunk cb is complete, and nobody still reads chunk cb ^ 1;
                    // the barrier also makes every epilogue thread's decision to
                    // go on (or to give up after a timeout) the same
                    ok = epi_barrier_and(S::kEpiThreads, ok);
                    if (!ok)
                        break;
                    float nxt[kCh];
                    if (kb0 + kCh < KB)
                        load_chunk(kb0 + kCh, nxt);
                    const int nu = min(kCh, KB - kb0);
                    for (int u = 0; u < nu; ++u, ++step) {
                        const int ab = step % S::kAccBufs;
                        const uint32_t par = (uint32_t)(step / S::kAccBufs) & 1;
                        if (!gemm_wait(bar_accf + 8 * ab, par, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const float sag = sac[(cb * kCh + u) * kGemmBM + 32 * wq + lane];
                        const float *sws = swc + (cb * kCh + u) * BN;
#pragma unroll
                        for (int c = 0; c < HALF / 16; ++c) {
                            uint32_t r[16];
                            __syncwarp();
                            tmem_ld16(lane_addr + ab * BN + col0 + 16 * c, r);
                            tmem_wait_ld16(r);
                            if (c == HALF / 16 - 1) {
                                tc_fence_before();
                                mbar_arrive(bar_acce + 8 * ab);
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
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == S::kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, S::kTmemCols);
    }
}

}  // namespace quarot
