// kron_quant.cuh -- full rotation for K = 11008 = 344 * 32 fused with symmetric
// INT4 round-to-nearest quantization and nibble packing.
//
//   x' = (x * diag(s)) * (H_344 (x) H_32) / sqrt(K),   element i = a * 32 + b
//
// H_344 is a Hadamard matrix of order 344 that is not a power of two (QuaRot
// summary, Elamur Research: its references give Sloane's library of Hadamard
// matrices as the source of such factors; the library builds one by Paley's
// first construction over GF(7^3)), H_32 the Sylvester matrix.  Viewing a row
// as the 344 x 32 matrix X, the rotated row is H_344^T X H_32.
//
// The H_344 product is a dense contraction and runs on the tensor cores
// (tcgen05.mma kind::f16, fp32 accumulation in tensor memory); its operands
// are exact in fp16 (x is fp16, the factor is +-1), so the only roundings are
// the fp32 sums.  The H_32 product is a 5-stage Walsh-Hadamard transform in
// registers in the epilogue.  A tile is 4 tokens (MMA N = 4 * 32 = 128):
//
//   D_t[a' - 128 t][r * 32 + b] = sum_a H^T[a'][a] * (x_r * s)[a * 32 + b],  t = 0, 1, 2
//
// A = H^T, zero-padded to 384 x 384 fp16 (K-major, 128-byte swizzle), comes
//     from global memory (L2-resident) by TMA in 128 x 64 blocks;
// B = the tile's (x * s)^T, 128 rows (r, b) x 352 reduction columns a, kept
//     as six 64-column slots: the copy engine brings each 64-column slice of
//     the 4 rows (4 x 4 KB, contiguous in x) into a staging ring; eight
//     transposer warps flip the sign bits, transpose 8 x 8 fp16 blocks in
//     registers and store them in the swizzled K-major layout;
// the MMAs run a'-tile by a'-tile (t outer, k inner), so accumulator D_t is
// complete, and handed to the epilogue, after its 22 MMAs; slot kb of B is
// refilled with the next tile as soon as the last a'-tile has used it, and
// the next tile's D_t starts as soon as the epilogue has drained D_t, so
// transposition, MMAs and epilogue of neighbouring tiles overlap.
// Eight epilogue warps read the 3 accumulators (384 tensor-memory columns):
// warps w and w + 4 share lanes 32 (w mod 4) .. + 31 and take tokens
// {0, 1} and {2, 3}; lane a' holds 32 consecutive outputs a' * 32 + b of a
// token, transforms them along b, and writes their 16 packed bytes.
//  * per-token scale: a first pass finds max|x'| of each token (reduction
//    over the 128 lanes and 3 tiles), a second pass quantizes;
//  * group 128: a group is 4 consecutive a' (4 adjacent lanes): the scale
//    comes from a 2-step shuffle maximum.
// Warp roles: 0-7 epilogue, 8-15 transposers (two groups taking alternate
// 64-column slices; signs flipped through a 256-entry mask table), 16 x
// loader, 17 factor loader, 18 MMA issuer.  Every wait is bounded (an abort flag stops all roles).
#pragma once

#include <cuda.h>

#include "int4_gemm.cuh"
#include "rotate_quant.cuh"
#include "tc_ptx.cuh"

namespace quarot {

constexpr int kKronM = 344;                    // Paley factor order
constexpr int kKronN = 32;                     // Sylvester factor order
constexpr int kKronK = kKronM * kKronN;        // 11008
constexpr int kKronAPad = 384;                 // H^T padded to 384 x 384 in global memory
constexpr int kKronRows = 4;                   // tokens per tile
constexpr int kKronKB = 6;                     // 64-column blocks of the reduction (352 used)
constexpr int kKronAT = 3;                     // 128-row blocks of a' (384)
constexpr int kKronBlock = 16384;              // bytes of one 128 x 64 fp16 block
constexpr int kKronAStages = 4, kKronXStages = 3;
constexpr int kKronEpiWarps = 8;
constexpr int kKronTrWarp0 = 8;                // transposers: warps 8-15, two groups of 4
constexpr int kKronXWarp = 16, kKronAWarp = 17, kKronMmaWarp = 18;
constexpr int kKronThreads = 19 * 32;

struct KronSmem {
    static constexpr int kAOff = 0;
    static constexpr int kBOff = kAOff + kKronAStages * kKronBlock;     // 6 slots, one per k-block
    static constexpr int kXOff = kBOff + kKronKB * kKronBlock;
    static constexpr int kBarOff = kXOff + kKronXStages * kKronBlock;
    static constexpr int kNumBars = 2 * kKronXStages + 2 * kKronKB + 2 * kKronAStages + 2 * kKronAT + 1;
    static constexpr int kMiscOff = kBarOff + 8 * kNumBars;
    static constexpr int kLutOff = (kMiscOff + 16 + 4 * kKronEpiWarps * 2 + 15) / 16 * 16;   // after slot/flag, reduction
    static constexpr int kSignOff = kLutOff + 256 * 16;                         // 256 sign-mask patterns
    static constexpr int kBytes = kSignOff + 4 * kKronM + 1024;                 // sign bytes [4][344], alignment
    static_assert(kLutOff % 16 == 0 && kSignOff % 16 == 0 && kMiscOff % 8 == 0, "shared-memory alignment");
    static_assert(kBytes <= 232448, "shared memory per block");
};

// Instruction descriptor for kind::f16: fp32 accumulator, fp16 A and B, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N)
{
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, fp16 operands, fp32 accumulator.
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Unnormalized Walsh-Hadamard transform of 32 values (Sylvester order).
__device__ __forceinline__ void fwht32(float (&v)[32])
{
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; i += 2 * h) {
            if (h == 1) {
                const float a = v[i], b = v[i + 1];
                v[i] = a + b;
                v[i + 1] = a - b;
            } else {
#pragma unroll
                for (int j = i; j < i + h; j += 2)
                    bfly_x2(v[j], v[j + 1], v[j + h], v[j + h + 1]);
            }
        }
    }
}

// 32 codes -> 16 packed bytes.  GROUP == 0: |v r| <= 7 (1 + 2^-23), no clamp;
// otherwise clamp (matters only for a subnormal fp16 scale).
template <int GROUP>
__device__ __forceinline__ uint4 quant_pack32(const float (&v)[32], float r)
{
    uint32_t pk[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        uint32_t acc = 0;
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
            float f0, f1;
            if (GROUP == 0) {
                fma_x2(v[8 * g + k], v[8 * g + k + 1], r, 12582912.0f, f0, f1);
            } else {
                f0 = fminf(fmaxf(v[8 * g + k] * r, -8.f), 7.f) + 12582912.0f;
                f1 = fminf(fmaxf(v[8 * g + k + 1] * r, -8.f), 7.f) + 12582912.0f;
            }
            acc = push_nibble(acc, __float_as_uint(f0));
            acc = push_nibble(acc, __float_as_uint(f1));
        }
        pk[g] = acc;
    }
    return make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

// XOR masks that flip the signs of 8 fp16 values (4 words) whose sign bits
// are the 8 bits of v: word w gets bit 15 from bit 2w and bit 31 from bit 2w + 1.
__device__ __forceinline__ uint4 sign_mask_pattern(uint32_t v)
{
    uint32_t m[4];
#pragma unroll
    for (int w = 0; w < 4; ++w)
        m[w] = (((v >> (2 * w)) & 1u) << 15) | (((v >> (2 * w + 1)) & 1u) << 31);
    return make_uint4(m[0], m[1], m[2], m[3]);
}

template <int GROUP>
__global__ void __launch_bounds__(kKronThreads, 1)
kron_quant_kernel(const __grid_constant__ CUtensorMap tma_h,     // H^T, fp16 [384][384], box {64, 128}, SW128
                  const __half *__restrict__ x,                  // [M, 11008]
                  int64_t M, const int8_t *__restrict__ signs,   // [11008]
                  uint8_t *__restrict__ q,                       // [M, 5504]
                  void *__restrict__ scales,                     // fp32 [M] or fp16 [M, 86]
                  float scale_mul, float sqrt_n)
{
    using S = KronSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_xfull = sbase + S::kBarOff;
    const uint32_t bar_xempty = bar_xfull + 8 * kKronXStages;
    const uint32_t bar_bfull = bar_xempty + 8 * kKronXStages;
    const uint32_t bar_bempty = bar_bfull + 8 * kKronKB;
    const uint32_t bar_afull = bar_bempty + 8 * kKronKB;
    const uint32_t bar_aempty = bar_afull + 8 * kKronAStages;
    const uint32_t bar_tfull = bar_aempty + 8 * kKronAStages;
    const uint32_t bar_tempty = bar_tfull + 8 * kKronAT;
    const uint32_t bar_drain = bar_tempty + 8 * kKronAT;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + S::kMiscOff + 4);
    float *red = reinterpret_cast<float *>(smem + S::kMiscOff + 16);     // [8 warps][2 tokens]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t tiles = (M + kKronRows - 1) / kKronRows;
    const int my_tiles = (int64_t)blockIdx.x < tiles ? (int)((tiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kKronXStages; ++s) {
            mbar_init(bar_xfull + 8 * s, 1);
            mbar_init(bar_xempty + 8 * s, 4);
        }
        for (int s = 0; s < kKronKB; ++s) {
            mbar_init(bar_bfull + 8 * s, 4);
            mbar_init(bar_bempty + 8 * s, 1);
        }
        for (int s = 0; s < kKronAStages; ++s) {
            mbar_init(bar_afull + 8 * s, 1);
            mbar_init(bar_aempty + 8 * s, 1);
        }
        for (int t = 0; t < kKronAT; ++t) {
            mbar_init(bar_tfull + 8 * t, 1);
            mbar_init(bar_tempty + 8 * t, kKronEpiWarps);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kKronMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    // sign bits of x as bytes sbyte[j][a] (bit bb = s[32 a + 8 j + bb] < 0) and
    // the 256 mask patterns, so that the transposers flip signs from shared memory
    {
        uint4 *lut = reinterpret_cast<uint4 *>(smem + S::kLutOff);
        uint8_t *sbyte = smem + S::kSignOff;
        for (int v = threadIdx.x; v < 256; v += kKronThreads)
            lut[v] = sign_mask_pattern((uint32_t)v);
        for (int i = threadIdx.x; i < 4 * kKronM; i += kKronThreads) {
            const int j = i / kKronM, a = i - j * kKronM;
            const uint2 sb = __ldg(reinterpret_cast<const uint2 *>(signs + a * kKronN + 8 * j));
            uint32_t bits = 0;
#pragma unroll
            for (int bb = 0; bb < 8; ++bb) {
                const uint32_t byte = ((bb < 4 ? sb.x : sb.y) >> (8 * (bb & 3))) & 0xFFu;
                bits |= ((byte >> 7) & 1u) << bb;
            }
            sbyte[i] = (uint8_t)bits;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kKronXWarp) {
        // ------------------------------------------------------------ x loader
        if (lane == 0) {
            bool ok = true;
            int step = 0;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                const int64_t row0 = (blockIdx.x + (int64_t)lt * gridDim.x) * kKronRows;
                const int nr = (int)min((int64_t)kKronRows, M - row0);
                for (int kb = 0; kb < kKronKB; ++kb, ++step) {
                    const int s = step % kKronXStages;
                    if (!gemm_wait(bar_xempty + 8 * s, ((uint32_t)(step / kKronXStages) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // columns a in [64 kb, 64 kb + 64) of a row: 2048 fp16 (the last block: 24 a)
                    const uint32_t bytes = kb < kKronKB - 1 ? 4096u : (uint32_t)(kKronM - 64 * (kKronKB - 1)) * 64u;
                    mbar_arrive_expect_tx(bar_xfull + 8 * s, bytes * nr);
                    for (int r = 0; r < nr; ++r)
                        bulk_load(sbase + S::kXOff + s * kKronBlock + r * 4096,
                                  x + (row0 + r) * kKronK + (int64_t)kb * 64 * kKronN, bytes, bar_xfull + 8 * s);
                }
            }
            // every copy issued lands before the CTA can exit: at most the
            // last kKronXStages steps can still be in flight (each stage was
            // consumed before it was refilled)
            for (int j = step - kKronXStages; j < step; ++j)
                if (j >= 0)
                    gemm_wait_drain(bar_xfull + 8 * (j % kKronXStages), (uint32_t)(j / kKronXStages) & 1);
        }
        __syncwarp();
    } else if (warp == kKronAWarp) {
        // ------------------------------------------------------------ factor loader (MMA order: t, then kb)
        if (lane == 0) {
            tma_prefetch_desc(&tma_h);
            bool ok = true;
            int step = 0;
            for (int lt = 0; lt < my_tiles && ok; ++lt)
                for (int t = 0; t < kKronAT && ok; ++t)
                    for (int kb = 0; kb < kKronKB; ++kb, ++step) {
                        const int s = step % kKronAStages;
                        if (!gemm_wait(bar_aempty + 8 * s, ((uint32_t)(step / kKronAStages) & 1) ^ 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(bar_afull + 8 * s, kKronBlock);
                        tma_load_2d(sbase + S::kAOff + s * kKronBlock, &tma_h, kb * 64, t * 128, bar_afull + 8 * s);
                    }
            // as for x: the copies of the last kKronAStages steps land before exit
            for (int j = step - kKronAStages; j < step; ++j)
                if (j >= 0)
                    gemm_wait_drain(bar_afull + 8 * (j % kKronAStages), (uint32_t)(j / kKronAStages) & 1);
        }
        __syncwarp();
    } else if (warp == kKronMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(128, 128);
            bool ok = true;
            int astep = 0;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                for (int t = 0; t < kKronAT && ok; ++t) {
                    // the epilogue has drained D_t of the previous tile
                    if (lt > 0) {
                        if (!gemm_wait(bar_tempty + 8 * t, (uint32_t)(lt - 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    for (int kb = 0; kb < kKronKB; ++kb, ++astep) {
                        if (t == 0) {
                            if (!gemm_wait(bar_bfull + 8 * kb, (uint32_t)lt & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        const int as = astep % kKronAStages;
                        if (!gemm_wait(bar_afull + 8 * as, (uint32_t)(astep / kKronAStages) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t asm_ = sbase + S::kAOff + as * kKronBlock;
                        const uint32_t bsm = sbase + S::kBOff + kb * kKronBlock;
                        const int nks = kb < kKronKB - 1 ? 4 : 2;        // 352 = 5 * 64 + 2 * 16
                        for (int ks = 0; ks < nks; ++ks)
                            umma_f16_ss(tmem_base + t * 128, desc_kmajor_sw128(asm_ + 32 * ks),
                                        desc_kmajor_sw128(bsm + 32 * ks), idesc, (kb > 0 || ks > 0) ? 1u : 0u);
                        umma_commit(bar_aempty + 8 * as);
                        if (t == kKronAT - 1)
                            umma_commit(bar_bempty + 8 * kb);            // slot kb may take the next tile
                    }
                    if (ok)
                        umma_commit(bar_tfull + 8 * t);
                }
            }
            umma_commit(bar_drain);
            gemm_wait_drain(bar_drain, 0);
        }
        __syncwarp();
    } else if (warp >= kKronTrWarp0) {
        // ------------------------------------------------------------ transposers
        // group g = 0 / 1 takes the k-blocks kb = g, g + 2, g + 4 of every tile.
        // thread u of a group: token r = u / 32 (its warp), 8 x 8 block (c, j):
        // columns a = 64 kb + 8 c + i (i = 0..7), b = 8 j .. 8 j + 7
        const int tg = (warp - kKronTrWarp0) >> 2;
        const int u = threadIdx.x - 32 * kKronTrWarp0 - 128 * tg;
        const int r = u >> 5, c = (u >> 2) & 7, j = u & 3;
        const uint4 *lut = reinterpret_cast<const uint4 *>(smem + S::kLutOff);
        const uint8_t *sbyte = smem + S::kSignOff + j * kKronM;
        bool ok = true;
        for (int lt = 0; lt < my_tiles && ok; ++lt) {
            for (int kb = tg; kb < kKronKB; kb += 2) {
                const int step = lt * kKronKB + kb;
                const int xs = step % kKronXStages;
                ok = gemm_wait_warp(bar_xfull + 8 * xs, (uint32_t)(step / kKronXStages) & 1, abort_flag) &&
                     gemm_wait_warp(bar_bempty + 8 * kb, ((uint32_t)lt & 1) ^ 1, abort_flag);
                if (!ok)
                    break;
                const int a0 = 64 * kb + 8 * c;
                uint8_t *bdst = smem + S::kBOff + kb * kKronBlock;
                if (a0 < kKronM) {
                    const uint8_t *src = smem + S::kXOff + xs * kKronBlock + r * 4096 + (8 * c) * 64 + 16 * j;
                    const uint2 sw = *reinterpret_cast<const uint2 *>(sbyte + a0);     // sign bytes of a0 .. a0 + 7
                    uint4 in[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        in[i] = *reinterpret_cast<const uint4 *>(src + 64 * i);
                        const uint4 m = lut[((i < 4 ? sw.x : sw.y) >> (8 * (i & 3))) & 0xFFu];
                        in[i].x ^= m.x;
                        in[i].y ^= m.y;
                        in[i].z ^= m.z;
                        in[i].w ^= m.w;
                    }
                    // out[bb] = the 8 values of column b = 8 j + bb, a = a0 .. a0 + 7
#pragma unroll
                    for (int bb = 0; bb < 8; ++bb) {
                        const uint32_t sel = (bb & 1) ? 0x7632u : 0x5410u;
                        uint32_t w[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint4 v = in[i];
                            const int wi = bb >> 1;
                            w[i] = wi == 0 ? v.x : wi == 1 ? v.y : wi == 2 ? v.z : v.w;
                        }
                        const uint4 o = make_uint4(__byte_perm(w[0], w[1], sel), __byte_perm(w[2], w[3], sel),
                                                   __byte_perm(w[4], w[5], sel), __byte_perm(w[6], w[7], sel));
                        const int n = r * 32 + 8 * j + bb;
                        *reinterpret_cast<uint4 *>(bdst + n * 128 + ((c ^ bb) << 4)) = o;
                    }
                } else if (a0 == kKronM) {
                    // reduction columns 344 .. 351 are zero
#pragma unroll
                    for (int bb = 0; bb < 8; ++bb) {
                        const int n = r * 32 + 8 * j + bb;
                        *reinterpret_cast<uint4 *>(bdst + n * 128 + ((c ^ bb) << 4)) = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bar_bfull + 8 * kb);
                    mbar_arrive(bar_xempty + 8 * xs);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // warp e: TMEM lanes 32 (e mod 4) .. + 31, tokens 2 (e / 4) and 2 (e / 4) + 1
        const int wq = warp & 3;
        const int rbase = 2 * (warp >> 2);
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * wq) << 16);
        constexpr int kEpiThreads = 32 * kKronEpiWarps;
        bool ok = true;
        for (int lt = 0; lt < my_tiles && ok; ++lt) {
            const int64_t row0 = (blockIdx.x + (int64_t)lt * gridDim.x) * kKronRows;
            float rr[2] = {0.f, 0.f};
            if (GROUP == 0) {
                // pass 1: max|x'| of the two tokens over this warp's lanes and all 3 tiles
                float amax[2] = {0.f, 0.f};
                for (int t = 0; t < kKronAT; ++t) {
                    ok = epi_barrier_and(kEpiThreads, gemm_wait_warp(bar_tfull + 8 * t, (uint32_t)lt & 1, abort_flag));
                    if (!ok)
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        uint32_t u[32];
                        tmem_ld32(lane_addr + t * 128 + (rbase + k) * 32, u);
                        tmem_wait_ld(u);
                        float v[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            v[i] = __uint_as_float(u[i]);
                        fwht32(v);
#pragma unroll
                        for (int i = 0; i < 32; i += 2)
                            amax[k] = max3f(amax[k], fabsf(v[i]), fabsf(v[i + 1]));
                    }
                }
                if (!ok)
                    break;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    amax[k] = warp_max(amax[k], 32);
                    if (lane == 0)
                        red[warp * 2 + k] = amax[k];
                }
                epi_barrier_and(kEpiThreads, true);
                const int h = warp >> 2;          // warps 4 h .. 4 h + 3 hold these two tokens
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float a = fmaxf(fmaxf(red[(4 * h) * 2 + k], red[(4 * h + 1) * 2 + k]),
                                          fmaxf(red[(4 * h + 2) * 2 + k], red[(4 * h + 3) * 2 + k]));
                    rr[k] = a > 0.f ? 7.0f / a : 0.f;
                    float *sdst = reinterpret_cast<float *>(scales) + row0 + rbase + k;
                    if (wq == 0 && lane == 0 && row0 + rbase + k < M && QUAROT_IN_RANGE(sdst, 4, scales, M * 4))
                        *sdst = a * scale_mul;
                }
                epi_barrier_and(kEpiThreads, true);      // red is free for the next tile
            }
            // pass 2 (the only pass with group scales): quantize, pack, store; D_t is
            // released as soon as both token pairs are done with it
            for (int t = 0; t < kKronAT; ++t) {
                if (GROUP != 0) {
                    ok = epi_barrier_and(kEpiThreads, gemm_wait_warp(bar_tfull + 8 * t, (uint32_t)lt & 1, abort_flag));
                    if (!ok)
                        break;
                    tc_fence_after();
                }
                const int ap = t * 128 + wq * 32 + lane;            // a'
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int64_t row = row0 + rbase + k;
                    const bool rvalid = row < M;
                    uint32_t u[32];
                    tmem_ld32(lane_addr + t * 128 + (rbase + k) * 32, u);
                    tmem_wait_ld(u);
                    if (k == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(bar_tempty + 8 * t);
                    }
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        v[i] = __uint_as_float(u[i]);
                    fwht32(v);
                    float rq;
                    if (GROUP == 0) {
                        rq = rr[k];
                    } else {
                        float gmax = 0.f;
#pragma unroll
                        for (int i = 0; i < 32; i += 2)
                            gmax = max3f(gmax, fabsf(v[i]), fabsf(v[i + 1]));
                        gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 1));
                        gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, 2));
                        __half s16;
                        rq = group_scale(gmax, scale_mul, sqrt_n, s16);
                        __half *sdst = reinterpret_cast<__half *>(scales) + row * (kKronK / 128) + ap / 4;
                        if (rvalid && ap < kKronM && (lane & 3) == 0 &&
                            QUAROT_IN_RANGE(sdst, 2, scales, M * (kKronK / 128) * 2))
                            *sdst = s16;
                    }
                    const uint4 pk = quant_pack32<GROUP>(v, rq);
                    uint8_t *qdst = q + row * (kKronK / 2) + ap * 16;
                    if (rvalid && ap < kKronM && QUAROT_IN_RANGE(qdst, 16, q, M * (kKronK / 2)))
                        *reinterpret_cast<uint4 *>(qdst) = pk;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kKronMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace quarot
