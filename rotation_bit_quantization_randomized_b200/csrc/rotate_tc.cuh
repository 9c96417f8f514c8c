// rotate_tc.cuh -- the full randomized Hadamard rotation of the activations
// (K = 2^p, 256 <= K <= 8192) with its first factor on the tensor cores,
// fused with symmetric round-to-nearest quantization.
//
// What it computes is exactly what fwht_quant_kernel computes (QuaRot
// summary "Summary" / "Key points": random Hadamard rotations applied
// online, activations quantized on the fly with RTN; QuaRot article:
// randomized Hadamard):
//
//   x' = (x * diag(s)) * H_K / sqrt(K),  s = max|x'| / qmax per row (or per
//   128-group, fp16),  code = rint(x' / s)
//
// Sylvester's H_K factors as H_m (x) H_128 with m = K / 128: writing element
// i = 128 a + b, H_K[128a + b][128a' + b'] = H_m[a][a'] H_128[b][b'].  So with
// X[a][b] = (x * diag(s))[128 a + b] the rotated row is (H_m X H_128)[a'][b'].
//
//  * H_m X is a dense contraction with exact operands (x is fp16, H is +-1),
//    so it runs on the tensor cores (tcgen05.mma kind::f16, fp32
//    accumulation in tensor memory) and costs no precision beyond the fp32
//    sums.  One MMA group rotates G = 256 / m tokens: M = 128 rows (P = 128 /
//    m tokens of m rows a'), N = 256 columns (2 tokens x 128 columns b),
//    K = 128 (P tokens x m rows a), with A = I_P (x) H_m (block diagonal,
//    built once per CTA in shared memory) and B read straight from the
//    copy engine's tiles in the MN-major 128-byte-swizzled layout:
//      D[(p, a')][(c, b)] = sum_a H_m[a'][a] X_{token c P + p}[a][b].
//  * The copy engine brings a group as four 16 KB boxes (64 columns b x 128
//    rows (token, a)): for a fixed c the P tokens' rows are consecutive in x.
//  * Two sign warps flip the fp16 sign bits of the staged tiles in place
//    (a thread owns rows r and r + 64, which share a = r mod m, so its 128
//    signs are 4 registers) before the MMAs read them.
//  * The H_128 factor is a 7-stage Walsh-Hadamard transform in registers:
//    tensor-memory lane (p, a') holds, for its token, the 128 values b of row
//    a', which are exactly the 128 contiguous outputs 128 a' .. 128 a' + 127.
//    The thread transforms them, takes their maximum, quantizes and stores
//    its 64 packed bytes (or 128 code bytes) -- a 128-group is one thread.
//  * Ring of three 64 KB stages; two 256-column accumulators (all of tensor
//    memory), so the copies, sign flips, MMAs and epilogue of neighbouring
//    groups overlap.  One CTA per SM, persistent over groups.
// Warp roles: 0-7 epilogue (two sets of four warps on alternate groups;
// warp w reads lanes 32 (w mod 4) .. + 31), 8-9 sign flips, 10 copies, 11 MMAs.
// Every wait is bounded; on expiry the CTA records a timeout, waits for the
// copies and MMAs it issued, frees tensor memory and exits.
#pragma once

#include <cuda.h>

#include "int4_gemm.cuh"
#include "kron_quant.cuh"
#include "rotate_quant.cuh"
#include "tc_ptx.cuh"

namespace quarot {

constexpr int kRtStages = 3;
constexpr int kRtStageBytes = 4 * 16384;          // four 64-column x 128-row fp16 boxes
constexpr int kRtEpiWarps = 8;
constexpr int kRtSignWarp0 = 8, kRtTmaWarp = 10, kRtMmaWarp = 11;
constexpr int kRtThreads = 12 * 32;

struct RtSmem {
    static constexpr int kAOff = 0;                                   // A = I_P (x) H_m, two 16 KB K panels
    static constexpr int kXOff = 32768;
    static constexpr int kBarOff = kXOff + kRtStages * kRtStageBytes;
    static constexpr int kNumBars = 3 * kRtStages + 2 * 2 + 1;
    static constexpr int kMiscOff = kBarOff + 8 * kNumBars;           // tmem slot, abort flag
    static constexpr int kRedOff = kMiscOff + 16;                     // [set][c][warp] maxima
    static constexpr int kBytes = kRedOff + 64 + 1024;                // + alignment slack
    static_assert(kBytes <= 232448, "shared memory per block");
    static_assert(kXOff % 1024 == 0 && kBarOff % 8 == 0, "alignment");
};

// Named barrier `id` among 64 threads (two warps) that also returns the AND
// of every participant's `p`.
__device__ __forceinline__ bool pair_barrier_and(int id, bool p)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, 64, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(id)
        : "memory");
    return r != 0;
}

template <int LOGM, int GROUP, int BITS>
__global__ void __launch_bounds__(kRtThreads, 1)
had_tc_quant_kernel(const __grid_constant__ CUtensorMap tmap,   // x as fp16 [M * m, 128], box {64, 128}, SW128
                    int64_t M, const int8_t *__restrict__ signs, // [K]
                    uint8_t *__restrict__ q,                     // [M, K/2] (4-bit) or [M, K] (6-, 8-bit)
                    void *__restrict__ scales,                   // fp32 [M] or fp16 [M, K/128]
                    float scale_mul,                             // 1 / (qmax sqrt(K))
                    float sqrt_n)                                // sqrt(K), rounded to fp32
{
    static_assert(LOGM >= 1 && LOGM <= 6, "K = 128 m with 2 <= m <= 64");
    static_assert(BITS == 4 || ((BITS == 6 || BITS == 8) && GROUP == 0), "6- and 8-bit codes use one scale per row");
    constexpr int m = 1 << LOGM;
    constexpr int K = 128 * m;
    constexpr int P = 128 / m;                   // tokens along the MMA's M (and its K)
    constexpr int G = 2 * P;                     // tokens per group
    constexpr float kQmax = code_qmax(BITS);
    constexpr int kCodeBytes = BITS == 4 ? 64 : 128;
    using S = RtSmem;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_xfull = sbase + S::kBarOff;
    const uint32_t bar_sfull = bar_xfull + 8 * kRtStages;
    const uint32_t bar_xempty = bar_sfull + 8 * kRtStages;
    const uint32_t bar_accf = bar_xempty + 8 * kRtStages;
    const uint32_t bar_acce = bar_accf + 16;
    const uint32_t bar_drain = bar_acce + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + S::kMiscOff + 4);
    float *red = reinterpret_cast<float *>(smem + S::kRedOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t groups = (M + G - 1) / G;
    const int my_groups = (int64_t)blockIdx.x < groups ? (int)((groups - 1 - blockIdx.x) / gridDim.x + 1) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRtStages; ++s) {
            mbar_init(bar_xfull + 8 * s, 1);
            mbar_init(bar_sfull + 8 * s, 2);
            mbar_init(bar_xempty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_accf + 8 * b, 1);
            mbar_init(bar_acce + 8 * b, kRtEpiWarps / 2);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kRtMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    // A = I_P (x) H_m as fp16, K-major, 128-byte swizzle: row R = (p, a'),
    // column C = (p', a) in panel C / 64, 16-byte chunk (C mod 64) / 8 stored
    // at chunk ((C mod 64) / 8) ^ (R mod 8) of the row
    for (int i = threadIdx.x; i < 128 * 16; i += kRtThreads) {
        const int R = i >> 4, ch = i & 15;               // row, logical 8-column chunk of the 128 columns
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t h = 0;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int C = 8 * ch + 2 * e + k;
                uint16_t v = 0;                          // +0.0 off the diagonal blocks
                if ((R >> LOGM) == (C >> LOGM))
                    v = (__popc((R & (m - 1)) & (C & (m - 1))) & 1) ? 0xBC00 : 0x3C00;
                h |= (uint32_t)v << (16 * k);
            }
            w[e] = h;
        }
        const int panel = ch >> 3, pc = (ch & 7) ^ (R & 7);
        *reinterpret_cast<uint4 *>(smem + S::kAOff + panel * 16384 + R * 128 + pc * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kRtTmaWarp) {
        // ------------------------------------------------------------ copies
        if (lane == 0) {
            tma_prefetch_desc(&tmap);
            int lg = 0;
            for (; lg < my_groups; ++lg) {
                const int s = lg % kRtStages;
                if (!gemm_wait(bar_xempty + 8 * s, ((uint32_t)(lg / kRtStages) & 1) ^ 1, abort_flag))
                    break;
                const int64_t g = blockIdx.x + (int64_t)lg * gridDim.x;
                const uint32_t dst = sbase + S::kXOff + s * kRtStageBytes;
                mbar_arrive_expect_tx(bar_xfull + 8 * s, kRtStageBytes);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int bh = 0; bh < 2; ++bh)
                        tma_load_2d(dst + (2 * c + bh) * 16384, &tmap, 64 * bh, (int)((g * G + c * P) * m),
                                    bar_xfull + 8 * s);
            }
            // the copies of the last stages land before the CTA can exit
            for (int j = lg - kRtStages; j < lg; ++j)
                if (j >= 0)
                    gemm_wait_drain(bar_xfull + 8 * (j % kRtStages), (uint32_t)(j / kRtStages) & 1);
        }
        __syncwarp();
    } else if (warp == kRtMmaWarp) {
        // ------------------------------------------------------------ MMAs
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(128, 256) | (1u << 16);     // B MN-major
            for (int lg = 0; lg < my_groups; ++lg) {
                const int s = lg % kRtStages;
                const int ab = lg & 1;
                if (!gemm_wait(bar_sfull + 8 * s, (uint32_t)(lg / kRtStages) & 1, abort_flag))
                    break;
                if (!gemm_wait(bar_acce + 8 * ab, ((uint32_t)(lg >> 1) & 1) ^ 1, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t xs = sbase + S::kXOff + s * kRtStageBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16_ss(tmem_base + ab * 256,
                                desc_kmajor_sw128(sbase + S::kAOff + 16384 * (kk >> 2) + 32 * (kk & 3)),
                                desc_mnmajor_sw128(xs + 2048 * kk, 16384), idesc, kk > 0 ? 1u : 0u);
                umma_commit(bar_xempty + 8 * s);
                umma_commit(bar_accf + 8 * ab);
            }
            umma_commit(bar_drain);
            gemm_wait_drain(bar_drain, 0);
        }
        __syncwarp();
    } else if (warp >= kRtSignWarp0) {
        // ------------------------------------------------------------ sign flips
        // thread u: K rows u and u + 64 (both a = u mod m), every box and chunk
        const int u = threadIdx.x - 32 * kRtSignWarp0;
        const int a = u & (m - 1);
        uint32_t sgn[4];
        build_sign_words(signs, [&](int j) { return 128 * a + 2 * j; }, sgn);
        // XOR masks of the 16 chunks (64-column half bh, chunk cl) of row a
        uint32_t msk[2][8][4];
#pragma unroll
        for (int bh = 0; bh < 2; ++bh)
#pragma unroll
            for (int cl = 0; cl < 8; ++cl)
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    msk[bh][cl][w] = apply_sign_pair(0u, sgn, 32 * bh + 4 * cl + w);
        for (int lg = 0; lg < my_groups; ++lg) {
            const int s = lg % kRtStages;
            if (!gemm_wait_warp(bar_xfull + 8 * s, (uint32_t)(lg / kRtStages) & 1, abort_flag))
                break;
            uint8_t *xs = smem + S::kXOff + s * kRtStageBytes;
            // one 128-byte line (8 chunks) at a time: eight loads in flight,
            // then the flips, then eight stores
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = u + 64 * h;
                uint8_t *row = xs + r * 128;
#pragma unroll
                for (int box = 0; box < 4; ++box) {
                    const int bh = box & 1;
                    uint4 v[8];
#pragma unroll
                    for (int cl = 0; cl < 8; ++cl)
                        v[cl] = *reinterpret_cast<const uint4 *>(row + box * 16384 + ((cl ^ (r & 7)) << 4));
#pragma unroll
                    for (int cl = 0; cl < 8; ++cl) {
                        v[cl].x ^= msk[bh][cl][0];
                        v[cl].y ^= msk[bh][cl][1];
                        v[cl].z ^= msk[bh][cl][2];
                        v[cl].w ^= msk[bh][cl][3];
                    }
#pragma unroll
                    for (int cl = 0; cl < 8; ++cl)
                        *reinterpret_cast<uint4 *>(row + box * 16384 + ((cl ^ (r & 7)) << 4)) = v[cl];
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_sfull + 8 * s);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // two sets of four warps take alternate groups (set k: accumulator k),
        // so that one set's tensor-memory loads, reductions and stores overlap
        // the other's arithmetic; warp w of a set reads lanes 32 (w mod 4) ..
        // + 31 and does the two token halves c = 0, 1 one after the other
        const int set = warp >> 2;
        const int wq = warp & 3;
        const int L = 32 * wq + lane;                    // accumulator row (p, a')
        const int p = L >> LOGM, ap = L & (m - 1);
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * wq) << 16) + set * 256;
        const int pair_bar = 2 + 2 * set + (wq >> 1);  // the two warps of a token when m = 64
        for (int lg = set; lg < my_groups; lg += 2) {
            bool ok = gemm_wait_warp(bar_accf + 8 * set, (uint32_t)(lg >> 1) & 1, abort_flag);
            if (m == 64)
                ok = pair_barrier_and(pair_bar, ok);     // the pair goes on (or gives up) together
            if (!ok)
                break;
            tc_fence_after();
            const int64_t g = blockIdx.x + (int64_t)lg * gridDim.x;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                const int64_t t = g * G + c * P + p;
                const bool valid = t < M;
                float v[128];
                {
                    uint32_t u0[32], u1[32], u2[32], u3[32];
                    const uint32_t ta = lane_addr + c * 128;
                    tmem_ld32(ta, u0);
                    tmem_ld32(ta + 32, u1);
                    tmem_ld32(ta + 64, u2);
                    tmem_ld32(ta + 96, u3);
                    tmem_wait_ld(u0);
                    tmem_wait_ld(u1);
                    tmem_wait_ld(u2);
                    tmem_wait_ld(u3);
                    if (c == 1) {
                        // the whole accumulator has been read: the MMAs of the
                        // group after next may overwrite it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(bar_acce + 8 * set);
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        v[i] = __uint_as_float(u0[i]);
                        v[32 + i] = __uint_as_float(u1[i]);
                        v[64 + i] = __uint_as_float(u2[i]);
                        v[96 + i] = __uint_as_float(u3[i]);
                    }
                }
                fwht_bits<0, 7>(v);
                float amax = absmax128(v);
                float r;
                bool clamp = false;
                if (GROUP == 0) {
                    // the token's m rows: lanes p m .. p m + m - 1 (two warps of
                    // the set when m = 64, which exchange their maxima)
                    amax = warp_max(amax, m < 32 ? m : 32);
                    if (m == 64) {
                        if (lane == 0)
                            red[(set * 2 + c) * 4 + wq] = amax;
                        pair_barrier_and(pair_bar, true);
                        amax = fmaxf(amax, red[(set * 2 + c) * 4 + (wq ^ 1)]);
                    }
                    r = amax > 0.f ? kQmax / amax : 0.f;
                    if (valid && ap == 0 && QUAROT_IN_RANGE(reinterpret_cast<float *>(scales) + t, 4, scales, M * 4))
                        reinterpret_cast<float *>(scales)[t] = amax * scale_mul;
                } else {
                    __half s16;
                    r = group_scale(amax, scale_mul, sqrt_n, s16);
                    clamp = scale_needs_clamp(s16);
                    __half *sdst = reinterpret_cast<__half *>(scales) + t * m + ap;
                    if (valid && QUAROT_IN_RANGE(sdst, 2, scales, M * m * 2))
                        *sdst = s16;
                }
                uint8_t *dst = q + (valid ? t : 0) * ((int64_t)K * kCodeBytes / 128) + ap * kCodeBytes;
                const bool st_ok = valid && QUAROT_IN_RANGE(dst, kCodeBytes, q, M * ((int64_t)K * kCodeBytes / 128));
                if (BITS == 4)
                    quant_pack_store<GROUP>(v, r, dst, st_ok, clamp);
                else
                    quant_store_i8(v, r, reinterpret_cast<int8_t *>(dst), st_ok);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kRtMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
    // a dependent GEMM launched with programmatic serialization may start now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace quarot
