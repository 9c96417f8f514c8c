// rotate_quant.cuh -- online randomized Hadamard rotation fused with symmetric
// INT4 round-to-nearest quantization and nibble packing.
//
// What it computes (QuaRot summary "Summary" / "Key points": random Hadamard
// rotations applied online, activations quantized on the fly with RTN,
// group-wise variant with groups of 128; QuaRot article: randomized Hadamard;
// DuQuant Knowl 2 / 12: block-diagonal Hadamard of block 128):
//
//   x' = (x * diag(s)) * H_n / sqrt(n)   (n = K, or n = 128 block by block)
//   per-token: scale = max|x'| / 7 (fp32), code = rint(x' / scale)
//   group-128: scale = fp16(max over the group |x'| / 7),
//              code = clamp(rint(x' / scale), -8, 7); zero scale -> zero codes
//   byte i of a row = code[2i] | code[2i+1] << 4
//
// Design (HBM-bound: 2 bytes read + 0.5 byte written per element):
//  * The unnormalized transform y = (x*diag(s)) H_n is computed in fp32
//    registers; 1/sqrt(n) is folded into the stored scale because the codes
//    rint(7 y / max|y|) do not depend on it.
//  * Sign flips are XORs of the fp16 sign bits; each thread packs the signs
//    of the 128 elements it touches into 4 words once per CTA (the CTAs are
//    persistent over rows).
//  * Full transform (n = 2^p, 256 <= n <= 8192): each row is owned by
//    T = n/128 threads holding 128 values each.  Phase A loads fp16 pairs so
//    that a thread holds element bit 0 and the top six element bits, and
//    applies the Walsh-Hadamard along those 7 bits in registers.  A padded
//    shared-memory transpose then gives each thread 128 contiguous elements
//    (bits 0-6) for phase B, which finishes bits 1..min(6, p-7).  Because
//    H_n = H_2 (x) ... (x) H_2 (Sylvester), stages along different bits
//    commute, so the two phases together are exactly H_n.
//  * Block transform (n = 128): one thread owns one 128-block of a row and
//    does all 7 stages in registers; no exchange at all.  Rows of more than
//    128 blocks give each thread several blocks; with a per-token scale the
//    thread then transforms its blocks twice (once for the row maximum, once
//    to quantize) instead of keeping them all in registers.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace quarot {

// Largest code magnitude of the symmetric RTN at a code width: 2^(b-1) - 1.
// 4-bit codes are packed two per byte; 6- and 8-bit codes are stored one
// signed byte each.
__host__ __device__ constexpr float code_qmax(int bits) { return bits == 8 ? 127.0f : bits == 6 ? 31.0f : 7.0f; }

constexpr int kFwhtThreads = 64;
constexpr int kBlockThreads = 128;

// Quantizes 128 values of one thread and stores the 64 packed bytes.
//  GROUP == 0: r = 7 / max|y| of the row; |v r| <= 7 (1 + 2^-23) so the
//              rounding never leaves [-7, 7] and no clamp is needed.
//  GROUP != 0: r = 1 / (sqrt(n) * fp16 scale); with a normal fp16 scale
//              |v r| <= 7 (1 + 2^-10) as well, so the clamp is needed (and
//              taken, `clamp`) only when the fp16 scale is subnormal.
template <int GROUP>
__device__ __forceinline__ void quant_pack_store(const float (&v)[128], float r, uint8_t *dst, bool valid,
                                                 bool clamp = true)
{
    uint32_t pk[16];
#pragma unroll
    for (int g = 0; g < 16; ++g) {
        uint32_t acc = 0;
        if (GROUP == 0 || !clamp) {
            // two codes per packed fma: rint(t r) lands in the low mantissa bits
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
                float f0, f1;
                fma_x2(v[8 * g + k], v[8 * g + k + 1], r, 12582912.0f, f0, f1);
                acc = push_nibble(acc, __float_as_uint(f0));
                acc = push_nibble(acc, __float_as_uint(f1));
            }
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float z = fminf(fmaxf(v[8 * g + k] * r, -8.f), 7.f);
                acc = push_nibble(acc, __float_as_uint(z + 12582912.0f));
            }
        }
        pk[g] = acc;
    }
    if (valid) {
        uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            d[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
}

// Asymmetric 4-bit codes of 128 values of one thread (packed as usual) and
// their sum.  cz = 1.5 * 2^23 + z (z the integer zero point), r = 1 / step:
// fma(v, r, cz) holds rint(v r) + z in its low mantissa bits, clamped in
// float to [0, 15] before the nibble is taken.
__device__ __forceinline__ uint32_t quant_pack_store_asym(const float (&v)[128], float r, float cz, uint8_t *dst,
                                                          bool valid)
{
    constexpr float C = 12582912.0f;
    uint32_t pk[16];
    uint32_t sum = 0;
#pragma unroll
    for (int g = 0; g < 16; ++g) {
        uint32_t acc = 0;
#pragma unroll
        for (int k = 0; k < 8; k += 2) {
            float f0, f1;
            fma_x2(v[8 * g + k], v[8 * g + k + 1], r, cz, f0, f1);
            f0 = fminf(fmaxf(f0, C), C + 15.0f);
            f1 = fminf(fmaxf(f1, C), C + 15.0f);
            acc = push_nibble(acc, __float_as_uint(f0));
            acc = push_nibble(acc, __float_as_uint(f1));
        }
        pk[g] = acc;
        // the eight nibbles of acc: pairwise byte sums, then the byte total
        const uint32_t b = (acc & 0x0F0F0F0Fu) + ((acc >> 4) & 0x0F0F0F0Fu);
        sum += (b * 0x01010101u) >> 24;
    }
    if (valid) {
        uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            d[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
    return sum;
}

// Outputs of the asymmetric quantizer beyond codes and steps.
struct AsymOut {
    int32_t *zeros;      // [M] zero points
    int32_t *rowsums;    // [M] sums of the row's codes
    float clip;          // clipping ratio of the row's min and max
};

// Rounds 128 values of one thread to signed codes of one byte each and stores
// the 128 bytes (the 6- and 8-bit variants of the same RTN).  r = qmax / max|y|
// of the row (qmax = 31 or 127), so |v r| <= qmax (1 + 2^-23) and no clamp is
// needed; the low byte of the bit pattern of fma(v, r, 1.5 * 2^23) is the
// two's-complement code.
__device__ __forceinline__ void quant_store_i8(const float (&v)[128], float r, int8_t *dst, bool valid)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t pk[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int e = 16 * i + 4 * w;
            float f0, f1, f2, f3;
            fma_x2(v[e], v[e + 1], r, 12582912.0f, f0, f1);
            fma_x2(v[e + 2], v[e + 3], r, 12582912.0f, f2, f3);
            const uint32_t lo = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x0040);
            const uint32_t hi = __byte_perm(__float_as_uint(f2), __float_as_uint(f3), 0x0040);
            pk[w] = __byte_perm(lo, hi, 0x5410);
        }
        if (valid)
            reinterpret_cast<uint4 *>(dst)[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

// fp16 group scale of a block and the matching code multiplier.
__device__ __forceinline__ float group_scale(float amax, float scale_mul, float sqrt_n, __half &s16)
{
    s16 = __float2half_rn(amax * scale_mul);
    const float sf = __half2float(s16);
    return (sf > 0.f && sf <= 65504.f) ? 1.0f / (sf * sqrt_n) : 0.f;
}

// Whether the codes under fp16 scale s16 can leave [-7, 7]: only a nonzero
// subnormal scale rounds far enough below max|y| / 7.
__device__ __forceinline__ bool scale_needs_clamp(__half s16)
{
    const unsigned short b = __half_as_ushort(s16);
    return (b & 0x7C00u) == 0 && (b & 0x03FFu) != 0;
}

// ---------------------------------------------------------------------------
// Full transform, K = 2^LOGN with 8 <= LOGN <= 13.
// ---------------------------------------------------------------------------

// Shared-memory plan of fwht_quant_kernel (dynamic shared memory).
template <int LOGN>
struct FwhtSmem {
    static constexpr int N = 1 << LOGN;
    static constexpr int T = N / 128;                   // threads per row
    static constexpr int R = kFwhtThreads / T;          // rows per CTA iteration
    // staging: one slot per row, padded so that the phase-A reads of a warp
    // spanning several rows fall on different banks
    static constexpr int kPadWords = (T >= 32 || T < 4) ? 4 : T;
    static constexpr int kStageRowBytes = N * 2 + 4 * kPadWords;
    static constexpr int kStageBytes = R * kStageRowBytes;
    // transpose buffer: each 128-element chunk padded to 132 floats and each
    // row by 4 more (8 at K = 1024), so that the phase-A writes of a warp take
    // 2 wavefronts per 256 B and its phase-B reads 4 per 512 B (the minimum)
    // at every K, and every address is a per-thread base plus a constant
    static constexpr int kChunk = 132;
    static constexpr int kRowFloats = (N / 128) * kChunk + (LOGN == 10 ? 8 : 4);
    static constexpr int kBufOffset = kStageBytes;
    static constexpr int kBarOffset = kBufOffset + R * kRowFloats * 4;
    static constexpr int kBytes = kBarOffset + 16 + 32;   // mbarrier, then 8 reduction words
    static_assert(kStageRowBytes % 16 == 0 && kBufOffset % 16 == 0, "16-byte aligned staging and buffer");
};

template <int LOGN, int GROUP, int BITS = 4, bool ASYM = false>
__global__ void __launch_bounds__(kFwhtThreads, 4)
fwht_quant_kernel(const uint32_t *__restrict__ x,      // [M, K/2] fp16 pairs
                  int64_t M, const int8_t *__restrict__ signs,
                  uint8_t *__restrict__ q,             // [M, K/2] (4-bit) or [M, K] (8-bit)
                  void *__restrict__ scales,           // fp32 [M] or fp16 [M, K/128]
                  float scale_mul,                     // 1 / (qmax sqrt(K)) (asymmetric: 1 / sqrt(K))
                  float sqrt_n,                        // sqrt(K), rounded to fp32
                  AsymOut asym)                        // asymmetric variant only
{
    static_assert(LOGN >= 8 && LOGN <= 13, "full transform covers 256..8192");
    static_assert(BITS == 4 || ((BITS == 6 || BITS == 8) && GROUP == 0), "6- and 8-bit codes use one scale per row");
    static_assert(!ASYM || (GROUP == 0 && BITS == 4), "asymmetric codes: 4 bits, one step per row");
    using S = FwhtSmem<LOGN>;
    constexpr float kQmax = code_qmax(BITS);
    constexpr int N = S::N;
    constexpr int T = S::T;
    constexpr int R = S::R;
    constexpr int SH = LOGN - 6;            // element shift of the phase-A pair index j
    constexpr int PB = (LOGN - 7) < 6 ? (LOGN - 7) : 6;   // phase-B bits 1..PB
    constexpr int kChunk = S::kChunk;
    constexpr int kRowFloats = S::kRowFloats;

    extern __shared__ __align__(128) uint8_t fwht_smem[];
    float *buf = reinterpret_cast<float *>(fwht_smem + S::kBufOffset);
    const uint32_t bar = smem_u32(fwht_smem + S::kBarOffset);
    float *red = reinterpret_cast<float *>(fwht_smem + S::kBarOffset + 16);

    const int tid = threadIdx.x;
    const int rl = tid / T;                 // row within the CTA iteration
    const int tr = tid % T;                 // thread within the row

    // phase A pair j covers elements (j << SH) + 2 tr and the next one
    uint32_t sgn[4];
    build_sign_words(signs, [&](int j) { return (j << SH) + 2 * tr; }, sgn);

    // The fp16 rows of the next iteration are copied by the bulk copy engine
    // into the staging slots while this iteration finishes (issued once every
    // thread has read the slots), so no register holds data in flight.
    const int64_t stride = (int64_t)gridDim.x * R;
    auto issue = [&](int64_t r0) {
        const int nrows = (int)min((int64_t)R, M - r0);
        mbar_arrive_expect_tx(bar, (uint32_t)(nrows * N * 2));
        for (int rr = 0; rr < nrows; ++rr)
            bulk_load(smem_u32(fwht_smem + rr * S::kStageRowBytes), x + (r0 + rr) * (N / 2), N * 2, bar);
    };
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (tid == 0 && (int64_t)blockIdx.x * R < M)
        issue((int64_t)blockIdx.x * R);

    const uint32_t *stage = reinterpret_cast<const uint32_t *>(fwht_smem + rl * S::kStageRowBytes);
    int it = 0;
    bool ok = true, aborted = false;
    for (int64_t row0 = (int64_t)blockIdx.x * R; row0 < M; row0 += stride, ++it) {
        const int64_t row = row0 + rl;
        const bool valid = row < M;

        if (!mbar_try_wait(bar, (uint32_t)it & 1)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(bar, (uint32_t)it & 1)) {
                if (globaltimer_ns() - t0 > 2000000000ull) {
                    record_timeout();
                    ok = false;
                    break;
                }
            }
        }
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }

        // ---- phase A: register r = 2 j + b holds element (j << SH) + 2 tr + b
        // (rows past M were not copied: their slots hold stale data, and
        // nothing computed from them is stored)
        float v[128];
#pragma unroll
        for (int j = 0; j < 64; ++j) {
            const float2 f = half2_bits_to_float2(apply_sign_pair(stage[(j << (SH - 1)) + tr], sgn, j));
            v[2 * j] = f.x;
            v[2 * j + 1] = f.y;
        }
        fwht_bits<0, 7>(v);

        // ---- transpose through shared memory: element e of the row goes to
        // chunk e >> 7, offset e & 127; 2 tr < 2^SH never carries into the
        // chunk index, so only the thread's base 2 tr is not a constant
        float *rb = buf + rl * kRowFloats;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
            const int e0 = j << SH;
            *reinterpret_cast<float2 *>(rb + 2 * tr + (e0 >> 7) * kChunk + (e0 & 127)) =
                make_float2(v[2 * j], v[2 * j + 1]);
        }
        __syncthreads();
        // every thread has read its staging slot: refill it for the next iteration
        if (tid == 0 && row0 + stride < M)
            issue(row0 + stride);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float4 f = *reinterpret_cast<const float4 *>(rb + tr * kChunk + 4 * i);
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }

        // ---- phase B: this thread holds elements tr*128 + i, i = 0..127
        fwht_bits<1, PB + 1>(v);

        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 128; i += 2)
            amax = max3f(amax, fabsf(v[i]), fabsf(v[i + 1]));

        if (ASYM) {
            // per-row min and max, clipped range, step, zero point; then the
            // codes and the row's code sum
            float amx = v[0], amn = v[0];
#pragma unroll
            for (int i = 0; i < 128; i += 2) {
                amx = max3f(amx, v[i], v[i + 1]);
                amn = min3f(amn, v[i], v[i + 1]);
            }
            if (T <= 32) {
                amx = warp_max(amx, T);
                amn = warp_min(amn, T);
                __syncthreads();                      // buffer reads done before reuse
            } else {
                amx = warp_max(amx, 32);
                amn = warp_min(amn, 32);
                if ((tid & 31) == 0) {
                    red[tid >> 5] = amx;
                    red[2 + (tid >> 5)] = amn;
                }
                __syncthreads();
                amx = fmaxf(red[0], red[1]);
                amn = fminf(red[2], red[3]);
            }
            const float lo = asym.clip * amn, hi = asym.clip * amx;
            const float dv = (hi - lo) / 15.0f;
            const float z = dv > 0.f ? rintf(-lo / dv) : 0.f;
            const float r = dv > 0.f ? 1.0f / dv : 0.f;
            uint8_t *qdst = q + (valid ? row : 0) * (N / 2) + tr * 64;
            uint32_t csum = quant_pack_store_asym(v, r, 12582912.0f + z, qdst,
                                                  valid && QUAROT_IN_RANGE(qdst, 64, q, M * (N / 2)));
            if (T <= 32) {
                csum = warp_sum(csum, T);
            } else {
                csum = warp_sum(csum, 32);
                if ((tid & 31) == 0)
                    reinterpret_cast<uint32_t *>(red)[4 + (tid >> 5)] = csum;
                __syncthreads();
                csum = reinterpret_cast<uint32_t *>(red)[4] + reinterpret_cast<uint32_t *>(red)[5];
            }
            if (valid && tr == 0 && QUAROT_IN_RANGE(reinterpret_cast<float *>(scales) + row, 4, scales, M * 4) &&
                QUAROT_IN_RANGE(asym.zeros + row, 4, asym.zeros, M * 4) &&
                QUAROT_IN_RANGE(asym.rowsums + row, 4, asym.rowsums, M * 4)) {
                reinterpret_cast<float *>(scales)[row] = dv * scale_mul;
                asym.zeros[row] = (int32_t)z;
                asym.rowsums[row] = (int32_t)csum;
            }
            continue;
        }

        float r;
        if (GROUP == 0) {
            if (T <= 32) {
                amax = warp_max(amax, T);
                __syncthreads();                      // buffer reads done before reuse
            } else {
                amax = warp_max(amax, 32);
                if ((tid & 31) == 0)
                    red[tid >> 5] = amax;
                __syncthreads();
                amax = fmaxf(red[0], red[1]);
            }
            r = amax > 0.f ? kQmax / amax : 0.f;
            if (valid && tr == 0 && QUAROT_IN_RANGE(reinterpret_cast<float *>(scales) + row, 4, scales, M * 4))
                reinterpret_cast<float *>(scales)[row] = amax * scale_mul;
        } else {
            __syncthreads();
            __half s16;
            r = group_scale(amax, scale_mul, sqrt_n, s16);
            __half *sdst = reinterpret_cast<__half *>(scales) + row * (N / 128) + tr;
            if (valid && QUAROT_IN_RANGE(sdst, 2, scales, M * (N / 128) * 2))
                *sdst = s16;
        }
        if (BITS != 4) {
            int8_t *qdst = reinterpret_cast<int8_t *>(q) + (valid ? row : 0) * N + tr * 128;
            quant_store_i8(v, r, qdst, valid && QUAROT_IN_RANGE(qdst, 128, q, M * N));
        } else {
            uint8_t *qdst = q + (valid ? row : 0) * (N / 2) + tr * 64;
            quant_pack_store<GROUP>(v, r, qdst, valid && QUAROT_IN_RANGE(qdst, 64, q, M * (N / 2)));
        }
    }
    // after an abort the copy of the iteration that was given up was issued
    // (in the previous iteration, or before the loop) and may still be in
    // flight into this CTA's memory: wait for it before exiting
    if (aborted && tid == 0)
        mbar_wait_drain(bar, (uint32_t)it & 1, 2000000000ull);
    // a dependent GEMM launched with programmatic serialization may start now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Block transform: each thread owns 128-wide blocks of one row.
//  nb <= 128 blocks per row: one block per thread, 128 / nb rows per CTA.
//  nb >  128: one row per CTA of 128 threads, blocks b, b+128, ... per thread.
// ROTATE = false skips the sign flip and the transform (value cache).
// GROUP = 0: one fp32 scale per row; GROUP = 128: one fp16 scale per block.
// ---------------------------------------------------------------------------
template <bool ROTATE>
__device__ __forceinline__ void load_block(const uint4 *__restrict__ src, bool valid, const uint32_t (&sgn)[4],
                                           float (&v)[128])
{
    uint4 w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        w[i] = valid ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t ww[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t t = ROTATE ? apply_sign_pair(ww[k], sgn, 4 * i + k) : ww[k];
            const float2 f = half2_bits_to_float2(t);
            v[8 * i + 2 * k] = f.x;
            v[8 * i + 2 * k + 1] = f.y;
        }
    }
    if (ROTATE)
        fwht_bits<0, 7>(v);
}

template <bool ROTATE, int GROUP, bool MULTI, int BITS = 4>
__global__ void __launch_bounds__(kBlockThreads)
block128_quant_kernel(const uint4 *__restrict__ x,     // [M, K] fp16, 8 per uint4
                      int64_t M, int K, int rows_per_cta,
                      const int8_t *__restrict__ signs,
                      uint8_t *__restrict__ q,         // [M, K/2] (4-bit) or [M, K] (8-bit)
                      void *__restrict__ scales,
                      float scale_mul, float sqrt_n)
{
    static_assert(BITS == 4 || ((BITS == 6 || BITS == 8) && GROUP == 0), "6- and 8-bit codes use one scale per row");
    constexpr float kQmax = code_qmax(BITS);
    constexpr int kCodeBytes = BITS == 4 ? 64 : 128;   // bytes of one 128-block's codes
    constexpr int BPT = MULTI ? 4 : 1;                 // blocks per thread, at most
    __shared__ unsigned int rowmax[kBlockThreads];
    __shared__ uint32_t sgn_multi[MULTI ? BPT * 4 * kBlockThreads : 1];   // [block i][word][thread]
    const int nb = K >> 7;
    const int tid = threadIdx.x;
    const int rl = MULTI ? 0 : tid / nb;
    const int b0 = MULTI ? tid : tid - rl * nb;
    const bool active = MULTI ? true : rl < rows_per_cta;

    // sign words of this thread's blocks: registers for one block, shared
    // memory (indexed by block) when a thread owns several
    uint32_t sgn[4] = {0u, 0u, 0u, 0u};
    if (!MULTI) {
        if (ROTATE && active)
            build_sign_words(signs, [&](int j) { return b0 * 128 + 2 * j; }, sgn);
    } else {
#pragma unroll 1
        for (int i = 0; i < BPT; ++i) {
            const int b = b0 + i * kBlockThreads;
            uint32_t t[4] = {0u, 0u, 0u, 0u};
            if (ROTATE && b < nb)
                build_sign_words(signs, [&](int j) { return b * 128 + 2 * j; }, t);
#pragma unroll
            for (int w = 0; w < 4; ++w)
                sgn_multi[(i * 4 + w) * kBlockThreads + tid] = t[w];
        }
    }
    auto block_signs = [&](int i, uint32_t (&d)[4]) {
#pragma unroll
        for (int w = 0; w < 4; ++w)
            d[w] = MULTI ? sgn_multi[(i * 4 + w) * kBlockThreads + tid] : sgn[w];
    };

    for (int64_t row0 = (int64_t)blockIdx.x * rows_per_cta; row0 < M;
         row0 += (int64_t)gridDim.x * rows_per_cta) {
        const int64_t row = row0 + rl;
        const bool row_ok = active && row < M;
        const uint4 *xrow = x + (row_ok ? row : 0) * (K / 8);
        uint8_t *qrow = q + (row_ok ? row : 0) * ((int64_t)K * kCodeBytes / 128);

        if (GROUP != 0) {
            // independent blocks
#pragma unroll 1
            for (int i = 0; i < BPT; ++i) {
                const int b = b0 + i * kBlockThreads;
                const bool ok = row_ok && b < nb;
                if (MULTI && !__any_sync(0xffffffffu, ok))
                    break;
                uint32_t sg[4];
                block_signs(i, sg);
                float v[128];
                load_block<ROTATE>(xrow + (ok ? b : 0) * 16, ok, sg, v);
                const float amax = absmax128(v);
                __half s16;
                const float r = group_scale(amax, scale_mul, sqrt_n, s16);
                __half *sdst = reinterpret_cast<__half *>(scales) + row * nb + b;
                if (ok && QUAROT_IN_RANGE(sdst, 2, scales, M * nb * 2))
                    *sdst = s16;
                uint8_t *qdst = qrow + (ok ? b : 0) * 64;
                quant_pack_store<GROUP>(v, r, qdst, ok && QUAROT_IN_RANGE(qdst, 64, q, M * (K / 2)),
                                        scale_needs_clamp(s16));
            }
        } else {
            // one scale per row: reduce the row maximum over the row's threads
            float v[128];
            float amax = 0.f;
#pragma unroll 1
            for (int i = 0; i < BPT; ++i) {
                const int b = b0 + i * kBlockThreads;
                const bool ok = row_ok && b < nb;
                uint32_t sg[4];
                block_signs(i, sg);
                load_block<ROTATE>(xrow + (ok ? b : 0) * 16, ok, sg, v);
#pragma unroll
                for (int k = 0; k < 128; k += 2)
                    amax = max3f(amax, fabsf(v[k]), fabsf(v[k + 1]));
            }
            if (tid < rows_per_cta)
                rowmax[tid] = 0u;
            __syncthreads();
            if (active)
                atomicMax(&rowmax[rl], __float_as_uint(amax));   // amax >= 0: bit order = value order
            __syncthreads();
            amax = active ? __uint_as_float(rowmax[rl]) : 0.f;
            __syncthreads();
            const float r = amax > 0.f ? kQmax / amax : 0.f;
            if (row_ok && b0 == 0 && QUAROT_IN_RANGE(reinterpret_cast<float *>(scales) + row, 4, scales, M * 4))
                reinterpret_cast<float *>(scales)[row] = amax * scale_mul;
            auto store = [&](uint8_t *dst, bool ok) {
                ok = ok && QUAROT_IN_RANGE(dst, kCodeBytes, q, M * (int64_t)K * kCodeBytes / 128);
                if (BITS != 4)
                    quant_store_i8(v, r, reinterpret_cast<int8_t *>(dst), ok);
                else
                    quant_pack_store<0>(v, r, dst, ok);
            };
            if (!MULTI) {
                store(qrow + b0 * kCodeBytes, row_ok);
            } else {
#pragma unroll 1
                for (int i = 0; i < BPT; ++i) {
                    const int b = b0 + i * kBlockThreads;
                    const bool ok = row_ok && b < nb;
                    uint32_t sg[4];
                    block_signs(i, sg);
                    load_block<ROTATE>(xrow + (ok ? b : 0) * 16, ok, sg, v);
                    store(qrow + (ok ? b : 0) * kCodeBytes, ok);
                }
            }
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace quarot
