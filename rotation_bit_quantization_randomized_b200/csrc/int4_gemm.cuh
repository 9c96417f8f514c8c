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
// This header holds what the GEMM kernels share (int4_gemm_pair.cuh: the
// INT4 linear on CTA pairs, per token / per channel and with 128-wide K
// groups; int8_gemm_pair.cuh: the INT8 variant; mma_peak.cuh: the tensor-rate
// probe): the epilogue kinds, the K step, the argument block, the grouped
// tile raster and the bounded waits.  Packed nibbles are widened to int8 =
// 16 * code (the nibble in the top half of its byte, so the sign comes for
// free); both operands carry the factor 16, so the accumulator holds
// 256 * acc, removed exactly in the epilogue (|256 acc| <= 2^14 K < 2^31 for
// K <= 65536).  Every wait is bounded in time; on expiry the waiting thread
// records a timeout in the device status word and raises the CTA's abort
// flag, and the kernel drains its issued copies and MMAs before it frees
// tensor memory.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace quarot {

enum : int { kEpiScaledF16 = 0, kEpiS32 = 1, kEpiGroupF16 = 2, kEpiAsymF16 = 3 };

constexpr int kGemmBK = 128;            // int8 elements of K per stage (one 128-byte row)
constexpr int kGemmGroupM = 16;         // tiles along M that share a band of N tiles
constexpr uint64_t kWaitLimitNs = 2000000000ull;

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

}  // namespace quarot
