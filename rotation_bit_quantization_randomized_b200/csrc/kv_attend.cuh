// kv_attend.cuh -- the rest of one decode step of attention over the INT4
// value cache (QuaRot abstract: the KV cache in 4 bits; DuQuant Knowl 12: the
// attention output x value product on quantized values, the softmax outputs
// unquantized):
//
//   p[b,hq,t]   = softmax over t of scores[b,hq,t] / sqrt(128)
//   out[b,hq,d] = sum_t p[b,hq,t] * vs[b,t,h] * vcode[b,t,h,d],   h = hq / G
//
// The value rows were stored unrotated, so no inverse rotation follows.
// One CTA per (batch, kv-head) covers all tokens for the G query heads that
// share the head, so every value nibble is read once and used G times:
//  1. two passes over the G rows of scores (L2-resident after the first)
//     give each head's maximum and sum of exponentials;
//  2. per chunk of 64 tokens the threads stage the weights p * vs (one per
//     head and token) and the 64-byte code rows in shared memory; thread d
//     then accumulates out[g, d] over the chunk, G multiply-adds per nibble.
#pragma once

#include "common.cuh"

namespace quarot {

constexpr int kAttThreads = 128;          // one per head dimension
constexpr int kAttChunk = 64;             // tokens staged per step

__device__ __forceinline__ float block_reduce_max(float v, float *red)
{
    v = warp_max(v, 32);
    __syncthreads();
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = v;
    __syncthreads();
    return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

__device__ __forceinline__ float block_reduce_sum(float v, float *red)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = v;
    __syncthreads();
    return (red[0] + red[1]) + (red[2] + red[3]);
}

template <int G>
__global__ void __launch_bounds__(kAttThreads)
kv_attend_kernel(const float *__restrict__ scores,    // [B, Hq, T]
                 const uint8_t *__restrict__ vq,      // [B, T, Hkv, 64 bytes]
                 const __half *__restrict__ vs,       // [B, T, Hkv]
                 int64_t T, int Hkv, float *__restrict__ out)   // [B, Hq, 128]
{
    __shared__ __align__(16) float pw[kAttChunk][G];           // p * vs per token and head
    __shared__ __align__(16) uint32_t vc[kAttChunk][16];       // code rows (64 bytes each)
    __shared__ float red[4];
    __shared__ float smax[G], sinv[G];

    const int h = blockIdx.x;
    const int64_t b = blockIdx.y;
    const int Hq = Hkv * G;
    const int tid = threadIdx.x;
    const float kInvSqrtD = 0.08838834764831845f;             // 1/sqrt(128)

    // ---- 1. softmax statistics of the G heads
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
        const float *sr = scores + (b * Hq + (int64_t)h * G + g) * T;
        float mx = -INFINITY;
        for (int64_t t = tid; t < T; t += kAttThreads)
            mx = fmaxf(mx, sr[t] * kInvSqrtD);
        mx = block_reduce_max(mx, red);
        float z = 0.f;
        for (int64_t t = tid; t < T; t += kAttThreads)
            z += expf(sr[t] * kInvSqrtD - mx);
        z = block_reduce_sum(z, red);
        if (tid == 0) {
            smax[g] = mx;
            sinv[g] = 1.0f / z;
        }
    }
    __syncthreads();

    // ---- 2. weighted sum of the dequantized value rows
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
        acc[g] = 0.f;
    const int byte = tid >> 1;                 // this dimension's byte in a code row
    const int shift = 4 * (tid & 1);           // and its nibble
#pragma unroll 1
    for (int64_t t0 = 0; t0 < T; t0 += kAttChunk) {
        const int nt = (int)min((int64_t)kAttChunk, T - t0);
        // weights: kAttChunk * G values, spread over the threads
        for (int i = tid; i < kAttChunk * G; i += kAttThreads) {
            const int tt = i / G, g = i - tt * G;
            float w = 0.f;
            if (tt < nt) {
                const int64_t t = t0 + tt;
                const float s = scores[(b * Hq + (int64_t)h * G + g) * T + t] * kInvSqrtD;
                w = expf(s - smax[g]) * sinv[g] * __half2float(vs[(b * T + t) * Hkv + h]);
            }
            pw[tt][g] = w;
        }
        // code rows: 16 words per token, 8 tokens per pass of 128 threads
        for (int i = tid; i < kAttChunk * 16; i += kAttThreads) {
            const int tt = i >> 4, wd = i & 15;
            vc[tt][wd] = tt < nt ? reinterpret_cast<const uint32_t *>(vq + ((b * T + t0 + tt) * Hkv + h) * 64)[wd]
                                 : 0x88888888u;
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < nt; ++tt) {
            const uint32_t word = vc[tt][byte >> 2];
            // nibble -> float exactly: (2^23 + (c ^ 8)) - (2^23 + 8) = c
            const float c = __uint_as_float(((word >> (8 * (byte & 3) + shift)) & 0xFu) ^ 0x4B000008u) - 8388616.0f;
#pragma unroll
            for (int g = 0; g < G; ++g)
                acc[g] = fmaf(pw[tt][g], c, acc[g]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
        out[(b * Hq + (int64_t)h * G + g) * 128 + tid] = acc[g];
}

}  // namespace quarot
