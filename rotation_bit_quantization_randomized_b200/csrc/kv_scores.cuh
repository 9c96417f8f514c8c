// kv_scores.cuh -- one decode step of query-key scores over the INT4 key cache.
//
// QuaRot abstract (ISTA record): the KV cache is kept in 4 bits and the
// rotation also covers aspects of the attention mechanism; DuQuant Knowl 12:
// the query-key product is transformed by a fixed Hadamard (+-1/sqrt(2^n))
// with per-head quantization.  Keys were stored rotated by diag(s_h) H_128 /
// sqrt(128), so the query is rotated the same way and
//   scores[b, hq, t] = ks[b,t,h] * sum_d q'[b,hq,d] * code[b,t,h,d],
//   q' = (q * diag(s_h)) H_128 / sqrt(128) in fp32, h = hq / G (grouped-query).
//
// One CTA streams a chunk of tokens of one (batch, kv-head); the G query
// heads that share the kv-head are rotated once per CTA into shared memory
// and every code nibble is used G times.  HBM traffic: 64 B of codes + 2 B of
// scale per (b, t, h), 4 B per score written.
#pragma once

#include "common.cuh"

namespace quarot {

constexpr int kScoreThreads = 128;
constexpr int kScoreTokPerThread = 4;
constexpr int kScoreTokPerCta = kScoreThreads * kScoreTokPerThread;

template <int G>
__global__ void __launch_bounds__(kScoreThreads)
kv_scores_kernel(const __half *__restrict__ q,        // [B, Hq, 128]
                 const int8_t *__restrict__ signs,    // [Hkv, 128]
                 const uint4 *__restrict__ kq,        // [B, T, Hkv, 64 bytes]
                 const __half *__restrict__ ks,       // [B, T, Hkv]
                 int64_t T, int Hkv, float *__restrict__ scores)   // [B, Hq, T]
{
    __shared__ __align__(16) float qs[128][G];        // rotated queries, [d][g]

    const int h = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int Hq = Hkv * G;
    const int tid = threadIdx.x;

    // rotate the G queries of this kv-head: thread g < G owns head g
    if (tid < G) {
        const __half2 *qh = reinterpret_cast<const __half2 *>(q + (b * Hq + (int64_t)h * G + tid) * 128);
        const int8_t *sg = signs + h * 128;
        float v[128];
#pragma unroll
        for (int j = 0; j < 64; ++j) {
            float2 f = __half22float2(qh[j]);
            v[2 * j] = sg[2 * j] < 0 ? -f.x : f.x;
            v[2 * j + 1] = sg[2 * j + 1] < 0 ? -f.y : f.y;
        }
        fwht_bits<0, 7>(v);
        const float inv = 0.08838834764831845f;       // 1/sqrt(128)
#pragma unroll
        for (int d = 0; d < 128; ++d)
            qs[d][tid] = v[d] * inv;
    }
    __syncthreads();

    const int64_t t0 = (int64_t)blockIdx.x * kScoreTokPerCta + tid;
    const uint4 *src[kScoreTokPerThread];
    bool tok_ok[kScoreTokPerThread];
    float acc[kScoreTokPerThread][G];
#pragma unroll
    for (int i = 0; i < kScoreTokPerThread; ++i) {
        const int64_t t = t0 + (int64_t)i * kScoreThreads;
        tok_ok[i] = t < T;
        src[i] = kq + ((b * T + (tok_ok[i] ? t : 0)) * Hkv + h) * 4;
#pragma unroll
        for (int g = 0; g < G; ++g)
            acc[i][g] = 0.f;
    }

    // 16 bytes (32 codes) of every token per iteration; the loop is not
    // unrolled so that the body stays in the instruction cache
    uint4 cur[kScoreTokPerThread];
#pragma unroll
    for (int i = 0; i < kScoreTokPerThread; ++i)
        cur[i] = tok_ok[i] ? __ldg(src[i]) : make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
#pragma unroll 1
    for (int qd = 0; qd < 4; ++qd) {
        uint4 nx[kScoreTokPerThread];
#pragma unroll
        for (int i = 0; i < kScoreTokPerThread; ++i)
            nx[i] = (qd < 3 && tok_ok[i]) ? __ldg(src[i] + qd + 1) : cur[i];
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int d = qd * 32 + wd * 8 + k;
                float qv[G];
#pragma unroll
                for (int g = 0; g < G; g += 4) {
                    if (G >= 4) {
                        const float4 f = *reinterpret_cast<const float4 *>(&qs[d][g]);
                        qv[g] = f.x; qv[g + 1] = f.y; qv[g + 2] = f.z; qv[g + 3] = f.w;
                    } else {
#pragma unroll
                        for (int gg = 0; gg < G; ++gg)
                            qv[gg] = qs[d][gg];
                    }
                }
#pragma unroll
                for (int i = 0; i < kScoreTokPerThread; ++i) {
                    const uint32_t word = wd == 0 ? cur[i].x : wd == 1 ? cur[i].y : wd == 2 ? cur[i].z : cur[i].w;
                    // nibble -> float exactly: (2^23 + (c ^ 8)) - (2^23 + 8) = c
                    const uint32_t u = ((word >> (4 * k)) & 0xFu) ^ 0x4B000008u;
                    const float c = __uint_as_float(u) - 8388616.0f;
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        acc[i][g] = fmaf(qv[g], c, acc[i][g]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kScoreTokPerThread; ++i)
            cur[i] = nx[i];
    }

#pragma unroll
    for (int i = 0; i < kScoreTokPerThread; ++i) {
        const int64_t t = t0 + (int64_t)i * kScoreThreads;
        if (t < T) {
            const float s = __half2float(ks[(b * T + t) * Hkv + h]);
#pragma unroll
            for (int g = 0; g < G; ++g)
                scores[(b * Hq + (int64_t)h * G + g) * T + t] = acc[i][g] * s;
        }
    }
}

}  // namespace quarot
