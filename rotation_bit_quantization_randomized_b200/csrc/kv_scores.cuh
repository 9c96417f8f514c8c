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

    // rotate the G queries of this kv-head cooperatively: 16 threads per
    // query (a half warp), thread p of a query holding elements 8p .. 8p+7;
    // the Walsh-Hadamard stages on element bits 0-2 run in registers, those
    // on bits 3-6 (= bits of p) through half-warp shuffles
    {
        const int p = tid & 15;
        const int8_t *sg = signs + h * 128 + 8 * p;
#pragma unroll
        for (int g0 = 0; g0 < G; g0 += kScoreThreads / 16) {
            // every lane runs the shuffles; lanes of a query index >= G only
            // skip their load and store
            const int g = g0 + (tid >> 4);
            const bool gv = G % (kScoreThreads / 16) == 0 || g < G;
            {
                const uint4 raw = gv ? *reinterpret_cast<const uint4 *>(q + (b * Hq + (int64_t)h * G + g) * 128 + 8 * p)
                                     : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
                float v[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 f = half2_bits_to_float2(w4[k]);
                    v[2 * k] = sg[2 * k] < 0 ? -f.x : f.x;
                    v[2 * k + 1] = sg[2 * k + 1] < 0 ? -f.y : f.y;
                }
#pragma unroll
                for (int hb = 1; hb < 8; hb <<= 1)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if ((i & hb) == 0) {
                            const float a = v[i], c = v[i + hb];
                            v[i] = a + c;
                            v[i + hb] = a - c;
                        }
#pragma unroll
                for (int lb = 1; lb < 16; lb <<= 1) {
                    const bool upper = (p & lb) != 0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float o = __shfl_xor_sync(0xffffffffu, v[i], lb);
                        v[i] = upper ? o - v[i] : v[i] + o;
                    }
                }
                const float inv = 0.08838834764831845f;   // 1/sqrt(128)
                if (gv) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        qs[8 * p + i][g] = v[i] * inv;
                }
            }
        }
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
            for (int k = 0; k < 8; k += 2) {
                const int d = qd * 32 + wd * 8 + k;
                float qv0[G], qv1[G];                 // queries at d and d + 1
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    qv0[g] = qs[d][g];
                    qv1[g] = qs[d + 1][g];
                }
#pragma unroll
                for (int i = 0; i < kScoreTokPerThread; ++i) {
                    const uint32_t word = wd == 0 ? cur[i].x : wd == 1 ? cur[i].y : wd == 2 ? cur[i].z : cur[i].w;
                    // two nibbles -> two floats exactly with one packed subtract:
                    // (2^23 + (c ^ 8)) - (2^23 + 8) = c
                    float c0, c1;
                    sub_x2(__uint_as_float(((word >> (4 * k)) & 0xFu) ^ 0x4B000008u),
                           __uint_as_float(((word >> (4 * k + 4)) & 0xFu) ^ 0x4B000008u), 8388616.0f, c0, c1);
#pragma unroll
                    for (int g = 0; g + 1 < G; g += 2) {
                        fma_x2_acc(qv0[g], qv0[g + 1], c0, acc[i][g], acc[i][g + 1]);
                        fma_x2_acc(qv1[g], qv1[g + 1], c1, acc[i][g], acc[i][g + 1]);
                    }
                    if (G & 1) {
                        acc[i][G - 1] = fmaf(qv0[G - 1], c0, acc[i][G - 1]);
                        acc[i][G - 1] = fmaf(qv1[G - 1], c1, acc[i][G - 1]);
                    }
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
            for (int g = 0; g < G; ++g) {
                float *dst = scores + (b * Hq + (int64_t)h * G + g) * T + t;
                if (QUAROT_IN_RANGE(dst, 4, scores, (int64_t)gridDim.z * Hq * T * 4))
                    *dst = acc[i][g] * s;
            }
        }
    }
}

}  // namespace quarot
