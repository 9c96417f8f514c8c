// kv_attend.cuh -- the rest of one decode step of attention over the INT4
// value cache (QuaRot abstract: the KV cache in 4 bits; DuQuant Knowl 12: the
// attention output x value product on quantized values, the softmax outputs
// unquantized):
//
//   p[b,hq,t]   = softmax over t of scores[b,hq,t] / sqrt(128)
//   out[b,hq,d] = sum_t p[b,hq,t] * vs[b,t,h] * vcode[b,t,h,d],   h = hq / G
//
// The value rows were stored unrotated, so no inverse rotation follows.
//
// A cluster of S CTAs (S = 1, 2, 4 or 8, chosen on the host from T and from
// how many clusters can be resident at once) covers one (batch, kv-head) pair; CTA r takes the r-th slice of the tokens, for all G query heads that
// share the head, so each value nibble is read once and used G times.  Within
// its slice a CTA walks chunks of 256 tokens with the running-maximum form of
// the softmax (per head: maximum m, sum of exponentials l, and the
// accumulator rescaled by exp(m_old - m_new) when the maximum grows):
//  * warp g % 4 of the CTA computes head g's chunk maximum, the exponentials
//    e = exp(s - m) and their weights e * vs in shared memory;
//  * the chunk's 64-byte code rows are copied into shared memory with 16-byte
//    asynchronous copies during that work; warp w then takes the tokens w, w + 4, ..., lane l the head
//    dimensions 4l .. 4l + 3, accumulating G x 4 outputs with packed fp32x2
//    multiply-adds.
// At the end the four warps' partial sums are added in shared memory and the
// S CTAs of the cluster combine their (m, l, acc) through distributed shared
// memory:  out = sum_r exp(m_r - M) acc_r / sum_r exp(m_r - M) l_r, M = max m_r.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace quarot {

constexpr int kAttThreads = 128;
constexpr int kAttChunk = 256;             // tokens per chunk, 64 per warp
constexpr int kAttMaxSplit = 8;            // CTAs per cluster (portable limit)

template <int G>
struct AttSmem {
    // chunk stage: weights [256][G] fp32 and code rows [256][64] bytes; after
    // the last chunk the same bytes hold the warps' partial sums [4][G][128]
    static constexpr int kWeightBytes = kAttChunk * G * 4;
    static constexpr int kCodeBytes = kAttChunk * 64;
    static constexpr int kPartBytes = 4 * G * 128 * 4;
    static constexpr int kStageBytes =
        (kWeightBytes + kCodeBytes > kPartBytes) ? kWeightBytes + kCodeBytes : kPartBytes;
};

__device__ __forceinline__ float warp_sum_f(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// 16-byte global -> shared copy that does not pass through registers
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t cluster_addr)
{
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
    return v;
}

template <int G>
__global__ void __launch_bounds__(kAttThreads)
kv_attend_kernel(const float *__restrict__ scores,    // [B, Hq, T]
                 const uint8_t *__restrict__ vq,      // [B, T, Hkv, 64 bytes]
                 const __half *__restrict__ vs,       // [B, T, Hkv]
                 int64_t T, int Hkv, float *__restrict__ out)   // [B, Hq, 128]
{
    using S_ = AttSmem<G>;
    __shared__ __align__(16) uint8_t stage[S_::kStageBytes];
    __shared__ __align__(16) float fin[G][128];          // this CTA's accumulator, summed over warps
    __shared__ float sm_m[G], sm_l[G], sm_alpha[G];

    float *wgt = reinterpret_cast<float *>(stage);                       // [256][G]
    const uint16_t *codes16 = reinterpret_cast<const uint16_t *>(stage + S_::kWeightBytes);
    const uint32_t codes_s = smem_u32(stage + S_::kWeightBytes);
    float *part = reinterpret_cast<float *>(stage);                      // [4][G][128]

    const int nsplit = gridDim.x;
    const int r = blockIdx.x;                  // = rank in the cluster (cluster spans x)
    const int h = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int Hq = Hkv * G;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float kInvSqrtD = 0.08838834764831845f;             // 1/sqrt(128)

    const int64_t slice = (T + nsplit - 1) / nsplit;
    const int64_t ts = min(T, (int64_t)r * slice);
    const int64_t te = min(T, ts + slice);

    if (tid < G) {
        sm_m[tid] = -INFINITY;
        sm_l[tid] = 0.f;
    }
    float acc[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int k = 0; k < 4; ++k)
            acc[g][k] = 0.f;
    __syncthreads();

    const float *srow = scores + (b * Hq + (int64_t)h * G) * T;
#pragma unroll 1
    for (int64_t t0 = ts; t0 < te; t0 += kAttChunk) {
        const int nt = (int)min((int64_t)kAttChunk, te - t0);
        // code rows of the chunk (4 x 16 bytes per token), copied while the
        // statistics below are computed
#pragma unroll
        for (int j = 0; j < kAttChunk * 4 / kAttThreads; ++j) {
            const int i = tid + j * kAttThreads;
            if (i < nt * 4)
                cp_async16(codes_s + 16 * i, vq + ((b * T + t0 + (i >> 2)) * Hkv + h) * 64 + 16 * (i & 3));
        }
        // value scales of the tokens lane + 32 j (the same for every head)
        float vsv[kAttChunk / 32];
#pragma unroll
        for (int j = 0; j < kAttChunk / 32; ++j) {
            const int tt = lane + 32 * j;
            vsv[j] = tt < nt ? __half2float(vs[(b * T + t0 + tt) * Hkv + h]) : 0.f;
        }
        // chunk statistics and weights of the heads this warp owns
        for (int g = warp; g < G; g += 4) {
            float sv[kAttChunk / 32];
            float cm = -INFINITY;
#pragma unroll
            for (int j = 0; j < kAttChunk / 32; ++j) {
                const int tt = lane + 32 * j;
                sv[j] = tt < nt ? srow[(int64_t)g * T + t0 + tt] * kInvSqrtD : -INFINITY;
                cm = fmaxf(cm, sv[j]);
            }
            cm = warp_max(cm, 32);
            const float m_old = sm_m[g];
            const float m_new = fmaxf(m_old, cm);
            float ls = 0.f;
#pragma unroll
            for (int j = 0; j < kAttChunk / 32; ++j) {
                const int tt = lane + 32 * j;
                if (tt < nt) {
                    const float e = expf(sv[j] - m_new);
                    ls += e;
                    wgt[tt * G + g] = e * vsv[j];
                }
            }
            ls = warp_sum_f(ls);
            __syncwarp();
            if (lane == 0) {
                const float alpha = m_old == -INFINITY ? 0.f : expf(m_old - m_new);
                sm_alpha[g] = alpha;
                sm_l[g] = sm_l[g] * alpha + ls;
                sm_m[g] = m_new;
            }
        }
        cp_async_wait_all();
        __syncthreads();
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float a = sm_alpha[g];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                acc[g][k] *= a;
        }
        // weighted sum over this warp's tokens of the chunk
#pragma unroll 2
        for (int tt = warp; tt < nt; tt += 4) {
            const uint32_t x = codes16[tt * 32 + lane];      // dims 4l .. 4l+3, low nibble first
            // nibble -> float exactly: (2^23 + (c ^ 8)) - (2^23 + 8) = c
            float c0 = __uint_as_float((x & 0xFu) ^ 0x4B000008u);
            float c1 = __uint_as_float(((x >> 4) & 0xFu) ^ 0x4B000008u);
            float c2 = __uint_as_float(((x >> 8) & 0xFu) ^ 0x4B000008u);
            float c3 = __uint_as_float((x >> 12) ^ 0x4B000008u);
            sub_x2(c0, c1, 8388616.0f, c0, c1);
            sub_x2(c2, c3, 8388616.0f, c2, c3);
            const float *wr = wgt + tt * G;
            float wv[G];
            if constexpr (G % 4 == 0) {
#pragma unroll
                for (int g = 0; g < G; g += 4) {
                    const float4 w4 = *reinterpret_cast<const float4 *>(wr + g);
                    wv[g] = w4.x;
                    wv[g + 1] = w4.y;
                    wv[g + 2] = w4.z;
                    wv[g + 3] = w4.w;
                }
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g)
                    wv[g] = wr[g];
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                fma_x2_acc(c0, c1, wv[g], acc[g][0], acc[g][1]);
                fma_x2_acc(c2, c3, wv[g], acc[g][2], acc[g][3]);
            }
        }
        __syncthreads();
    }

    // the four warps' partial sums -> fin
#pragma unroll
    for (int g = 0; g < G; ++g)
        *reinterpret_cast<float4 *>(part + (warp * G + g) * 128 + 4 * lane) =
            make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g)
        fin[g][tid] = (part[(0 * G + g) * 128 + tid] + part[(1 * G + g) * 128 + tid]) +
                      (part[(2 * G + g) * 128 + tid] + part[(3 * G + g) * 128 + tid]);

    // combine the slices of the cluster: CTA r finishes heads r, r + S, ...
    cluster_sync_all();
    const uint32_t a_fin = smem_u32(&fin[0][0]);
    const uint32_t a_m = smem_u32(&sm_m[0]);
    const uint32_t a_l = smem_u32(&sm_l[0]);
    for (int g = r; g < G; g += nsplit) {
        // every remote load is issued before any of them is used
        float mq[kAttMaxSplit], lq[kAttMaxSplit], fq[kAttMaxSplit];
#pragma unroll
        for (int q = 0; q < kAttMaxSplit; ++q) {
            if (q < nsplit) {
                mq[q] = ld_dsmem_f32(mapa_shared(a_m + 4 * g, q));
                lq[q] = ld_dsmem_f32(mapa_shared(a_l + 4 * g, q));
                fq[q] = ld_dsmem_f32(mapa_shared(a_fin + 4 * (g * 128 + tid), q));
            } else {
                mq[q] = -INFINITY;
                lq[q] = 0.f;
                fq[q] = 0.f;
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kAttMaxSplit; ++q)
            M = fmaxf(M, mq[q]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int q = 0; q < kAttMaxSplit; ++q) {
            const float f = mq[q] == -INFINITY ? 0.f : expf(mq[q] - M);
            den = fmaf(f, lq[q], den);
            num = fmaf(f, fq[q], num);
        }
        float *dst = out + (b * Hq + (int64_t)h * G + g) * 128 + tid;
        if (QUAROT_IN_RANGE(dst, 4, out, (int64_t)gridDim.z * Hq * 128 * 4))
            *dst = num / den;
    }
    // no CTA leaves while another may still read its shared memory
    cluster_sync_all();
}

}  // namespace quarot
