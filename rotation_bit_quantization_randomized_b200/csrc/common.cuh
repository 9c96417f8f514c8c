// common.cuh -- small device helpers shared by the libquarot kernels.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace quarot {

// Device-side error word, one bit per kind of failure: a bounded wait in a
// kernel expired, or (bounds-checking builds only) a store fell outside its
// output.  Read and cleared on the host by quarot_get_device_status().
__device__ int g_device_status;

enum : int { kDevOk = 0, kDevTimeout = 1, kDevBounds = 2 };

__device__ __forceinline__ void record_timeout() { atomicOr(&g_device_status, kDevTimeout); }

// Bounds-checking builds (QUAROT_DEBUG_BOUNDS defined): before each global
// store of an output, QUAROT_IN_RANGE(p, bytes, base, total) checks that the
// `bytes` written at p lie inside the output [base, base + total) as the
// kernel's size arguments give it; on failure it sets the bounds bit of the
// device status word and yields false, so that the store is skipped.  In
// normal builds it is the constant true and its arguments are not evaluated.
#ifdef QUAROT_DEBUG_BOUNDS
__device__ __forceinline__ bool debug_in_range(const void *p, size_t bytes, const void *base, size_t total)
{
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(base);
    const bool ok = a >= b && a + bytes <= b + total;
    if (!ok)
        atomicOr(&g_device_status, kDevBounds);
    return ok;
}
#define QUAROT_IN_RANGE(p, bytes, base, total) \
    (::quarot::debug_in_range((const void *)(p), (size_t)(bytes), (const void *)(base), (size_t)(total)))
#else
#define QUAROT_IN_RANGE(p, bytes, base, total) (true)
#endif

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits until the phase of the mbarrier at shared address `bar` with parity
// `parity` has completed, for at most `limit_ns`; on expiry records a timeout
// in the device status word and returns false.  Used to drain copies a
// thread issued before it exits (the wait ignores any abort of the caller).
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    uint32_t done;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done)
            return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_timeout();
            return false;
        }
    }
}

// Round-to-nearest-even of v into the low mantissa bits of a float: for
// |v| < 2^22, 1.5*2^23 + v has unit spacing, so the single rounding of the
// addition is the integer rounding (ties to even) and the low 4 bits of the
// bit pattern are the two's-complement nibble of the integer.
__device__ __forceinline__ uint32_t rne_code_bits(float v, float r)
{
    return __float_as_uint(fmaf(v, r, 12582912.0f));
}

// Appends the low nibble of `code_bits` as the new top nibble of `acc`,
// shifting acc right by 4: eight calls in element order leave element 0 in
// bits 0-3 and element 7 in bits 28-31.
__device__ __forceinline__ uint32_t push_nibble(uint32_t acc, uint32_t code_bits)
{
    return __funnelshift_r(acc, code_bits, 4);
}

// Butterflies on two pairs at once with the packed fp32x2 adds of sm_100:
// (a0, a1), (b0, b1) <- (a0 + b0, a1 + b1), (a0 - b0, a1 - b1).
__device__ __forceinline__ void bfly_x2(float &a0, float &a1, float &b0, float &b1)
{
#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ >= 1000)
    asm("{\n\t.reg .b64 ra, rb, rs, rd;\n\t"
        "mov.b64 ra, {%0, %1};\n\t"
        "mov.b64 rb, {%2, %3};\n\t"
        "add.rn.f32x2 rs, ra, rb;\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rs;\n\t"
        "mov.b64 {%2, %3}, rd;\n\t}"
        : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
#else
    float s0 = a0 + b0, s1 = a1 + b1, d0 = a0 - b0, d1 = a1 - b1;
    a0 = s0; a1 = s1; b0 = d0; b1 = d1;
#endif
}

// Unnormalized Walsh-Hadamard transform over register-index bits
// [LO, HI) of a 128-entry array (Sylvester order: H_2 applied along each
// selected bit).  Stages on bit 0 use scalar adds; higher bits use the
// packed pair form on adjacent registers.
template <int LO, int HI>
__device__ __forceinline__ void fwht_bits(float (&v)[128])
{
#pragma unroll
    for (int bit = LO; bit < HI; ++bit) {
        const int h = 1 << bit;
        if (bit == 0) {
#pragma unroll
            for (int i = 0; i < 128; i += 2) {
                float a = v[i], b = v[i + 1];
                v[i] = a + b;
                v[i + 1] = a - b;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 128; i += 2) {
                if ((i & h) == 0)
                    bfly_x2(v[i], v[i + 1], v[i + h], v[i + h + 1]);
            }
        }
    }
}

// Sign flags of 64 fp16 pairs packed into 4 words: pair j uses word j >> 4,
// bit 15 - (j & 15) for its first element and bit 31 - (j & 15) for its
// second, so (word << (j & 15)) & 0x80008000 is the XOR mask of the pair.
template <typename PairElem>
__device__ __forceinline__ void build_sign_words(const int8_t *__restrict__ signs, PairElem first_of_pair,
                                                 uint32_t (&sw)[4])
{
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t v = 0;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int e = first_of_pair(16 * w + k);
            v |= (signs[e] < 0 ? 1u : 0u) << (15 - k);
            v |= (signs[e + 1] < 0 ? 1u : 0u) << (31 - k);
        }
        sw[w] = v;
    }
}

// Flips the fp16 sign bits of pair j (compile-time j) of a half2 word.
__device__ __forceinline__ uint32_t apply_sign_pair(uint32_t pair, const uint32_t (&sw)[4], int j)
{
    return pair ^ ((sw[j >> 4] << (j & 15)) & 0x80008000u);
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t bits)
{
    __half2 h;
    memcpy(&h, &bits, sizeof(h));
    return __half22float2(h);
}

// max(a, b, c): the three-input form of sm_100 (one instruction).
__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// max |v[i]| over 128 values as a tree of three-input maxima (depth 5, not a
// 64-long dependent chain).
__device__ __forceinline__ float absmax128(const float (&v)[128])
{
    float a[43];
#pragma unroll
    for (int j = 0; j < 42; ++j)
        a[j] = max3f(fabsf(v[3 * j]), fabsf(v[3 * j + 1]), fabsf(v[3 * j + 2]));
    a[42] = fmaxf(fabsf(v[126]), fabsf(v[127]));
    float b[15];
#pragma unroll
    for (int j = 0; j < 14; ++j)
        b[j] = max3f(a[3 * j], a[3 * j + 1], a[3 * j + 2]);
    b[14] = a[42];
    float c[5];
#pragma unroll
    for (int j = 0; j < 5; ++j)
        c[j] = max3f(b[3 * j], b[3 * j + 1], b[3 * j + 2]);
    return max3f(max3f(c[0], c[1], c[2]), c[3], c[4]);
}

// (d0, d1) = (a0 * b + c, a1 * b + c) with one packed fp32x2 fused multiply-add.
__device__ __forceinline__ void fma_x2(float a0, float a1, float b, float c, float &d0, float &d1)
{
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
        "mov.b64 rc, {%5, %5};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b), "f"(c));
}

// (d0, d1) = (a0 - c, a1 - c) with one packed fp32x2 subtract.
__device__ __forceinline__ void sub_x2(float a0, float a1, float c, float &d0, float &d1)
{
    asm("{\n\t.reg .b64 ra, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rc, {%4, %4};\n\t"
        "sub.rn.f32x2 rd, ra, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(c));
}

// (d0, d1) = (a0 * b0, a1 * b1) with one packed fp32x2 multiply.
__device__ __forceinline__ void mul_x2(float a0, float a1, float b0, float b1, float &d0, float &d1)
{
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// (acc0, acc1) += (a0 * b, a1 * b) with one packed fp32x2 fused multiply-add.
__device__ __forceinline__ void fma_x2_acc(float a0, float a1, float b, float &acc0, float &acc1)
{
    asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
        "mov.b64 rc, {%0, %1};\n\tfma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(acc0), "+f"(acc1)
        : "f"(a0), "f"(a1), "f"(b));
}

// min(a, b, c): the three-input form of sm_100 (one instruction).
__device__ __forceinline__ float min3f(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float warp_min(float v, int width)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        if (o < width)
            v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ uint32_t warp_sum(uint32_t v, int width)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        if (o < width)
            v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v, int width)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        if (o < width)
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

}  // namespace quarot
