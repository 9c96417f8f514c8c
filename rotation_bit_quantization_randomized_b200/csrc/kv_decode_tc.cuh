// kv_decode_tc.cuh -- one fused decode step of attention over the INT4 KV
// cache on the tensor cores: the query rotation, the query-key scores, the
// softmax and the product with the value cache in one kernel, so that the
// key and value codes are read once and the scores never reach global memory
// (QuaRot abstract: the KV cache in 4 bits and the rotation applied to
// aspects of the attention mechanism; DuQuant Knowl 12: a fixed Hadamard on
// the query-key product, per-head quantization, the softmax output times the
// quantized values; QuaRot summary, References: FlashInfer):
//
//   q'[g]      = (q[g] * diag(s_h)) H_128 / sqrt(128)                (fp32)
//   s[g, t]    = ks[t] * sum_d q'[g, d] kcode[t, d]
//   p[g, t]    = softmax over t of s[g, t] / sqrt(128)
//   out[g, d]  = sum_t p[g, t] vs[t] vcode[t, d]
//
// for the G query heads g of one KV head h.  Both contractions run as
// tcgen05.mma kind::f16 with fp32 accumulation in tensor memory, on exact
// operands: the codes are small integers (exact in fp16), and the fp32 query
// and weights are split into two fp16 rows each, hi = fp16(x 2^e) and lo =
// fp16((x 2^e - hi) 2^11), with a per-head power of two e, so that hi + lo
// 2^-11 carries 22 bits of x and every product with a code is exact:
//   scores:  D_s[t][n] = sum_p A_k[t][p] B_q[n][p]    (M 128 tokens, N rows n of B_q, K 128)
//   values:  D_o[p][n] = sum_t A_v[p][t] B_w[n][t]    (M 128 dims, N rows n of B_w, K 128 tokens)
// where row n < G of B is head n's hi part and row G + n its lo part (rows
// past 2 G, when G < 8, only feed accumulator columns that are never read).  A_k
// (key codes, K-major) and A_v (value codes, MN-major: the dims of a token
// are contiguous) have the same 128 x 128 fp16 tile layout in shared memory
// (two tiles), so one conversion routine serves both; it emits the dims of every group of
// four in the order (0, 2, 1, 3) (two nibble bytes become a low-nibble and a
// high-nibble half2 word), and the query rows use the same order, so each dot
// product is unchanged and output lane p holds dim d(p).
//
// A cluster of S CTAs covers one (batch, KV head); CTA r walks its slice of
// the tokens in tiles of 128 with the running-maximum softmax (in base 2: the
// scores carry the factor log2(e) / sqrt(128) and the exponentials are exp2):
// per tile the key codes are converted and multiplied, the value codes are
// converted while those MMAs run, the 128 threads (one per token) read their
// scores, the tile maximum updates the running maximum m and the sum l, the
// value accumulator D_o is rescaled in tensor memory when m grows, the
// weights e * vs (one power-of-two scale for the whole slice, from its
// largest value scale) are written as B_w, and the value MMAs into D_o run
// while the next tile's keys are converted.  Each thread loads its token's
// key and value rows of the next tile into registers one tile ahead.  At the
// end the CTAs of the cluster combine their (m, l, acc) through distributed
// shared memory: out = sum_r exp(m_r - M) acc_r / sum_r exp(m_r - M) l_r,
// M = max_r m_r.  Several CTAs share an SM (about 73 KB of shared memory and
// 32 or 64 tensor-memory columns each), so one CTA's conversions overlap
// another's waits.  Every wait is bounded.
#pragma once

#include "common.cuh"
#include "kron_quant.cuh"
#include "kv_attend.cuh"
#include "tc_ptx.cuh"

namespace quarot {

constexpr int kDecCompute = 128;                 // warps 0-3: one thread per token of a tile
constexpr int kDecThreads = kDecCompute + 32;    // warp 4 issues the MMAs
constexpr int kDecTile = 128;                    // tokens per tile
constexpr int kDecMaxSplit = 8;
constexpr uint64_t kDecWaitLimitNs = 2000000000ull;

template <int G>
struct DecShape {
    static constexpr int NP = G <= 8 ? 16 : 32;            // MMA N: G hi rows, G lo rows, zero padding
    static constexpr int kTmemCols = G <= 8 ? 32 : 64;     // D_s at column 0, D_o at column NP
    static constexpr int kKTileOff = 0;                    // key tile: 2 panels of 128 rows x 128 B
    static constexpr int kVTileOff = 32768;                // value tile, the same shape
    static constexpr int kBqOff = 65536;                   // B_q: 2 panels of NP rows x 128 B
    static constexpr int kBwOff = kBqOff + 2 * NP * 128;   // B_w: the same shape
    static constexpr int kMiscOff = kBwOff + 2 * NP * 128;
    // misc: mbarriers "scores done" (8), tmem slot (4), pad (4), drain (8),
    // "values done" (8), "key tile ready" (8), "value tile ready" (8), abort
    // flag (4), pad, then floats:
    //   red[4][G + 1]  per-warp tile maxima of each head's scores
    //   m[G], l[G], lpart[4][G], inv_qs[G], vmx[4]
    static constexpr int kRedOff = kMiscOff + 64;
    static constexpr int kQmaxOff = kRedOff + 4 * (G + 1) * 4;
    static constexpr int kMOff = kQmaxOff + 4 * G * 4;
    static constexpr int kLOff = kMOff + G * 4;
    static constexpr int kLpOff = kLOff + G * 4;
    static constexpr int kIqOff = kLpOff + 4 * G * 4;       // 1 / 2^e of each head's query
    static constexpr int kVmOff = kIqOff + G * 4;           // per-warp maxima of the slice's value scales
    static constexpr int kBytes = kVmOff + 16 + 1024;
    // the value tile is free after the last tile: there every CTA of the
    // cluster receives, for the heads it finishes, the other CTAs' partial
    // results: recv[rank][slot][128] fp32, then their m and l
    static constexpr int kOwnMax = G;                          // heads one CTA finishes, at most
    static constexpr int kRecvOff = kVTileOff;
    static constexpr int kRecvMlOff = kVTileOff + 16384;
    static_assert(kBqOff % 1024 == 0 && kBwOff % 1024 == 0 && kMiscOff % 16 == 0, "alignment");
};

// dim held by position p of a converted row: (0, 2, 1, 3) within each group of four
__host__ __device__ constexpr int dec_dim(int p) { return (p & ~3) | ((p & 1) << 1) | ((p >> 1) & 1); }

// Converts one token's 64 bytes of packed codes (four uint4) into its row of
// the fp16 tile (row t; 128-byte-swizzled chunks in two 64-column panels).
// Bytes j, j + 1 -> x = b_j | b_{j+1} << 16 (biased by XOR 0x88: u = c + 8);
// low nibbles: half2 (0x6400 | u) - 1032 = c; high nibbles: half2 (0x6400 |
// 16 u) * 1/16 - 72 = c; both exact.
__device__ __forceinline__ void dec_convert_row(const uint4 (&w)[4], uint8_t *tile, int t)
{
    const __half2 kSub = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));   // 1032
    const __half2 kMul = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));   // 1/16
    const __half2 kOff = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));   // -72
#pragma unroll
    for (int c = 0; c < 16; ++c) {                      // 16-byte output chunk c: dims 8c .. 8c + 7
        const uint4 in = w[c >> 2];
        const uint32_t word = ((c & 3) == 0 ? in.x : (c & 3) == 1 ? in.y : (c & 3) == 2 ? in.z : in.w) ^ 0x88888888u;
        uint32_t o[4];
#pragma unroll
        for (int hpair = 0; hpair < 2; ++hpair) {
            const uint32_t x = __byte_perm(word, 0u, hpair == 0 ? 0x4140 : 0x4342);
            const uint32_t lo = (x & 0x000F000Fu) | 0x64006400u;
            const uint32_t hi = (x & 0x00F000F0u) | 0x64006400u;
            __half2 hl, hh;
            memcpy(&hl, &lo, 4);
            memcpy(&hh, &hi, 4);
            hl = __hsub2(hl, kSub);
            hh = __hfma2(hh, kMul, kOff);
            memcpy(&o[2 * hpair], &hl, 4);
            memcpy(&o[2 * hpair + 1], &hh, 4);
        }
        const int panel = c >> 3, ch = c & 7;
        *reinterpret_cast<uint4 *>(tile + panel * 16384 + t * 128 + ((ch ^ (t & 7)) << 4)) =
            make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Writes x (fp32) as the hi / lo fp16 pair of rows n and n + G at column k of
// a K-major B tile (two 64-column panels of NP rows x 128 B, 128-byte swizzle).
template <int G>
__device__ __forceinline__ void dec_put_split(uint8_t *b, int n, int k, float xs)
{
    constexpr int NP = DecShape<G>::NP;
    const __half hi = __float2half_rn(xs);
    const __half lo = __float2half_rn((xs - __half2float(hi)) * 2048.0f);
    const int panel = k >> 6, kk = k & 63;
    auto at = [&](int row) {
        return reinterpret_cast<__half *>(b + panel * (NP * 128) + row * 128 + ((((kk >> 3) ^ (row & 7))) << 4)) +
               (kk & 7);
    };
    *at(n) = hi;
    *at(G + n) = lo;
}

// The maxima over a warp's 32 tokens of each of the G heads' scores, into
// red_w[g].  Halving exchanges: at the level of lane bit m the two partners
// keep complementary halves of the values still held, each taking the larger
// of its own and the partner's value for the half it keeps; after log2(G)
// levels every lane holds one head's partial maximum, and plain butterfly
// levels over the remaining lane bits finish it (G - 1 + 5 - log2(G)
// shuffles instead of 5 G).
template <int G>
__device__ __forceinline__ void dec_tile_max(const float (&s)[G], float *red_w, int lane)
{
    constexpr int L = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : 4;
    static_assert((1 << L) == G, "G is a power of two up to 16");
    float v[G];
#pragma unroll
    for (int i = 0; i < G; ++i)
        v[i] = s[i];
    int g = 0;
#pragma unroll
    for (int lv = 0; lv < L; ++lv) {
        const int mask = 16 >> lv;
        const int half = G >> (lv + 1);
        const bool upper = (lane & mask) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[half + i];
            const float keep = upper ? v[half + i] : v[i];
            v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, mask));
        }
        g += upper ? half : 0;
    }
#pragma unroll
    for (int mask = 16 >> L; mask >= 1; mask >>= 1)
        v[0] = fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], mask));
    if ((lane & ((32 >> L) - 1)) == 0)
        red_w[g] = v[0];
}

// 2^x by the SM's base-2 exponential instruction (ex2.approx, subnormal
// results flushed to zero): the softmax weights and their rescale factors.
// Its relative error is a few units in the last place of fp32; a weight's
// error moves the normalized output by at most twice that relative error
// times the largest value, and a rescale factor's error cancels, because the
// accumulator and the sum of weights are scaled by the same computed factor.
__device__ __forceinline__ float dec_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Brings the line holding p into L2 ahead of its load (no register, no
// wait); only issued for addresses inside the caches.
__device__ __forceinline__ void prefetch_l2(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Barrier of the four compute warps (named barrier 1, 128 threads); the MMA
// warp never takes part.
__device__ __forceinline__ void dec_bar_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// The same barrier, returning the AND of every compute thread's predicate.
__device__ __forceinline__ bool dec_bar_and(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Store of a float to the shared memory of a CTA of the cluster (a
// shared::cluster address from mapa_shared).
__device__ __forceinline__ void st_dsmem_f32(uint32_t cluster_addr, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}

// Bounded wait for the phase of `bar` with the given parity; false (and the
// device status set) when the limit passed.
__device__ __forceinline__ bool dec_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kDecWaitLimitNs) {
            record_timeout();
            return false;
        }
    }
    return true;
}

// Power of two 2^e that brings max|x| (> 0) into [2^14, 2^15): hi parts then
// stay far from fp16 overflow and lo parts keep 11 more bits.  Built from the
// exponent bits, so 2^e and its inverse are exact; 1 for a zero maximum.
__device__ __forceinline__ float dec_pow2_scale(float amax, float &inv)
{
    const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFFu);     // biased exponent of amax
    if (!(amax > 0.f) || ex == 0xFF) {
        inv = 1.0f;
        return 1.0f;
    }
    const int e = min(max(14 - (ex - 127), -126), 126);
    inv = __uint_as_float((uint32_t)(127 - e) << 23);
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

// The G queries of one KV head rotated and written as the B operand of the
// score MMAs (threads 0-127; 16 threads per query, 8 elements each: bits 0-2
// of the element index in registers, bits 3-6 through half-warp shuffles):
//   q'[g] = (q[g] * diag(s_h)) H_128 / sqrt(128)  in fp32,
// then per query the power of two 2^e of dec_pow2_scale and its hi / lo fp16
// rows (dec_put_split) in the converted dim order; inv_qs[g] = 2^-e.
// qg: the G query rows [G][128] fp16; sg: the head's 128 signs.
template <int G>
__device__ __forceinline__ void dec_rotate_queries(const __half *__restrict__ qg, const int8_t *__restrict__ sgn,
                                                   uint8_t *bq, float *inv_qs, int tid)
{
    const float kInvSqrtD = 0.08838834764831845f;
    const int p = tid & 15;
    const int8_t *sg = sgn + 8 * p;
#pragma unroll
    for (int g0 = 0; g0 < G; g0 += kDecCompute / 16) {
        const int g = g0 + (tid >> 4);
        const bool gv = G % (kDecCompute / 16) == 0 || g < G;
        const uint4 raw = gv ? *reinterpret_cast<const uint4 *>(qg + (int64_t)g * 128 + 8 * p)
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
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[i] *= kInvSqrtD;
            mx = fmaxf(mx, fabsf(v[i]));
        }
#pragma unroll
        for (int lb = 1; lb < 16; lb <<= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, lb));
        float inv;
        const float sc = dec_pow2_scale(mx, inv);
        if (gv) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dec_put_split<G>(bq, g, 8 * p + dec_dim(i), v[i] * sc);
            if (p == 0)
                inv_qs[g] = inv;
        }
    }
}

template <int G>
__global__ void __launch_bounds__(kDecThreads, G <= 8 ? 3 : 2)
kv_decode_tc_kernel(const __half *__restrict__ q,        // [B, Hq, 128]
                    const int8_t *__restrict__ signs,    // [Hkv, 128]
                    const uint8_t *__restrict__ kq,      // [B, T, Hkv, 64 bytes]
                    const __half *__restrict__ ks,       // [B, T, Hkv]
                    const uint8_t *__restrict__ vq,      // [B, T, Hkv, 64 bytes]
                    const __half *__restrict__ vs,       // [B, T, Hkv]
                    int64_t T, int Hkv, float *__restrict__ out)   // [B, Hq, 128]
{
    using S = DecShape<G>;
    constexpr int NP = S::NP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ktile = smem + S::kKTileOff;
    uint8_t *vtile = smem + S::kVTileOff;
    uint8_t *bq = smem + S::kBqOff;
    uint8_t *bw = smem + S::kBwOff;
    const uint32_t bar_s = smem_u32(smem + S::kMiscOff);          // score MMAs done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOff + 8);
    const uint32_t bar_drain = smem_u32(smem + S::kMiscOff + 16);
    const uint32_t bar_o = smem_u32(smem + S::kMiscOff + 24);     // value MMAs done
    const uint32_t bar_k = smem_u32(smem + S::kMiscOff + 32);     // key tile and B_q ready
    const uint32_t bar_v = smem_u32(smem + S::kMiscOff + 40);     // value tile, B_w, D_o ready
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + S::kMiscOff + 48);
    float *red = reinterpret_cast<float *>(smem + S::kRedOff);      // [4][G + 1]
    float *lpart = reinterpret_cast<float *>(smem + S::kLpOff);     // [4][G]
    float *inv_qs = reinterpret_cast<float *>(smem + S::kIqOff);    // [G]
    float *vmx = reinterpret_cast<float *>(smem + S::kVmOff);       // [4]

    const int nsplit = gridDim.x;
    const int r = blockIdx.x;
    const int h = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int Hq = Hkv * G;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool compute = warp < kDecCompute / 32;
    // softmax in base 2: scores / sqrt(128) times log2(e), then exp2
    const float kScoreMul = 0.08838834764831845f * 1.4426950408889634f;
    const int64_t slice = (T + nsplit - 1) / nsplit;
    const int64_t ts = min(T, (int64_t)r * slice);
    const int64_t te = min(T, ts + slice);
    const int ntiles = (int)((te - ts + kDecTile - 1) / kDecTile);
    const int n_own = (G + nsplit - 1) / nsplit;       // heads this CTA finishes: r, r + nsplit, ...

    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        mbar_init(bar_drain, 1);
        mbar_init(bar_k, kDecCompute);
        mbar_init(bar_v, kDecCompute);
        *abort_flag = 0u;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
        tmem_relinquish();
    }
    // thread t holds token t's key and value rows of the next tile in
    // registers: loaded one tile ahead, converted into the tiles when due
    auto load_row = [&](const uint8_t *src, int j, uint4 (&w)[4]) {
        const int64_t t = ts + (int64_t)j * kDecTile + tid;
        if (j < ntiles && t < te) {
            const uint4 *p = reinterpret_cast<const uint4 *>(src + ((b * T + t) * Hkv + h) * 64);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                w[c] = __ldg(p + c);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                w[c] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    // token t of tile j, two tiles ahead of its register load: its code rows
    // and scales into L2
    auto prefetch_tile = [&](int j) {
        const int64_t t = ts + (int64_t)j * kDecTile + tid;
        if (j < ntiles && t < te) {
            const int64_t r = (b * T + t) * Hkv + h;
            prefetch_l2(kq + r * 64);
            prefetch_l2(vq + r * 64);
            prefetch_l2(ks + r);
            prefetch_l2(vs + r);
        }
    };
    uint4 krow[4], vrow[4];
    if (compute) {
        load_row(kq, 0, krow);
        load_row(vq, 0, vrow);
        prefetch_tile(1);
        // ---- the slice's largest value scale (the weights e * vs never
        // exceed it, so one power-of-two scale serves every tile of the slice)
        float vm = 0.f;
#pragma unroll 4
        for (int j = 0; j < ntiles; ++j) {
            const int64_t t = ts + (int64_t)j * kDecTile + tid;
            if (t < te)
                vm = fmaxf(vm, __half2float(vs[(b * T + t) * Hkv + h]));
        }
        vm = warp_max(vm, 32);
        if (lane == 0)
            vmx[warp] = vm;
        dec_rotate_queries<G>(q + (b * Hq + (int64_t)h * G) * 128, signs + h * 128, bq, inv_qs, tid);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (!compute) {
        // ---- warp 4: the MMAs of every tile, each once its operands are in
        // place (lane 0 issues; the warp waits together)
        constexpr uint32_t idesc_s = idesc_f16(128, NP);
        constexpr uint32_t idesc_o = idesc_f16(128, NP) | (1u << 15);    // A (values) MN-major
#pragma unroll 1
        for (int j = 0; j < ntiles; ++j) {
            if (!dec_wait(bar_k, j & 1) || *abort_flag)
                break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16_ss(tmem, desc_kmajor_sw128(smem_u32(ktile) + 16384 * (kk >> 2) + 32 * (kk & 3)),
                                desc_kmajor_sw128(smem_u32(bq) + NP * 128 * (kk >> 2) + 32 * (kk & 3)), idesc_s,
                                kk > 0 ? 1u : 0u);
                umma_commit(bar_s);
            }
            __syncwarp();
            if (!dec_wait(bar_v, j & 1) || *abort_flag)
                break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16_ss(tmem + NP, desc_mnmajor_sw128(smem_u32(vtile) + 2048 * kk, 16384),
                                desc_kmajor_sw128(smem_u32(bw) + NP * 128 * (kk >> 2) + 32 * (kk & 3)), idesc_o,
                                (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar_o);
            }
            __syncwarp();
        }
    }

    float inv_wsc = 1.0f;
    float m_run[G];                                   // running maximum (base-2 units)
    float lsum[G];                                    // this thread's share of sum exp2
    uint32_t dout[NP];                                // the CTA's value accumulator, lane = dim
#pragma unroll
    for (int g = 0; g < G; ++g) {
        lsum[g] = 0.f;
        m_run[g] = -INFINITY;
    }
    bool ok = true;
    if (compute) {
        const float wsc = dec_pow2_scale(fmaxf(fmaxf(vmx[0], vmx[1]), fmaxf(vmx[2], vmx[3])), inv_wsc);
        float inv_q[G];
#pragma unroll
        for (int g = 0; g < G; ++g)
            inv_q[g] = inv_qs[g];
        const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
        // the latest commit to `bar` has completed, for every compute thread
        auto wait_all = [&](uint32_t bar, int phase) { return dec_bar_and(dec_wait(bar, phase & 1)); };
        // scales of token t of tile j (loaded one tile ahead)
        auto load_scales = [&](int j, float &ksv, float &vsv) {
            const int64_t t = ts + (int64_t)j * kDecTile + tid;
            const bool tv = j < ntiles && t < te;
            ksv = tv ? __half2float(ks[(b * T + t) * Hkv + h]) : 0.f;
            vsv = tv ? __half2float(vs[(b * T + t) * Hkv + h]) : 0.f;
        };
        float ks_next, vs_next;
        load_scales(0, ks_next, vs_next);
        // Per tile j: keys converted -> (warp 4 issues the score MMAs) ->
        // (value MMAs of tile j - 1 done) values converted while the score
        // MMAs run -> scores, softmax weights -> (warp 4 issues the value
        // MMAs, which run while the next tile's keys are converted).  The
        // key tile is free at the top of an iteration: its MMAs were waited
        // for before the scores were read.
#pragma unroll 1
        for (int j = 0; j < ntiles; ++j) {
            const int64_t t = ts + (int64_t)j * kDecTile + tid;
            const bool tv = t < te;
            const float ksv = ks_next, vsv = vs_next;
            load_scales(j + 1, ks_next, vs_next);
            // ---- keys: convert, hand to the MMA warp
            dec_convert_row(krow, ktile, tid);
            load_row(kq, j + 1, krow);
            prefetch_tile(j + 2);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_k);
            // ---- values: the previous tile's value MMAs are done with the
            // value tile, B_w and D_o; convert while the score MMAs run
            if (j > 0 && !(ok = wait_all(bar_o, j - 1)))
                break;
            dec_convert_row(vrow, vtile, tid);
            load_row(vq, j + 1, vrow);
            if (!(ok = wait_all(bar_s, j)))
                break;
            tc_fence_after();
            // ---- scores of token t (lane t of D_s), the tile maxima
            float sc[G];
            {
                uint32_t d[NP];
                if constexpr (NP == 16) {
                    uint32_t (&d16)[16] = *reinterpret_cast<uint32_t (*)[16]>(d);
                    tmem_ld16(lane_base, d16);
                    tmem_wait_ld16(d16);
                } else {
                    uint32_t (&d32)[32] = *reinterpret_cast<uint32_t (*)[32]>(d);
                    tmem_ld32(lane_base, d32);
                    tmem_wait_ld(d32);
                }
                // score / sqrt(128) in base-2 units: (hi + lo 2^-11) 2^-e ks / sqrt(128) log2(e)
                const float km = ksv * kScoreMul;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float x = (__uint_as_float(d[g]) + __uint_as_float(d[G + g]) * (1.0f / 2048.0f)) * inv_q[g];
                    sc[g] = tv ? x * km : -INFINITY;
                }
            }
            dec_tile_max<G>(sc, red + warp * (G + 1), lane);
            dec_bar_sync();
            // ---- softmax: all tile maxima first, then the arithmetic, then
            // the stores of the weights (so that no load waits behind a store)
            float tmax[G];
#pragma unroll
            for (int g = 0; g < G; ++g)
                tmax[g] = fmaxf(fmaxf(red[g], red[(G + 1) + g]), fmaxf(red[2 * (G + 1) + g], red[3 * (G + 1) + g]));
            float beta[G], wgt[G];                    // rescale of the value accumulator, weights
            bool rescale = false;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float m_new = fmaxf(m_run[g], tmax[g]);
                const float alpha = m_run[g] == -INFINITY ? 0.f : dec_exp2(m_run[g] - m_new);
                beta[g] = alpha;
                rescale |= j > 0 && alpha != 1.0f;
                const float e = tv ? dec_exp2(sc[g] - m_new) : 0.f;
                lsum[g] = lsum[g] * alpha + e;
                m_run[g] = m_new;
                wgt[g] = e * vsv * wsc;
            }
#pragma unroll
            for (int g = 0; g < G; ++g)
                dec_put_split<G>(bw, g, tid, wgt[g]);
            // the value accumulator in the units of this tile (lane = dim)
            if (rescale) {
                uint32_t d[NP];
                if constexpr (NP == 16) {
                    uint32_t (&d16)[16] = *reinterpret_cast<uint32_t (*)[16]>(d);
                    tmem_ld16(lane_base + NP, d16);
                    tmem_wait_ld16(d16);
                } else {
                    uint32_t (&d32)[32] = *reinterpret_cast<uint32_t (*)[32]>(d);
                    tmem_ld32(lane_base + NP, d32);
                    tmem_wait_ld(d32);
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    d[g] = __float_as_uint(__uint_as_float(d[g]) * beta[g]);
                    d[G + g] = __float_as_uint(__uint_as_float(d[G + g]) * beta[g]);
                }
                if constexpr (NP == 16)
                    tmem_st16(lane_base + NP, *reinterpret_cast<uint32_t (*)[16]>(d));
                else
                    tmem_st32(lane_base + NP, *reinterpret_cast<uint32_t (*)[32]>(d));
                tmem_wait_st();
            }
            // ---- hand the value tile, B_w and D_o to the MMA warp
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_v);
        }
        if (!ok) {
            // the MMA warp may wait for this tile's values: release it
            *abort_flag = 1u;
            mbar_arrive(bar_v);
        }
        if (ok && ntiles > 0)
            ok = wait_all(bar_o, ntiles - 1);
        // ---- this CTA's partial result: the accumulator (lane = dim), m, l
        if (ok && ntiles > 0) {
            tc_fence_after();
            if constexpr (NP == 16) {
                tmem_ld16(lane_base + NP, *reinterpret_cast<uint32_t (*)[16]>(dout));
                tmem_wait_ld16(*reinterpret_cast<uint32_t (*)[16]>(dout));
            } else {
                tmem_ld32(lane_base + NP, *reinterpret_cast<uint32_t (*)[32]>(dout));
                tmem_wait_ld(*reinterpret_cast<uint32_t (*)[32]>(dout));
            }
        } else {
#pragma unroll
            for (int i = 0; i < NP; ++i)
                dout[i] = 0u;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float ls = warp_sum_f(lsum[g]);
            if (lane == 0)
                lpart[warp * G + g] = ls;
        }
        dec_bar_sync();
    }

    // ---- combine the slices of the cluster.  After the first cluster
    // barrier every CTA's loop is over and its value tile free; each CTA then
    // stores its partial result for head g into the value tile of the CTA
    // that finishes g (rank g mod nsplit, slot g div nsplit); after the
    // second barrier each CTA combines what it received:
    // out = sum_r exp2(m_r - M) acc_r / sum_r exp2(m_r - M) l_r, M = max_r m_r.
    float *recv = reinterpret_cast<float *>(smem + S::kRecvOff);         // [nsplit][n_own][128]
    float *recv_ml = reinterpret_cast<float *>(smem + S::kRecvMlOff);    // [2][nsplit][n_own]
    cluster_sync_all();
    if (compute) {
        const int dim = dec_dim(tid);
        const bool have = ok && ntiles > 0;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int owner = g % nsplit, slot = g / nsplit;
            const float v = (__uint_as_float(dout[g]) + __uint_as_float(dout[G + g]) * (1.0f / 2048.0f)) * inv_wsc;
            float *slot_p = recv + (r * n_own + slot) * 128 + dim;
            if (QUAROT_IN_RANGE(slot_p, 4, recv, S::kRecvMlOff - S::kRecvOff))
                st_dsmem_f32(mapa_shared(smem_u32(slot_p), owner), v);
        }
        if (tid < G) {
            const int g = tid, owner = g % nsplit, slot = g / nsplit;
            const float l = have ? (lpart[g] + lpart[G + g]) + (lpart[2 * G + g] + lpart[3 * G + g]) : 0.f;
            float m = -INFINITY;                     // m_run[g], selected without indexing by a variable
#pragma unroll
            for (int i = 0; i < G; ++i)
                m = (have && i == g) ? m_run[i] : m;
            st_dsmem_f32(mapa_shared(smem_u32(recv_ml + r * n_own + slot), owner), m);
            st_dsmem_f32(mapa_shared(smem_u32(recv_ml + nsplit * n_own + r * n_own + slot), owner), l);
        }
    }
    cluster_sync_all();
    if (compute) {
        for (int slot = 0; slot < n_own; ++slot) {
            const int g = r + slot * nsplit;
            if (g >= G)
                break;
            float M = -INFINITY;
            for (int qq = 0; qq < nsplit; ++qq)
                M = fmaxf(M, recv_ml[qq * n_own + slot]);
            float num = 0.f, den = 0.f;
            for (int qq = 0; qq < nsplit; ++qq) {
                const float mq = recv_ml[qq * n_own + slot];
                const float f = mq == -INFINITY ? 0.f : exp2f(mq - M);
                den = fmaf(f, recv_ml[nsplit * n_own + qq * n_own + slot], den);
                num = fmaf(f, recv[(qq * n_own + slot) * 128 + tid], num);
            }
            float *dst = out + (b * Hq + (int64_t)h * G + g) * 128 + tid;
            if (QUAROT_IN_RANGE(dst, 4, out, (int64_t)gridDim.z * Hq * 128 * 4))
                *dst = num / den;
        }
    }
    // every MMA this CTA issued has completed (also after a timeout)
    if (warp == kDecCompute / 32 && lane == 0) {
        umma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0, kDecWaitLimitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, S::kTmemCols);
    }
}

}  // namespace quarot
