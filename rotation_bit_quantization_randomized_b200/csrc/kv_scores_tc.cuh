// kv_scores_tc.cuh -- the decode-step scores against the INT4 key cache on
// the tensor cores (QuaRot abstract: the KV cache in 4 bits; DuQuant Knowl 12:
// a fixed Hadamard on the query-key product, per-head quantization):
//
//   q'[g]      = (q[g] * diag(s_h)) H_128 / sqrt(128)                (fp32)
//   s[g, t]    = ks[t] * sum_d q'[g, d] kcode[t, d]
//
// for the G query heads g of one KV head h, written as fp32 [B, Hq, T].  The
// contraction is the score half of the fused decode step: per tile of 128
// tokens one M 128 x N 16 (32 for G = 16) x K 128 tcgen05.mma kind::f16 group
// with fp32 accumulation in tensor memory, on exact operands (the codes are
// small integers, the fp32 query is split into fp16 hi and lo rows with a
// per-head power of two, dec_rotate_queries), so only the fp32 sums round.
//
// A CTA takes `tiles_per_cta` consecutive tiles of one (batch, KV head).
// Four compute warps (one thread per token) convert each tile's key codes
// into one of two fp16 tiles and hand it to a fifth warp that issues the
// MMAs into one of two accumulators; while the MMAs of tile j run, the
// compute warps convert tile j + 1, then read tile j's scores (lane = token)
// and store them, G coalesced rows.  Each thread loads its token's code row
// of the next tile into registers one tile ahead.  Every wait is bounded.
#pragma once

#include "kv_decode_tc.cuh"

namespace quarot {

template <int G>
struct ScShape {
    static constexpr int NP = DecShape<G>::NP;
    static constexpr int kTmemCols = 2 * NP <= 32 ? 32 : 64;   // two accumulators of NP columns
    static constexpr int kTileOff = 0;                         // two key tiles of 32 KB
    static constexpr int kBqOff = 65536;                       // B_q: 2 panels of NP rows x 128 B
    static constexpr int kMiscOff = kBqOff + 2 * NP * 128;
    // misc: "key tile ready" (8 per buffer), "scores done" (8 per
    // accumulator), drain (8), tmem slot (4), abort flag (4), then inv_qs[G]
    static constexpr int kIqOff = kMiscOff + 64;
    static constexpr int kBytes = kIqOff + 4 * G + 1024;
    static_assert(kBqOff % 1024 == 0 && kMiscOff % 16 == 0, "alignment");
};

template <int G>
__global__ void __launch_bounds__(kDecThreads, G <= 8 ? 3 : 2)
kv_scores_tc_kernel(const __half *__restrict__ q,        // [B, Hq, 128]
                    const int8_t *__restrict__ signs,    // [Hkv, 128]
                    const uint8_t *__restrict__ kq,      // [B, T, Hkv, 64 bytes]
                    const __half *__restrict__ ks,       // [B, T, Hkv]
                    int64_t T, int Hkv, int tiles_per_cta,
                    float *__restrict__ scores)          // [B, Hq, T]
{
    using S = ScShape<G>;
    constexpr int NP = S::NP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *bq = smem + S::kBqOff;
    // one barrier per key buffer and per accumulator: tile j uses index j % 2
    // and phase j / 2, so no barrier can complete a phase twice before its
    // waiter has seen the first (the compute warps hand over tile j + 1
    // before they wait for tile j's scores)
    auto bar_k = [&](int j) { return smem_u32(smem + S::kMiscOff + 8 * (j & 1)); };
    auto bar_s = [&](int j) { return smem_u32(smem + S::kMiscOff + 16 + 8 * (j & 1)); };
    auto phase = [](int j) { return (uint32_t)(j >> 1) & 1u; };
    const uint32_t bar_drain = smem_u32(smem + S::kMiscOff + 32);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kMiscOff + 40);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + S::kMiscOff + 44);
    float *inv_qs = reinterpret_cast<float *>(smem + S::kIqOff);

    const int h = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int Hq = Hkv * G;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool compute = warp < kDecCompute / 32;
    const int64_t all_tiles = (T + kDecTile - 1) / kDecTile;
    const int64_t j0 = (int64_t)blockIdx.x * tiles_per_cta;
    const int ntiles = (int)max((int64_t)0, min(j0 + tiles_per_cta, all_tiles) - j0);

    if (tid == 0) {
        mbar_init(bar_k(0), kDecCompute);
        mbar_init(bar_k(1), kDecCompute);
        mbar_init(bar_s(0), 1);
        mbar_init(bar_s(1), 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0u;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
        tmem_relinquish();
    }
    auto tile_of = [&](int j) { return smem + S::kTileOff + (j & 1) * 32768; };
    // token t of local tile j: its code row into registers (zeros past the end)
    auto load_row = [&](int j, uint4 (&w)[4]) {
        const int64_t t = (j0 + j) * kDecTile + tid;
        if (j < ntiles && t < T) {
            const uint4 *p = reinterpret_cast<const uint4 *>(kq + ((b * T + t) * Hkv + h) * 64);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                w[c] = __ldg(p + c);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                w[c] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    // token t of local tile j, two tiles ahead of its register load: its code
    // row and scale into L2
    auto prefetch_tile = [&](int j) {
        const int64_t t = (j0 + j) * kDecTile + tid;
        if (j < ntiles && t < T) {
            const int64_t r = (b * T + t) * Hkv + h;
            prefetch_l2(kq + r * 64);
            prefetch_l2(ks + r);
        }
    };
    uint4 krow[4];
    if (compute) {
        load_row(0, krow);
        prefetch_tile(1);
        dec_rotate_queries<G>(q + (b * Hq + (int64_t)h * G) * 128, signs + h * 128, bq, inv_qs, tid);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (!compute) {
        // ---- warp 4: the score MMAs of every tile, into accumulator j % 2
        constexpr uint32_t idesc_s = idesc_f16(128, NP);
#pragma unroll 1
        for (int j = 0; j < ntiles; ++j) {
            if (!dec_wait(bar_k(j), phase(j)) || *abort_flag)
                break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kt = smem_u32(tile_of(j));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16_ss(tmem + (j & 1) * NP, desc_kmajor_sw128(kt + 16384 * (kk >> 2) + 32 * (kk & 3)),
                                desc_kmajor_sw128(smem_u32(bq) + NP * 128 * (kk >> 2) + 32 * (kk & 3)), idesc_s,
                                kk > 0 ? 1u : 0u);
                umma_commit(bar_s(j));
            }
            __syncwarp();
        }
    } else {
        float inv_q[G];
#pragma unroll
        for (int g = 0; g < G; ++g)
            inv_q[g] = inv_qs[g];
        const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
        auto load_scale = [&](int j) {
            const int64_t t = (j0 + j) * kDecTile + tid;
            return (j < ntiles && t < T) ? __half2float(ks[(b * T + t) * Hkv + h]) : 0.f;
        };
        // scores of local tile j (its MMAs complete) from accumulator j % 2 to HBM
        auto store_tile = [&](int j, float ksv) {
            tc_fence_after();
            uint32_t d[NP];
            if constexpr (NP == 16) {
                uint32_t (&d16)[16] = *reinterpret_cast<uint32_t (*)[16]>(d);
                tmem_ld16(lane_base + (j & 1) * NP, d16);
                tmem_wait_ld16(d16);
            } else {
                uint32_t (&d32)[32] = *reinterpret_cast<uint32_t (*)[32]>(d);
                tmem_ld32(lane_base + (j & 1) * NP, d32);
                tmem_wait_ld(d32);
            }
            const int64_t t = (j0 + j) * kDecTile + tid;
            if (t < T) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float x = (__uint_as_float(d[g]) + __uint_as_float(d[G + g]) * (1.0f / 2048.0f)) * inv_q[g];
                    float *dst = scores + (b * Hq + (int64_t)h * G + g) * T + t;
                    if (QUAROT_IN_RANGE(dst, 4, scores, (int64_t)gridDim.z * Hq * T * 4))
                        *dst = x * ksv;
                }
            }
        };
        bool ok = true;
        float ks_cur = load_scale(0), ks_prev = 0.f;
#pragma unroll 1
        for (int j = 0; j < ntiles; ++j) {
            const float ks_next = load_scale(j + 1);
            // ---- tile j's keys: convert (tile j - 2's MMAs, which read this
            // buffer, were waited for in the previous iteration), hand over
            dec_convert_row(krow, tile_of(j), tid);
            load_row(j + 1, krow);
            prefetch_tile(j + 2);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_k(j));
            // ---- tile j - 1's scores, whose MMAs ran during the conversion
            if (j > 0) {
                if (!(ok = dec_bar_and(dec_wait(bar_s(j - 1), phase(j - 1)))))
                    break;
                store_tile(j - 1, ks_prev);
                tc_fence_before();
            }
            ks_prev = ks_cur;
            ks_cur = ks_next;
        }
        if (ok && ntiles > 0) {
            if ((ok = dec_bar_and(dec_wait(bar_s(ntiles - 1), phase(ntiles - 1)))))
                store_tile(ntiles - 1, ks_prev);
        }
        if (!ok) {
            // the MMA warp may wait for a key tile that will not come (the next
            // one, in either buffer): release it
            *abort_flag = 1u;
            mbar_arrive(bar_k(0));
            mbar_arrive(bar_k(1));
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
