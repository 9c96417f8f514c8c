// kv_quant.cuh -- INT4 KV-cache write with the rows staged by the copy engine
// (QuaRot abstract: the KV cache in 4 bits; DuQuant Knowl 12: a fixed
// Hadamard of size 128 on the query-key product, per-head quantization).
//
//   key row   k[b,t,h,:]: k' = (k * diag(signs[h,:])) * H_128 / sqrt(128)
//   value row v[b,t,h,:]: not rotated
//   s = fp16(max|row'| / 7), q = clamp(rint(row'/s), -8, 7), 64 packed bytes
//
// Each (b, t, h) row is 128 fp16 = 256 bytes and its own quantization group.
// The kernel is HBM-bound (2 bytes read, 0.5 written per element), so what
// matters is how many bytes each SM keeps in flight: a single thread copies
// tiles of 128 rows (32 KB) with the tensor copy engine into a 3-stage ring,
// two tiles ahead of the 128 threads that consume them, one row per thread.
// The tiles use the 128-byte swizzle (two boxes of 64 columns), so that the
// 16-byte chunk c of row r sits at chunk c ^ (r mod 8) of its 128-byte line
// and the row-per-thread reads of a warp hit every bank evenly.
// When Hkv divides 128, every row a thread handles belongs to the same KV
// head, and its sign words are built once; otherwise the CTA builds every
// head's sign words into a table in shared memory once, and each thread
// reads its row's entry per tile.  (The block rotation I_{K/128} (x) H_128
// with 128-groups is the same computation on the rows of x viewed as
// [M K/128, 128], with K/128 "heads" of 128 signs.)
#pragma once

#include <cuda.h>

#include "rotate_quant.cuh"
#include "tc_ptx.cuh"

namespace quarot {

constexpr int kKvTileRows = 128;
constexpr int kKvStages = 3;
constexpr int kKvStageBytes = kKvTileRows * 256;          // two 64-column boxes of 16 KB
constexpr int kKvMaxHeads = 512;                         // sign-word table: 16 bytes per head
constexpr int kKvSgnOffset = kKvStages * kKvStageBytes + 64;
constexpr int kKvSmemBytes = kKvSgnOffset + kKvMaxHeads * 16 + 1024;
constexpr uint64_t kKvWaitLimitNs = 2000000000ull;

template <bool ROTATE>
__global__ void __launch_bounds__(kKvTileRows, 2)
kv_quant_tma_kernel(const __grid_constant__ CUtensorMap tmap,   // fp16 [rows, 128], box {64, 128}, 128B swizzle
                    int64_t rows, int hkv, const int8_t *__restrict__ signs,
                    uint8_t *__restrict__ q,                    // [rows, 64]
                    __half *__restrict__ scales,                // [rows]
                    float scale_mul, float sqrt_n,
                    uint64_t wait_limit_ns,                     // bound of every wait
                    int64_t withheld_tile)                      // tile whose copy is never issued (-1: none)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + kKvStages * kKvStageBytes;
    const int t = threadIdx.x;
    const int64_t tiles = (rows + kKvTileRows - 1) / kKvTileRows;
    const int64_t first = blockIdx.x;
    const int64_t step = gridDim.x;

    if (t == 0) {
        for (int s = 0; s < kKvStages; ++s)
            mbar_init(bar_full + 8 * s, 1);
        mbar_fence_init();
        tma_prefetch_desc(&tmap);
    }
    // heads that change from tile to tile (hkv does not divide 128): every
    // head's sign words, built once per CTA
    const bool head_per_tile = ROTATE && (kKvTileRows % hkv) != 0;
    uint4 *sgn_tab = reinterpret_cast<uint4 *>(smem + kKvSgnOffset);
    if (head_per_tile)
        for (int hh = t; hh < hkv; hh += kKvTileRows) {
            uint32_t w4[4];
            build_sign_words(signs + (int64_t)hh * 128, [&](int j) { return 2 * j; }, w4);
            sgn_tab[hh] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
    __syncthreads();

    int issued = 0;                       // thread 0: tiles whose copies were issued (in tile order)
    auto issue = [&](int64_t tile, int s) {
        ++issued;
        if (tile == withheld_tile)
            return;                       // only the timeout test withholds a copy
        const uint32_t dst = sbase + s * kKvStageBytes;
        mbar_arrive_expect_tx(bar_full + 8 * s, kKvStageBytes);
        tma_load_2d(dst, &tmap, 0, (int)(tile * kKvTileRows), bar_full + 8 * s);
        tma_load_2d(dst + kKvStageBytes / 2, &tmap, 64, (int)(tile * kKvTileRows), bar_full + 8 * s);
    };
    if (t == 0) {
        for (int s = 0; s < kKvStages - 1; ++s)
            if (first + s * step < tiles)
                issue(first + s * step, s);
    }

    // sign words of this thread's head (the same for every tile when hkv divides 128)
    uint32_t sgn[4] = {0u, 0u, 0u, 0u};
    if (ROTATE && !head_per_tile) {
        const int8_t *sh = signs + (int64_t)(t % hkv) * 128;
        build_sign_words(sh, [&](int j) { return 2 * j; }, sgn);
    }

    int it = 0;
    bool ok = true;
    for (int64_t tile = first; tile < tiles; tile += step, ++it) {
        const int s = it % kKvStages;
        // the next-but-one tile goes into the stage freed at the end of the
        // previous iteration
        if (t == 0 && tile + (kKvStages - 1) * step < tiles)
            issue(tile + (kKvStages - 1) * step, (it + kKvStages - 1) % kKvStages);
        const uint32_t parity = (uint32_t)(it / kKvStages) & 1;
        if (!mbar_try_wait(bar_full + 8 * s, parity)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(bar_full + 8 * s, parity)) {
                if (globaltimer_ns() - t0 > wait_limit_ns) {
                    record_timeout();
                    ok = false;
                    break;
                }
            }
        }
        if (!__syncthreads_and(ok))
            break;
        // row t of the tile: chunk c (8 fp16) of half h at chunk c ^ (t & 7)
        const uint8_t *base = smem + s * kKvStageBytes + t * 128;
        uint4 w[16];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < 8; ++c)
                w[8 * h + c] = *reinterpret_cast<const uint4 *>(base + h * (kKvStageBytes / 2) + ((c ^ (t & 7)) << 4));
        __syncthreads();                  // every read of stage s is done: it may be refilled
        if (head_per_tile) {
            const uint4 w4 = sgn_tab[(tile * kKvTileRows + t) % hkv];
            sgn[0] = w4.x;
            sgn[1] = w4.y;
            sgn[2] = w4.z;
            sgn[3] = w4.w;
        }
        float v[128];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t ww[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t bits = ROTATE ? apply_sign_pair(ww[k], sgn, 4 * i + k) : ww[k];
                const float2 f = half2_bits_to_float2(bits);
                v[8 * i + 2 * k] = f.x;
                v[8 * i + 2 * k + 1] = f.y;
            }
        }
        if (ROTATE)
            fwht_bits<0, 7>(v);
        const float amax = absmax128(v);
        const int64_t row = tile * kKvTileRows + t;
        const bool valid = row < rows;
        __half s16;
        const float r = group_scale(amax, scale_mul, sqrt_n, s16);
        if (valid && QUAROT_IN_RANGE(scales + row, 2, scales, rows * 2))
            scales[row] = s16;
        uint8_t *qdst = q + (valid ? row : 0) * 64;
        quant_pack_store<128>(v, r, qdst, valid && QUAROT_IN_RANGE(qdst, 64, q, rows * 64), scale_needs_clamp(s16));
    }
    // copies issued beyond the consumed tiles (abort only) land before exit:
    // iterations it .. issued - 1 had their copies issued but were not waited for
    if (t == 0)
        for (int j = it; j < issued; ++j)
            mbar_wait_drain(bar_full + 8 * (j % kKvStages), (uint32_t)(j / kKvStages) & 1, wait_limit_ns);
}

}  // namespace quarot
