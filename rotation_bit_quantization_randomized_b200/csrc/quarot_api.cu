// quarot_api.cu -- the C ABI of libquarot (declared in include/quarot.h):
// argument validation, launch configuration and error reporting around the
// kernels of the csrc/*.cuh headers.
#include "quarot.h"

#include "common.cuh"
#include "int4_gemm.cuh"
#include "int4_gemm_pair.cuh"
#include "int8_gemm_pair.cuh"
#include "kron_quant.cuh"
#include "kv_attend.cuh"
#include "kv_decode_tc.cuh"
#include "kv_scores_tc.cuh"
#include "kv_quant.cuh"
#include "mma_peak.cuh"
#include "rotate_quant.cuh"
#include "rotate_tc.cuh"

#include <cuda.h>

#include <cmath>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

using namespace quarot;

// The staged KV-write launcher (defined below, outside the internal namespace).
template <bool ROTATE>
quarot_status_t launch_kv_tma(const void *x, int64_t rows, int hkv, const int8_t *signs, uint8_t *q, void *scales,
                              float scale_mul, float sqrt_n, cudaStream_t st, int dev, int sms,
                              uint64_t wait_limit_ns = kKvWaitLimitNs, int64_t withheld_tile = -1);

namespace {

thread_local std::string g_last_error;

quarot_status_t fail(quarot_status_t s, const std::string &msg)
{
    g_last_error = msg;
    return s;
}

quarot_status_t cuda_fail(cudaError_t e, const char *what)
{
    return fail(QUAROT_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Per-device facts and one-time kernel attributes.
struct DeviceInfo {
    bool init = false;
    bool ok = false;
    int sm_count = 0;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

quarot_status_t current_device(int &dev, DeviceInfo *&info)
{
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return fail(QUAROT_ERR_NO_DEVICE, "device ordinal out of range");
    std::lock_guard<std::mutex> lk(g_mutex);
    DeviceInfo &d = g_devices[dev];
    if (!d.init) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        d.ok = (major == 10 && minor == 0);
        d.init = true;
    }
    info = &d;
    if (!d.ok)
        return fail(QUAROT_ERR_NO_DEVICE, "libquarot needs an sm_100 (B200) device");
    return QUAROT_OK;
}

// Resident CTAs per SM of `kernel`, computed once per (kernel, device); also
// raises the dynamic shared-memory limit when the kernel needs it.
template <typename K>
quarot_status_t kernel_occupancy(K kernel, int dev, int threads, size_t dyn_smem, int &per_sm)
{
    struct Entry {
        const void *fn;
        int dev;
        int threads;
        int per_sm;
    };
    static Entry cache[256];
    static int n = 0;
    std::lock_guard<std::mutex> lk(g_mutex);
    for (int i = 0; i < n; ++i)
        if (cache[i].fn == (const void *)kernel && cache[i].dev == dev && cache[i].threads == threads) {
            per_sm = cache[i].per_sm;
            return QUAROT_OK;
        }
    cudaError_t e;
    if (dyn_smem > 48 * 1024) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_smem);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaFuncSetAttribute");
    }
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, dyn_smem);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (per_sm < 1)
        return fail(QUAROT_ERR_CUDA, "kernel does not fit on an SM");
    if (n < 256)
        cache[n++] = Entry{(const void *)kernel, dev, threads, per_sm};
    return QUAROT_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

int ilog2(int64_t v)
{
    int l = 0;
    while ((int64_t(1) << l) < v)
        ++l;
    return l;
}

quarot_status_t after_launch(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e, what);
    return QUAROT_OK;
}

// ----------------------------------------------------------------- rotate + quantize
quarot_status_t check_rotate_args(const void *x, int64_t M, int64_t K, const int8_t *signs, int had_block,
                                  int group, const void *q, const void *scales)
{
    if (M < 0 || K <= 0)
        return fail(QUAROT_ERR_INVALID_ARG, "M must be >= 0 and K > 0");
    if (had_block != 0 && had_block != 128)
        return fail(QUAROT_ERR_INVALID_ARG, "had_block must be 0 or 128");
    if (group != 0 && group != 128)
        return fail(QUAROT_ERR_INVALID_ARG, "group must be 0 or 128");
    if (had_block == 0 && (!is_pow2(K) || K < 128 || K > 8192))
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "full Hadamard needs K a power of two in [128, 8192]");
    if (had_block == 128 && (K % 128 != 0 || K > 65536))
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "block Hadamard needs K % 128 == 0 and K <= 65536");
    if (M == 0)
        return QUAROT_OK;
    if (!x || !signs || !q || !scales)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x) || !aligned16(q) || !aligned16(scales))
        return fail(QUAROT_ERR_MISALIGNED, "x, q_packed and scales must be 16-byte aligned");
    return QUAROT_OK;
}

// Smallest log2 K of the full transform that takes the tensor-core kernel
// (below it the register-only kernel).
constexpr int kTcMinLogK = 8;

// qmax of a code width: the largest code magnitude of the symmetric RTN.
constexpr double qmax_of(int bits) { return (double)code_qmax(bits); }

template <int LOGN, int GROUP, int BITS, bool ASYM = false>
quarot_status_t launch_fwht(const void *x, int64_t M, const int8_t *signs, uint8_t *q, void *scales,
                            cudaStream_t st, int dev, int sms, AsymOut asym = AsymOut{nullptr, nullptr, 1.0f})
{
    auto kern = fwht_quant_kernel<LOGN, GROUP, BITS, ASYM>;
    constexpr int smem = FwhtSmem<LOGN>::kBytes;
    int per_sm = 0;
    quarot_status_t s = kernel_occupancy(kern, dev, kFwhtThreads, smem, per_sm);
    if (s != QUAROT_OK)
        return s;
    constexpr int R = kFwhtThreads / ((1 << LOGN) / 128);
    const int64_t ctas = (M + R - 1) / R;
    const int grid = (int)std::min<int64_t>(ctas, (int64_t)sms * per_sm);
    const double n = double(1 << LOGN);
    const double mul = ASYM ? 1.0 / std::sqrt(n) : 1.0 / (qmax_of(BITS) * std::sqrt(n));
    kern<<<grid, kFwhtThreads, smem, st>>>(reinterpret_cast<const uint32_t *>(x), M, signs, q, scales, (float)mul,
                                           (float)std::sqrt(n), asym);
    return after_launch("fwht_quant_kernel launch");
}

template <int GROUP, int BITS>
quarot_status_t dispatch_fwht(int logn, const void *x, int64_t M, const int8_t *signs, uint8_t *q,
                              void *scales, cudaStream_t st, int dev, int sms)
{
    switch (logn) {
    case 8: return launch_fwht<8, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 9: return launch_fwht<9, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 10: return launch_fwht<10, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 11: return launch_fwht<11, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 12: return launch_fwht<12, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 13: return launch_fwht<13, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    default: return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "unsupported transform size");
    }
}

// The asymmetric quantizer (full transform, K a power of two in [256, 8192]).
quarot_status_t dispatch_fwht_asym(int logn, const void *x, int64_t M, const int8_t *signs, uint8_t *q,
                                   float *scales, AsymOut asym, cudaStream_t st, int dev, int sms)
{
    switch (logn) {
    case 8: return launch_fwht<8, 0, 4, true>(x, M, signs, q, scales, st, dev, sms, asym);
    case 9: return launch_fwht<9, 0, 4, true>(x, M, signs, q, scales, st, dev, sms, asym);
    case 10: return launch_fwht<10, 0, 4, true>(x, M, signs, q, scales, st, dev, sms, asym);
    case 11: return launch_fwht<11, 0, 4, true>(x, M, signs, q, scales, st, dev, sms, asym);
    case 12: return launch_fwht<12, 0, 4, true>(x, M, signs, q, scales, st, dev, sms, asym);
    case 13: return launch_fwht<13, 0, 4, true>(x, M, signs, q, scales, st, dev, sms, asym);
    default: return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "unsupported transform size");
    }
}

quarot_status_t encode_tiled_fn_checked(void *&fn);

// The full transform with its H_m factor on the tensor cores (K = 128 m).
template <int LOGM, int GROUP, int BITS>
quarot_status_t launch_had_tc(const void *x, int64_t M, const int8_t *signs, uint8_t *q, void *scales,
                              cudaStream_t st, int dev, int sms)
{
    constexpr int m = 1 << LOGM;
    constexpr int G = 256 / m;
    if (M > ((int64_t(1) << 31) - 512) / m)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "M * K / 128 must stay below 2^31");
    auto kern = had_tc_quant_kernel<LOGM, GROUP, BITS>;
    int per_sm = 0;
    quarot_status_t s = kernel_occupancy(kern, dev, kRtThreads, RtSmem::kBytes, per_sm);
    if (s != QUAROT_OK)
        return s;
    void *fnp = nullptr;
    s = encode_tiled_fn_checked(fnp);
    if (s != QUAROT_OK)
        return s;
    auto fn = reinterpret_cast<CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                            const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                            const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                            CUtensorMapL2promotion, CUtensorMapFloatOOBfill)>(fnp);
    // x viewed as fp16 [M * m, 128]: row (token, a), column b
    CUtensorMap map;
    const cuuint64_t dims[2] = {128, (cuuint64_t)M * m};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QUAROT_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    const int64_t groups = (M + G - 1) / G;
    const int grid = (int)std::min<int64_t>(groups, (int64_t)sms * per_sm);
    const double n = double(128 * m);
    kern<<<grid, kRtThreads, RtSmem::kBytes, st>>>(map, M, signs, q, scales,
                                                   (float)(1.0 / (code_qmax(BITS) * std::sqrt(n))),
                                                   (float)std::sqrt(n));
    return after_launch("had_tc_quant_kernel launch");
}

template <int GROUP, int BITS>
quarot_status_t dispatch_had_tc(int logn, const void *x, int64_t M, const int8_t *signs, uint8_t *q, void *scales,
                                cudaStream_t st, int dev, int sms)
{
    switch (logn) {
    case 8: return launch_had_tc<1, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 9: return launch_had_tc<2, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 10: return launch_had_tc<3, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 11: return launch_had_tc<4, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 12: return launch_had_tc<5, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    case 13: return launch_had_tc<6, GROUP, BITS>(x, M, signs, q, scales, st, dev, sms);
    default: return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "unsupported transform size");
    }
}

template <bool ROTATE, int GROUP, int BITS = 4>
quarot_status_t launch_block(const void *x, int64_t M, int64_t K, const int8_t *signs, uint8_t *q,
                             void *scales, float scale_mul, float sqrt_n, cudaStream_t st, int dev, int sms)
{
    const int nb = (int)(K / 128);
    const bool multi = nb > kBlockThreads;
    auto kern = multi ? block128_quant_kernel<ROTATE, GROUP, true, BITS>
                      : block128_quant_kernel<ROTATE, GROUP, false, BITS>;
    const int rows_per_cta = multi ? 1 : kBlockThreads / nb;
    const int threads = multi ? kBlockThreads : ((rows_per_cta * nb + 31) / 32) * 32;
    int per_sm = 0;
    quarot_status_t s = kernel_occupancy(kern, dev, threads, 0, per_sm);
    if (s != QUAROT_OK)
        return s;
    const int64_t ctas = (M + rows_per_cta - 1) / rows_per_cta;
    const int grid = (int)std::min<int64_t>(ctas, (int64_t)sms * per_sm);
    kern<<<grid, threads, 0, st>>>(reinterpret_cast<const uint4 *>(x), M, (int)K, rows_per_cta, signs, q,
                                   scales, scale_mul, sqrt_n);
    return after_launch("block128_quant_kernel launch");
}

// bits 6 and 8 imply group == 0 (checked by the callers).
quarot_status_t rotate_quant_launch(const void *x, int64_t M, int64_t K, const int8_t *signs, int had_block,
                                    int group, uint8_t *q, void *scales, cudaStream_t st, int bits = 4)
{
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    const int sms = info->sm_count;
    if (had_block == 0 && K >= 256) {
        const int logn = ilog2(K);
        if (logn >= kTcMinLogK) {
            // first factor H_{K/128} on the tensor cores, H_128 in registers
            if (bits == 8)
                return dispatch_had_tc<0, 8>(logn, x, M, signs, q, scales, st, dev, sms);
            if (bits == 6)
                return dispatch_had_tc<0, 6>(logn, x, M, signs, q, scales, st, dev, sms);
            return group == 0 ? dispatch_had_tc<0, 4>(logn, x, M, signs, q, scales, st, dev, sms)
                              : dispatch_had_tc<128, 4>(logn, x, M, signs, q, scales, st, dev, sms);
        }
        if (bits == 8)
            return dispatch_fwht<0, 8>(logn, x, M, signs, q, scales, st, dev, sms);
        if (bits == 6)
            return dispatch_fwht<0, 6>(logn, x, M, signs, q, scales, st, dev, sms);
        return group == 0 ? dispatch_fwht<0, 4>(logn, x, M, signs, q, scales, st, dev, sms)
                          : dispatch_fwht<128, 4>(logn, x, M, signs, q, scales, st, dev, sms);
    }
    const float mul = (float)(1.0 / (qmax_of(bits) * std::sqrt(128.0)));
    const float sq = (float)std::sqrt(128.0);
    const int64_t nb = K / 128;
    if (bits == 4 && group == 128 && nb <= kKvMaxHeads && M * nb < (int64_t(1) << 31) - kKvTileRows)
        // I_{K/128} (x) H_128 with 128-groups: the KV write's computation on x
        // viewed as [M K/128, 128] rows, head = block index
        return launch_kv_tma<true>(x, M * nb, (int)nb, signs, q, scales, mul, sq, st, dev, sms);
    if (bits == 8)
        return launch_block<true, 0, 8>(x, M, K, signs, q, scales, mul, sq, st, dev, sms);
    if (bits == 6)
        return launch_block<true, 0, 6>(x, M, K, signs, q, scales, mul, sq, st, dev, sms);
    return group == 0 ? launch_block<true, 0>(x, M, K, signs, q, scales, mul, sq, st, dev, sms)
                      : launch_block<true, 128>(x, M, K, signs, q, scales, mul, sq, st, dev, sms);
}

// ----------------------------------------------------------------- GEMM
quarot_status_t check_gemm_args(const void *qa, int64_t M, const void *qw, int64_t N, int64_t K,
                                const void *out, const void *sa, const void *sw, bool need_scales)
{
    if (M < 0 || N <= 0 || K <= 0)
        return fail(QUAROT_ERR_INVALID_ARG, "M must be >= 0, N and K > 0");
    if (N % 8 != 0)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "N must be a multiple of 8");
    if (K % 128 != 0 || K > 65536)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "K must be a multiple of 128 and at most 65536");
    if (M > (int64_t(1) << 31) - 128 || N > (int64_t(1) << 31) - 256)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "M or N too large");
    if (M == 0)
        return QUAROT_OK;
    if (!qa || !qw || !out || (need_scales && (!sa || !sw)))
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(qa) || !aligned16(qw) || !aligned16(out) || (need_scales && (!aligned16(sa) || !aligned16(sw))))
        return fail(QUAROT_ERR_MISALIGNED, "operands, scales and output must be 16-byte aligned");
    return QUAROT_OK;
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime so that
// the library does not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

quarot_status_t encode_tiled_fn(EncodeTiledFn &fn)
{
    static EncodeTiledFn cached = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if (!cached) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
        if (q != cudaDriverEntryPointSuccess || !p)
            return fail(QUAROT_ERR_CUDA, "the driver does not provide cuTensorMapEncodeTiled");
        cached = reinterpret_cast<EncodeTiledFn>(p);
    }
    fn = cached;
    return QUAROT_OK;
}

quarot_status_t encode_tiled_fn_checked(void *&fn)
{
    EncodeTiledFn f;
    quarot_status_t s = encode_tiled_fn(f);
    fn = reinterpret_cast<void *>(f);
    return s;
}

// Tensor map of a packed INT4 matrix [rows, K/2] bytes read in boxes of
// 64 bytes (128 codes) x box_rows rows; rows past the end read as zeros.
// With the 64-byte swizzle the 16-byte chunk c of box row r lands at chunk
// c ^ ((r / 2) % 4) of that row in shared memory.
quarot_status_t packed_map(CUtensorMap &map, const uint8_t *base, int64_t rows, int64_t K, int box_rows,
                           CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE)
{
    EncodeTiledFn fn;
    quarot_status_t s = encode_tiled_fn(fn);
    if (s != QUAROT_OK)
        return s;
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    const cuuint32_t box[2] = {(cuuint32_t)(kGemmBK / 2), (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QUAROT_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    return QUAROT_OK;
}


// N tile of the pair GEMM: two accumulator buffers of 224 columns leave
// tensor memory for two A stages.
constexpr int kPairBN = 224;

// The per-token / per-channel GEMM on CTA pairs (clusters of two); UNS for
// unsigned (asymmetric) codes.
template <int EPI, bool UNS = false>
quarot_status_t launch_gemm_pair(GemmArgs a, cudaStream_t st, bool pdl)
{
    // grouped scales: N tile 128 per pair (three accumulators in tensor memory)
    constexpr int BN = EPI == kEpiGroupF16 ? 128 : kPairBN;
    using S = PairShape<BN, EPI>;
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    auto kern = int4_gemm_pair_kernel<BN, EPI, UNS>;
    int per_sm = 0;
    s = kernel_occupancy(kern, dev, S::kThreads, S::kSmemBytes, per_sm);
    if (s != QUAROT_OK)
        return s;
    a.tiles_m = (int)((a.M + kPairBM - 1) / kPairBM);
    a.tiles_n = (int)((a.N + BN - 1) / BN);
    a.kblocks = (int)(a.K / kGemmBK);
    const int64_t tiles = (int64_t)a.tiles_m * a.tiles_n;
    if (tiles > 0x7fffffff)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "too many output tiles");
    CUtensorMap map_a, map_b;
    s = packed_map(map_a, a.qa, a.M, a.K, S::kRowsA, CU_TENSOR_MAP_SWIZZLE_64B);
    if (s != QUAROT_OK)
        return s;
    s = packed_map(map_b, a.qw, a.N, a.K, S::kRowsB);
    if (s != QUAROT_OK)
        return s;
    const int clusters = (int)std::min<int64_t>(tiles, (int64_t)(info->sm_count / 2));

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(S::kThreads);
    cfg.dynamicSmemBytes = S::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    int nattr = 1;
    if (pdl) {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        nattr = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, map_a, map_b);
    if (e != cudaSuccess)
        return cuda_fail(e, "int4_gemm_pair_kernel launch");
    return after_launch("int4_gemm_pair_kernel launch");
}

// Tensor map of an INT8 code matrix [rows, K] read in boxes of 128 bytes x
// 128 rows with the 128-byte swizzle -- the K-major layout the MMA reads;
// rows past the end read as zeros.
quarot_status_t i8_map(CUtensorMap &map, const int8_t *base, int64_t rows, int64_t K)
{
    EncodeTiledFn fn;
    quarot_status_t s = encode_tiled_fn(fn);
    if (s != QUAROT_OK)
        return s;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {(cuuint32_t)kGemmBK, (cuuint32_t)I8PairShape::kRows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QUAROT_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    return QUAROT_OK;
}

// The INT8 GEMM on CTA pairs (clusters of two); a.qa / a.qw hold int8 codes.
template <int EPI>
quarot_status_t launch_gemm_i8(GemmArgs a, cudaStream_t st, bool pdl)
{
    using S = I8PairShape;
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    auto kern = int8_gemm_pair_kernel<EPI>;
    int per_sm = 0;
    s = kernel_occupancy(kern, dev, S::kThreads, S::kSmemBytes, per_sm);
    if (s != QUAROT_OK)
        return s;
    a.tiles_m = (int)((a.M + kI8PairBM - 1) / kI8PairBM);
    a.tiles_n = (int)((a.N + kI8PairBN - 1) / kI8PairBN);
    a.kblocks = (int)(a.K / kGemmBK);
    const int64_t tiles = (int64_t)a.tiles_m * a.tiles_n;
    if (tiles > 0x7fffffff)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "too many output tiles");
    CUtensorMap map_a, map_b;
    s = i8_map(map_a, reinterpret_cast<const int8_t *>(a.qa), a.M, a.K);
    if (s != QUAROT_OK)
        return s;
    s = i8_map(map_b, reinterpret_cast<const int8_t *>(a.qw), a.N, a.K);
    if (s != QUAROT_OK)
        return s;
    const int clusters = (int)std::min<int64_t>(tiles, (int64_t)(info->sm_count / 2));

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(S::kThreads);
    cfg.dynamicSmemBytes = S::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    int nattr = 1;
    if (pdl) {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        nattr = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, map_a, map_b);
    if (e != cudaSuccess)
        return cuda_fail(e, "int8_gemm_pair_kernel launch");
    return after_launch("int8_gemm_pair_kernel launch");
}

quarot_status_t linear8_launch(const int8_t *qa, const float *sa, int64_t M, const int8_t *qw, const float *sw,
                               int64_t N, int64_t K, void *out, cudaStream_t st, bool pdl)
{
    GemmArgs a = {};
    a.qa = reinterpret_cast<const uint8_t *>(qa);
    a.sa = sa;
    a.qw = reinterpret_cast<const uint8_t *>(qw);
    a.sw = sw;
    a.out = out;
    a.M = M;
    a.N = N;
    a.K = K;
    return launch_gemm_i8<kEpiScaledF16>(a, st, pdl);
}

quarot_status_t linear_launch(const uint8_t *qa, const void *sa, int64_t M, const uint8_t *qw, const void *sw,
                              int64_t N, int64_t K, int group, void *out, cudaStream_t st, bool pdl)
{
    GemmArgs a = {};
    a.qa = qa;
    a.sa = sa;
    a.qw = qw;
    a.sw = sw;
    a.out = out;
    a.M = M;
    a.N = N;
    a.K = K;
    return group == 0 ? launch_gemm_pair<kEpiScaledF16>(a, st, pdl) : launch_gemm_pair<kEpiGroupF16>(a, st, pdl);
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Scratch of quarot_rotate_quant_linear_noalloc: a fixed device array that
// every GPU loading the library holds until exit.  In host code the name is
// only a host-side handle, never a device address: the kernels get the
// address cudaGetSymbolAddress returns, looked up once per device.
constexpr size_t kNoAllocScratchBytes = size_t(QUAROT_NOALLOC_SCRATCH_BYTES);
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
void *g_noalloc_addr[kMaxDevices];

quarot_status_t noalloc_scratch_address(int dev, void *&addr)
{
    std::lock_guard<std::mutex> lk(g_mutex);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress of the built-in scratch");
        g_noalloc_addr[dev] = p;
    }
    addr = g_noalloc_addr[dev];
    return QUAROT_OK;
}

// ----------------------------------------------------------------- full Kronecker rotation
// The Hadamard factor of order 344 by Paley's first construction: q = 343 =
// 7^3 = 3 mod 4, field GF(7)[x] / (x^3 + 2) (x^3 + 2 has no root in GF(7),
// whose cubes are 0, 1 and 6, so it is irreducible), element
// c0 + c1 x + c2 x^2 numbered c0 + 7 c1 + 49 c2.  With chi the quadratic
// character (found here by squaring every nonzero element):
//   H[0][j] = 1, H[i][0] = -1 (i > 0), H[i][i] = 1,
//   H[i][j] = chi(e_{i-1} - e_{j-1}) otherwise,
// so H H^T = 344 I.
void paley344(int8_t *H)
{
    constexpr int p = 7, q = 343, n = 344;
    auto digits = [](int a, int (&c)[3]) {
        c[0] = a % p;
        c[1] = (a / p) % p;
        c[2] = a / (p * p);
    };
    auto mul = [&](int a, int b) {
        int A[3], B[3];
        digits(a, A);
        digits(b, B);
        int P[5] = {0, 0, 0, 0, 0};
        for (int i = 0; i < 3; ++i)
            for (int j = 0; j < 3; ++j)
                P[i + j] += A[i] * B[j];
        P[1] += 5 * P[4];                  // x^4 = x * x^3 = 5 x
        P[0] += 5 * P[3];                  // x^3 = -2 = 5
        return P[0] % p + p * (P[1] % p) + p * p * (P[2] % p);
    };
    std::vector<int8_t> square(q, 0);
    for (int y = 1; y < q; ++y)
        square[mul(y, y)] = 1;
    auto chi_diff = [&](int a, int b) {
        int A[3], B[3];
        digits(a, A);
        digits(b, B);
        const int d = (A[0] - B[0] + p) % p + p * ((A[1] - B[1] + p) % p) + p * p * ((A[2] - B[2] + p) % p);
        return d == 0 ? 0 : (square[d] ? 1 : -1);
    };
    for (int j = 0; j < n; ++j)
        H[j] = 1;
    for (int i = 1; i < n; ++i) {
        H[(size_t)i * n] = -1;
        for (int j = 1; j < n; ++j)
            H[(size_t)i * n + j] = (int8_t)(i == j ? 1 : chi_diff(i - 1, j - 1));
    }
}

// H^T as fp16, zero-padded to 384 x 384 (the MMA operand): an array compiled
// into the library (nothing is allocated), filled once per device by a
// synchronous copy with that device current; the kernels get the address
// cudaGetSymbolAddress returns for that device.
static __device__ __align__(256) uint16_t g_kron_ht[kKronAPad * kKronAPad];
std::mutex g_kron_mutex;
void *g_kron_factor[kMaxDevices] = {};

quarot_status_t kron_factor_device(int dev, const void *&ptr)
{
    std::lock_guard<std::mutex> lk(g_kron_mutex);
    if (!g_kron_factor[dev]) {
        std::vector<int8_t> H((size_t)kKronM * kKronM);
        paley344(H.data());
        std::vector<uint16_t> Ht((size_t)kKronAPad * kKronAPad, 0);
        for (int ap = 0; ap < kKronM; ++ap)
            for (int a = 0; a < kKronM; ++a)
                Ht[(size_t)ap * kKronAPad + a] = H[(size_t)a * kKronM + ap] > 0 ? 0x3C00 : 0xBC00;
        cudaError_t e = cudaMemcpyToSymbol(g_kron_ht, Ht.data(), Ht.size() * 2);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaMemcpyToSymbol (Hadamard factor)");
        void *d = nullptr;
        e = cudaGetSymbolAddress(&d, g_kron_ht);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress (Hadamard factor)");
        g_kron_factor[dev] = d;
    }
    ptr = g_kron_factor[dev];
    return QUAROT_OK;
}

quarot_status_t kron_launch(const void *x, int64_t M, const int8_t *signs, int group, uint8_t *q, void *scales,
                            cudaStream_t st)
{
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    const void *ht;
    s = kron_factor_device(dev, ht);
    if (s != QUAROT_OK)
        return s;
    EncodeTiledFn fn;
    s = encode_tiled_fn(fn);
    if (s != QUAROT_OK)
        return s;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)kKronAPad, (cuuint64_t)kKronAPad};
    const cuuint64_t strides[1] = {(cuuint64_t)kKronAPad * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(ht), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QUAROT_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    const size_t smem = KronSmem::kBytes;
    const float scale_mul = (float)(1.0 / (7.0 * std::sqrt((double)kKronK)));
    const float sqrt_n = (float)std::sqrt((double)kKronK);
    const int64_t tiles = (M + kKronRows - 1) / kKronRows;
    int per_sm = 0;
    if (group == 0) {
        s = kernel_occupancy(kron_quant_kernel<0>, dev, kKronThreads, smem, per_sm);
        if (s != QUAROT_OK)
            return s;
        const int grid = (int)std::min<int64_t>(tiles, (int64_t)info->sm_count * per_sm);
        kron_quant_kernel<0><<<grid, kKronThreads, smem, st>>>(map, static_cast<const __half *>(x), M, signs, q,
                                                               scales, scale_mul, sqrt_n);
    } else {
        s = kernel_occupancy(kron_quant_kernel<128>, dev, kKronThreads, smem, per_sm);
        if (s != QUAROT_OK)
            return s;
        const int grid = (int)std::min<int64_t>(tiles, (int64_t)info->sm_count * per_sm);
        kron_quant_kernel<128><<<grid, kKronThreads, smem, st>>>(map, static_cast<const __half *>(x), M, signs, q,
                                                                 scales, scale_mul, sqrt_n);
    }
    return after_launch("kron_quant_kernel launch");
}

// Clusters of `split` attention CTAs (G query heads per KV head) that can be
// resident at once on the device, queried once per (device, G, split).
quarot_status_t attend_resident_clusters(int G, int split, int dev, int &fit)
{
    static int cache[kMaxDevices][5][4];
    static bool known[kMaxDevices][5][4];
    const int gi = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : 4;
    const int si = split == 1 ? 0 : split == 2 ? 1 : split == 4 ? 2 : 3;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (known[dev][gi][si]) {
            fit = cache[dev][gi][si];
            return QUAROT_OK;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)split, 1, 1);
    cfg.blockDim = dim3(kAttThreads);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    switch (G) {
    case 1: e = cudaOccupancyMaxActiveClusters(&fit, kv_attend_kernel<1>, &cfg); break;
    case 2: e = cudaOccupancyMaxActiveClusters(&fit, kv_attend_kernel<2>, &cfg); break;
    case 4: e = cudaOccupancyMaxActiveClusters(&fit, kv_attend_kernel<4>, &cfg); break;
    case 8: e = cudaOccupancyMaxActiveClusters(&fit, kv_attend_kernel<8>, &cfg); break;
    default: e = cudaOccupancyMaxActiveClusters(&fit, kv_attend_kernel<16>, &cfg); break;
    }
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaOccupancyMaxActiveClusters");
    std::lock_guard<std::mutex> lk(g_mutex);
    cache[dev][gi][si] = fit;
    known[dev][gi][si] = true;
    return QUAROT_OK;
}

// CTAs of a tensor-core decode kernel (the fused step or the scores) that can
// be resident on one SM, computed from the kernel's own resources: shared
// memory with the per-CTA reservation, registers in 256-register warp
// allocations, threads, CTA slots.  The runtime's occupancy queries report
// one CTA per SM for these kernels at any shared-memory size, while three are
// resident when they run (counted on B200 with %smid).  Also raises the
// kernel's dynamic shared-memory limit and asks for all of the unified L1 /
// shared storage as shared memory.
template <typename K>
quarot_status_t tc_decode_per_sm(K kernel, size_t smem, int dev, int &per_sm)
{
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute");
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute");
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFuncGetAttributes");
    int smem_sm = 0, smem_res = 0, regs_sm = 0, thr_sm = 0, blk_sm = 0;
    if (cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem_res, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&blk_sm, cudaDevAttrMaxBlocksPerMultiprocessor, dev) != cudaSuccess)
        return fail(QUAROT_ERR_CUDA, "cudaDeviceGetAttribute failed");
    const int warp_regs = ((fa.numRegs * 32 + 255) / 256) * 256;
    const int cta_regs = warp_regs * (kDecThreads / 32);
    const int cta_smem = (int)smem + (int)fa.sharedSizeBytes + smem_res;
    per_sm = std::min(std::min(smem_sm / cta_smem, regs_sm / std::max(cta_regs, 1)),
                      std::min(thr_sm / kDecThreads, blk_sm));
    if (per_sm < 1)
        return fail(QUAROT_ERR_CUDA, "a decode kernel does not fit on an SM");
    return QUAROT_OK;
}

// Clusters of `split` fused decode CTAs (G query heads per KV head) that can
// be resident at once (tc_decode_per_sm, computed once per (device, G)).
template <int G>
quarot_status_t decode_resident_clusters(int split, int dev, int &fit)
{
    static int cache[kMaxDevices];
    static bool known[kMaxDevices];
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (known[dev])
            per_sm = cache[dev];
    }
    if (per_sm == 0) {
        quarot_status_t s = tc_decode_per_sm(kv_decode_tc_kernel<G>, DecShape<G>::kBytes, dev, per_sm);
        if (s != QUAROT_OK)
            return s;
        std::lock_guard<std::mutex> lk(g_mutex);
        cache[dev] = per_sm;
        known[dev] = true;
    }
    int sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    fit = sms * per_sm / split;
    return QUAROT_OK;
}

// The scores on the tensor cores: CTAs of `tiles_per_cta` consecutive
// 128-token tiles of one (batch, KV head).  A CTA costs about its tiles plus
// half a tile of set-up (query rotation, tensor-memory allocation); the
// launch about ceil(CTAs / resident CTAs) such costs.  The tile count with the
// smallest estimate.
template <int G>
quarot_status_t launch_scores_tc(const __half *q, const int8_t *signs, const uint8_t *kq, const __half *ks,
                                 int64_t B, int64_t T, int Hkv, float *scores, cudaStream_t st, int dev)
{
    static int cache[kMaxDevices];
    static bool known[kMaxDevices];
    int per_sm = 0;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        if (known[dev])
            per_sm = cache[dev];
    }
    if (per_sm == 0) {
        quarot_status_t s = tc_decode_per_sm(kv_scores_tc_kernel<G>, ScShape<G>::kBytes, dev, per_sm);
        if (s != QUAROT_OK)
            return s;
        std::lock_guard<std::mutex> lk(g_mutex);
        cache[dev] = per_sm;
        known[dev] = true;
    }
    int sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute");
    const int64_t slots = (int64_t)sms * per_sm;
    const int64_t tiles = (T + kDecTile - 1) / kDecTile;
    int64_t best_tpc = 1;
    double best = -1.0;
    for (int64_t tpc = 1;; tpc *= 2) {
        const int64_t chunks = (tiles + tpc - 1) / tpc;
        const int64_t ctas = B * Hkv * chunks;
        const double est = (double)((ctas + slots - 1) / slots) * ((double)std::min(tpc, tiles) + 0.5);
        if (chunks <= 0x7fffffff && (best < 0.0 || est < best)) {
            best = est;
            best_tpc = tpc;
        }
        if (tpc >= tiles)
            break;
    }
    const int64_t chunks = (tiles + best_tpc - 1) / best_tpc;
    if (chunks > 0x7fffffff)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "T too large");
    dim3 grid((unsigned)chunks, (unsigned)Hkv, (unsigned)B);
    kv_scores_tc_kernel<G><<<grid, kDecThreads, ScShape<G>::kBytes, st>>>(q, signs, kq, ks, T, Hkv, (int)best_tpc,
                                                                          scores);
    return after_launch("kv_scores_tc_kernel launch");
}

template <int G>
quarot_status_t launch_decode_tc(const __half *q, const int8_t *signs, const uint8_t *kq, const __half *ks,
                                 const uint8_t *vq, const __half *vs, int64_t B, int64_t T, int Hkv, float *out,
                                 cudaStream_t st, int dev)
{
    // tokens split over a cluster of S CTAs, at least 128 tokens each.  A
    // CTA's time is about its tiles plus a fixed part (query rotation, the
    // cluster combine) that grows with S: 0.65 (1 + log2 S) tiles, as timed on
    // B200 at T 2048 for B 1 .. 64; the launch takes about ceil(clusters /
    // resident clusters) such CTA times.  The S with the smallest estimate.
    const int smax = T >= 1024 ? 8 : T >= 512 ? 4 : T >= 256 ? 2 : 1;
    int split = smax;
    double best = 0.0;
    for (int sp = 1, lg = 0; sp <= smax; sp *= 2, ++lg) {
        int fit = 0;
        quarot_status_t s = decode_resident_clusters<G>(sp, dev, fit);
        if (s != QUAROT_OK)
            return s;
        if (fit <= 0)
            continue;
        const int64_t clusters = B * Hkv;
        const int64_t waves = (clusters + fit - 1) / fit;
        const int64_t tiles = ((T + sp - 1) / sp + kDecTile - 1) / kDecTile;
        const double est = (double)waves * ((double)tiles + 0.65 * (1 + lg));
        if (sp == 1 || est < best) {
            best = est;
            split = sp;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)split, (unsigned)Hkv, (unsigned)B);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = DecShape<G>::kBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kv_decode_tc_kernel<G>, q, signs, kq, ks, vq, vs, T, Hkv, out);
    if (e != cudaSuccess)
        return cuda_fail(e, "kv_decode_tc_kernel launch");
    return after_launch("kv_decode_tc_kernel launch");
}

}  // namespace

// Tensor map of an fp16 [rows, 128] matrix (KV rows of one head) read in
// boxes of 64 columns x 128 rows with the 128-byte swizzle.
quarot_status_t kv_map(CUtensorMap &map, const void *base, int64_t rows)
{
    EncodeTiledFn fn;
    quarot_status_t s = encode_tiled_fn(fn);
    if (s != QUAROT_OK)
        return s;
    const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {64, (cuuint32_t)kKvTileRows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(QUAROT_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
    return QUAROT_OK;
}

// The staged KV-write kernel over `rows` rows of 128 elements, row r of head r mod hkv.
template <bool ROTATE>
quarot_status_t launch_kv_tma(const void *x, int64_t rows, int hkv, const int8_t *signs, uint8_t *q, void *scales,
                              float scale_mul, float sqrt_n, cudaStream_t st, int dev, int sms,
                              uint64_t wait_limit_ns, int64_t withheld_tile)
{
    auto kern = kv_quant_tma_kernel<ROTATE>;
    int per_sm = 0;
    quarot_status_t s = kernel_occupancy(kern, dev, kKvTileRows, kKvSmemBytes, per_sm);
    if (s != QUAROT_OK)
        return s;
    CUtensorMap map;
    s = kv_map(map, x, rows);
    if (s != QUAROT_OK)
        return s;
    const int64_t tiles = (rows + kKvTileRows - 1) / kKvTileRows;
    const int grid = (int)std::min<int64_t>(tiles, (int64_t)sms * per_sm);
    kern<<<grid, kKvTileRows, kKvSmemBytes, st>>>(map, rows, hkv, signs, q, static_cast<__half *>(scales), scale_mul,
                                                 sqrt_n, wait_limit_ns, withheld_tile);
    return after_launch("kv_quant_tma_kernel launch");
}

// ======================================================================= C ABI
extern "C" {

quarot_status_t quarot_rotate_quant(const void *x_f16, int64_t M, int64_t K, const int8_t *signs, int had_block,
                                    int group, uint8_t *q_packed, void *scales, quarot_stream_t stream)
{
    quarot_status_t s = check_rotate_args(x_f16, M, K, signs, had_block, group, q_packed, scales);
    if (s != QUAROT_OK || M == 0)
        return s;
    return rotate_quant_launch(x_f16, M, K, signs, had_block, group, q_packed, scales, (cudaStream_t)stream);
}

quarot_status_t quarot_rotate_quant_kron(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                         int64_t group, uint8_t *q_packed, void *scales, quarot_stream_t stream)
{
    if (M < 0)
        return fail(QUAROT_ERR_INVALID_ARG, "M must be >= 0");
    if (group != 0 && group != 128)
        return fail(QUAROT_ERR_INVALID_ARG, "group must be 0 or 128");
    if (K != kKronK)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "the full Kronecker rotation supports K = 11008 = 344 * 32");
    if (M == 0)
        return QUAROT_OK;
    if (!x_f16 || !signs || !q_packed || !scales)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x_f16) || !aligned16(signs) || !aligned16(q_packed) || !aligned16(scales))
        return fail(QUAROT_ERR_MISALIGNED, "x, signs, codes and scales must be 16-byte aligned");
    return kron_launch(x_f16, M, signs, (int)group, q_packed, scales, (cudaStream_t)stream);
}

quarot_status_t quarot_kron_factor(int64_t m, int8_t *h_out)
{
    if (m != kKronM)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "the library's non-power-of-two factor has order 344");
    if (!h_out)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    paley344(h_out);
    return QUAROT_OK;
}

quarot_status_t quarot_int4_linear(const uint8_t *qa, const void *s_a, int64_t M, const uint8_t *qw,
                                   const void *s_w, int64_t N, int64_t K, int group, void *out_f16,
                                   quarot_stream_t stream)
{
    if (group != 0 && group != 128)
        return fail(QUAROT_ERR_INVALID_ARG, "group must be 0 or 128");
    quarot_status_t s = check_gemm_args(qa, M, qw, N, K, out_f16, s_a, s_w, true);
    if (s != QUAROT_OK || M == 0)
        return s;
    return linear_launch(qa, s_a, M, qw, s_w, N, K, group, out_f16, (cudaStream_t)stream, false);
}

quarot_status_t quarot_int4_gemm_s32(const uint8_t *qa, int64_t M, const uint8_t *qw, int64_t N, int64_t K,
                                     int32_t *acc, quarot_stream_t stream)
{
    quarot_status_t s = check_gemm_args(qa, M, qw, N, K, acc, nullptr, nullptr, false);
    if (s != QUAROT_OK || M == 0)
        return s;
    GemmArgs a = {};
    a.qa = qa;
    a.qw = qw;
    a.out = acc;
    a.M = M;
    a.N = N;
    a.K = K;
    return launch_gemm_pair<kEpiS32>(a, (cudaStream_t)stream, false);
}

size_t quarot_rotate_quant_linear_workspace(int64_t M, int64_t K, int group)
{
    if (M <= 0 || K <= 0)
        return 0;
    const size_t q = align256((size_t)M * (size_t)(K / 2));
    const size_t sc = group == 0 ? (size_t)M * 4 : (size_t)M * (size_t)(K / 128) * 2;
    return q + align256(sc);
}

quarot_status_t quarot_rotate_quant_linear(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                           int had_block, int group, const uint8_t *qw, const void *s_w,
                                           int64_t N, void *workspace, size_t ws_bytes, void *out_f16,
                                           quarot_stream_t stream)
{
    quarot_status_t s = check_rotate_args(x_f16, M, K, signs, had_block, group, workspace, workspace);
    if (s != QUAROT_OK)
        return s;
    s = check_gemm_args(workspace, M, qw, N, K, out_f16, workspace, s_w, true);
    if (s != QUAROT_OK || M == 0)
        return s;
    const size_t need = quarot_rotate_quant_linear_workspace(M, K, group);
    if (ws_bytes < need)
        return fail(QUAROT_ERR_INVALID_ARG, "workspace too small");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(QUAROT_ERR_MISALIGNED, "workspace must be 256-byte aligned");
    uint8_t *qa = static_cast<uint8_t *>(workspace);
    void *sa = qa + align256((size_t)M * (size_t)(K / 2));
    cudaStream_t st = (cudaStream_t)stream;
    s = rotate_quant_launch(x_f16, M, K, signs, had_block, group, qa, sa, st);
    if (s != QUAROT_OK)
        return s;
    return linear_launch(qa, sa, M, qw, s_w, N, K, group, out_f16, st, true);
}

quarot_status_t quarot_rotate_quant_linear_noalloc(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                                   int had_block, int group, const uint8_t *qw, const void *s_w,
                                                   int64_t N, void *out_f16, quarot_stream_t stream)
{
    // the scratch stands in for the quantized activations and their scales
    quarot_status_t s = check_rotate_args(x_f16, M, K, signs, had_block, group, out_f16, out_f16);
    if (s != QUAROT_OK)
        return s;
    s = check_gemm_args(out_f16, M, qw, N, K, out_f16, out_f16, s_w, true);
    if (s != QUAROT_OK || M == 0)
        return s;
    const size_t need = quarot_rotate_quant_linear_workspace(M, K, group);
    if (need > kNoAllocScratchBytes)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE,
                    "these sizes need " + std::to_string(need) + " bytes of scratch; the built-in scratch holds " +
                        std::to_string(kNoAllocScratchBytes) + " (QUAROT_NOALLOC_SCRATCH_BYTES)");
    int dev;
    DeviceInfo *info;
    s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    void *scratch = nullptr;
    s = noalloc_scratch_address(dev, scratch);
    if (s != QUAROT_OK)
        return s;
    uint8_t *qa = static_cast<uint8_t *>(scratch);
    void *sa = qa + align256((size_t)M * (size_t)(K / 2));
    cudaStream_t st = (cudaStream_t)stream;
    s = rotate_quant_launch(x_f16, M, K, signs, had_block, group, qa, sa, st);
    if (s != QUAROT_OK)
        return s;
    return linear_launch(qa, sa, M, qw, s_w, N, K, group, out_f16, st, true);
}

quarot_status_t quarot_rotate_quant_i8(const void *x_f16, int64_t M, int64_t K, const int8_t *signs, int had_block,
                                       int8_t *q, float *scales, quarot_stream_t stream)
{
    quarot_status_t s = check_rotate_args(x_f16, M, K, signs, had_block, 0, q, scales);
    if (s != QUAROT_OK || M == 0)
        return s;
    return rotate_quant_launch(x_f16, M, K, signs, had_block, 0, reinterpret_cast<uint8_t *>(q), scales,
                               (cudaStream_t)stream, 8);
}

quarot_status_t quarot_rotate_quant_i6(const void *x_f16, int64_t M, int64_t K, const int8_t *signs, int had_block,
                                       int8_t *q, float *scales, quarot_stream_t stream)
{
    quarot_status_t s = check_rotate_args(x_f16, M, K, signs, had_block, 0, q, scales);
    if (s != QUAROT_OK || M == 0)
        return s;
    return rotate_quant_launch(x_f16, M, K, signs, had_block, 0, reinterpret_cast<uint8_t *>(q), scales,
                               (cudaStream_t)stream, 6);
}

quarot_status_t quarot_int8_linear(const int8_t *qa, const float *s_a, int64_t M, const int8_t *qw, const float *s_w,
                                   int64_t N, int64_t K, void *out_f16, quarot_stream_t stream)
{
    quarot_status_t s = check_gemm_args(qa, M, qw, N, K, out_f16, s_a, s_w, true);
    if (s != QUAROT_OK || M == 0)
        return s;
    return linear8_launch(qa, s_a, M, qw, s_w, N, K, out_f16, (cudaStream_t)stream, false);
}

quarot_status_t quarot_int8_gemm_s32(const int8_t *qa, int64_t M, const int8_t *qw, int64_t N, int64_t K,
                                     int32_t *acc, quarot_stream_t stream)
{
    quarot_status_t s = check_gemm_args(qa, M, qw, N, K, acc, nullptr, nullptr, false);
    if (s != QUAROT_OK || M == 0)
        return s;
    GemmArgs a = {};
    a.qa = reinterpret_cast<const uint8_t *>(qa);
    a.qw = reinterpret_cast<const uint8_t *>(qw);
    a.out = acc;
    a.M = M;
    a.N = N;
    a.K = K;
    return launch_gemm_i8<kEpiS32>(a, (cudaStream_t)stream, false);
}

size_t quarot_rotate_quant_linear_i8_workspace(int64_t M, int64_t K)
{
    if (M <= 0 || K <= 0)
        return 0;
    return align256((size_t)M * (size_t)K) + align256((size_t)M * 4);
}

namespace {
// The fused path of the byte-code variants (bits 6 or 8): quantizer into the
// workspace, then the INT8 tensor-core GEMM as its programmatic dependent.
quarot_status_t rotate_quant_linear_bytes(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                          int had_block, const int8_t *qw, const float *s_w, int64_t N,
                                          void *workspace, size_t ws_bytes, void *out_f16, quarot_stream_t stream,
                                          int bits)
{
    quarot_status_t s = check_rotate_args(x_f16, M, K, signs, had_block, 0, workspace, workspace);
    if (s != QUAROT_OK)
        return s;
    s = check_gemm_args(workspace, M, qw, N, K, out_f16, workspace, s_w, true);
    if (s != QUAROT_OK || M == 0)
        return s;
    const size_t need = quarot_rotate_quant_linear_i8_workspace(M, K);
    if (ws_bytes < need)
        return fail(QUAROT_ERR_INVALID_ARG, "workspace too small");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(QUAROT_ERR_MISALIGNED, "workspace must be 256-byte aligned");
    int8_t *qa = static_cast<int8_t *>(workspace);
    float *sa = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + align256((size_t)M * (size_t)K));
    cudaStream_t st = (cudaStream_t)stream;
    s = rotate_quant_launch(x_f16, M, K, signs, had_block, 0, reinterpret_cast<uint8_t *>(qa), sa, st, bits);
    if (s != QUAROT_OK)
        return s;
    return linear8_launch(qa, sa, M, qw, s_w, N, K, out_f16, st, true);
}
}  // namespace

quarot_status_t quarot_rotate_quant_linear_i8(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                              int had_block, const int8_t *qw, const float *s_w, int64_t N,
                                              void *workspace, size_t ws_bytes, void *out_f16,
                                              quarot_stream_t stream)
{
    return rotate_quant_linear_bytes(x_f16, M, K, signs, had_block, qw, s_w, N, workspace, ws_bytes, out_f16, stream,
                                     8);
}

quarot_status_t quarot_rotate_quant_linear_i6(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                              int had_block, const int8_t *qw, const float *s_w, int64_t N,
                                              void *workspace, size_t ws_bytes, void *out_f16,
                                              quarot_stream_t stream)
{
    return rotate_quant_linear_bytes(x_f16, M, K, signs, had_block, qw, s_w, N, workspace, ws_bytes, out_f16, stream,
                                     6);
}

quarot_status_t quarot_rotate_quant_asym(const void *x_f16, int64_t M, int64_t K, const int8_t *signs, int had_block,
                                         float clip, uint8_t *q_packed, float *scales, int32_t *zeros,
                                         int32_t *rowsums, quarot_stream_t stream)
{
    quarot_status_t s = check_rotate_args(x_f16, M, K, signs, had_block, 0, q_packed, scales);
    if (s != QUAROT_OK)
        return s;
    if (!(clip > 0.0f) || clip > 1.0f)
        return fail(QUAROT_ERR_INVALID_ARG, "clip must lie in (0, 1]");
    if (had_block != 0 || K < 256)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "asymmetric quantization needs the full Hadamard, 256 <= K <= 8192");
    if (M == 0)
        return QUAROT_OK;
    if (!zeros || !rowsums)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(zeros) || !aligned16(rowsums))
        return fail(QUAROT_ERR_MISALIGNED, "zeros and rowsums must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    return dispatch_fwht_asym(ilog2(K), x_f16, M, signs, q_packed, scales, AsymOut{zeros, rowsums, clip},
                              (cudaStream_t)stream, dev, info->sm_count);
}

quarot_status_t quarot_uint4_gemm_s32(const uint8_t *qa, int64_t M, const uint8_t *qw, int64_t N, int64_t K,
                                      int32_t *acc, quarot_stream_t stream)
{
    quarot_status_t s = check_gemm_args(qa, M, qw, N, K, acc, nullptr, nullptr, false);
    if (s != QUAROT_OK || M == 0)
        return s;
    GemmArgs a = {};
    a.qa = qa;
    a.qw = qw;
    a.out = acc;
    a.M = M;
    a.N = N;
    a.K = K;
    return launch_gemm_pair<kEpiS32, true>(a, (cudaStream_t)stream, false);
}

quarot_status_t quarot_int4_linear_asym(const uint8_t *qa, const float *s_a, const int32_t *z_a, const int32_t *r_a,
                                        int64_t M, const uint8_t *qw, const float *s_w, const int32_t *z_w,
                                        const int32_t *r_w, int64_t N, int64_t K, void *out_f16,
                                        quarot_stream_t stream)
{
    quarot_status_t s = check_gemm_args(qa, M, qw, N, K, out_f16, s_a, s_w, true);
    if (s != QUAROT_OK || M == 0)
        return s;
    if (!z_a || !r_a || !z_w || !r_w)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(z_a) || !aligned16(r_a) || !aligned16(z_w) || !aligned16(r_w))
        return fail(QUAROT_ERR_MISALIGNED, "zero points and code sums must be 16-byte aligned");
    GemmArgs a = {};
    a.qa = qa;
    a.sa = s_a;
    a.za = z_a;
    a.ra = r_a;
    a.qw = qw;
    a.sw = s_w;
    a.zw = z_w;
    a.rw = r_w;
    a.out = out_f16;
    a.M = M;
    a.N = N;
    a.K = K;
    return launch_gemm_pair<kEpiAsymF16, true>(a, (cudaStream_t)stream, false);
}

quarot_status_t quarot_kv_quant(const void *k_f16, const void *v_f16, int64_t B, int64_t T, int64_t Hkv, int64_t D,
                                const int8_t *signs, uint8_t *kq, void *ks_f16, uint8_t *vq, void *vs_f16,
                                quarot_stream_t stream)
{
    if (B < 0 || T < 0 || Hkv <= 0)
        return fail(QUAROT_ERR_INVALID_ARG, "B, T must be >= 0 and Hkv > 0");
    if (D != 128)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "head dimension must be 128");
    if (Hkv > 512)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "at most 512 KV heads");
    const int64_t rows = B * T;
    if (rows == 0)
        return QUAROT_OK;
    if (!k_f16 || !v_f16 || !signs || !kq || !ks_f16 || !vq || !vs_f16)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(k_f16) || !aligned16(v_f16) || !aligned16(kq) || !aligned16(vq) || !aligned16(ks_f16) ||
        !aligned16(vs_f16))
        return fail(QUAROT_ERR_MISALIGNED, "K, V, codes and scales must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    const int64_t W = Hkv * D;
    cudaStream_t st = (cudaStream_t)stream;
    const float kmul = (float)(1.0 / (7.0 * std::sqrt(128.0)));
    const float ksq = (float)std::sqrt(128.0);
    if (rows * Hkv < (int64_t(1) << 31) - kKvTileRows) {
        // rows of [B T Hkv, 128] staged by the copy engine
        const int64_t n = rows * Hkv;
        s = launch_kv_tma<true>(k_f16, n, (int)Hkv, signs, kq, ks_f16, kmul, ksq, st, dev, info->sm_count);
        if (s != QUAROT_OK)
            return s;
        return launch_kv_tma<false>(v_f16, n, (int)Hkv, nullptr, vq, vs_f16, (float)(1.0 / 7.0), 1.0f, st, dev,
                                    info->sm_count);
    }
    s = launch_block<true, 128>(k_f16, rows, W, signs, kq, ks_f16, kmul, ksq, st, dev, info->sm_count);
    if (s != QUAROT_OK)
        return s;
    return launch_block<false, 128>(v_f16, rows, W, nullptr, vq, vs_f16, (float)(1.0 / 7.0), 1.0f, st, dev,
                                    info->sm_count);
}

quarot_status_t quarot_kv_decode_scores(const void *q_f16, int64_t Hq, const int8_t *signs, const uint8_t *kq,
                                        const void *ks_f16, int64_t B, int64_t T, int64_t Hkv, int64_t D,
                                        float *scores, quarot_stream_t stream)
{
    if (B < 0 || T < 0 || Hkv <= 0 || Hq <= 0)
        return fail(QUAROT_ERR_INVALID_ARG, "B, T must be >= 0; Hq, Hkv > 0");
    if (D != 128)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "head dimension must be 128");
    if (Hq % Hkv != 0)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "Hq must be a multiple of Hkv");
    const int64_t G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "Hq / Hkv must be 1, 2, 4, 8 or 16");
    if (Hkv > 65535 || B > 65535)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "B and Hkv must be <= 65535");
    if (B == 0 || T == 0)
        return QUAROT_OK;
    if (!q_f16 || !signs || !kq || !ks_f16 || !scores)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q_f16) || !aligned16(kq) || !aligned16(ks_f16) || !aligned16(scores))
        return fail(QUAROT_ERR_MISALIGNED, "q, codes, scales and scores must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    cudaStream_t st = (cudaStream_t)stream;
    const __half *qh = static_cast<const __half *>(q_f16);
    const __half *ksh = static_cast<const __half *>(ks_f16);
    const int hkv = (int)Hkv;
    switch (G) {
    case 1: return launch_scores_tc<1>(qh, signs, kq, ksh, B, T, hkv, scores, st, dev);
    case 2: return launch_scores_tc<2>(qh, signs, kq, ksh, B, T, hkv, scores, st, dev);
    case 4: return launch_scores_tc<4>(qh, signs, kq, ksh, B, T, hkv, scores, st, dev);
    case 8: return launch_scores_tc<8>(qh, signs, kq, ksh, B, T, hkv, scores, st, dev);
    default: return launch_scores_tc<16>(qh, signs, kq, ksh, B, T, hkv, scores, st, dev);
    }
}

quarot_status_t quarot_kv_decode_attend(const float *scores, int64_t B, int64_t Hq, const uint8_t *vq,
                                        const void *vs_f16, int64_t T, int64_t Hkv, int64_t D, float *out,
                                        quarot_stream_t stream)
{
    if (B < 0 || T <= 0 || Hkv <= 0 || Hq <= 0)
        return fail(QUAROT_ERR_INVALID_ARG, "B must be >= 0; T, Hq, Hkv > 0");
    if (D != 128)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "head dimension must be 128");
    if (Hq % Hkv != 0)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "Hq must be a multiple of Hkv");
    const int64_t G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "Hq / Hkv must be 1, 2, 4, 8 or 16");
    if (Hkv > 65535 || B > 65535)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "B and Hkv must be <= 65535");
    if (B == 0)
        return QUAROT_OK;
    if (!scores || !vq || !vs_f16 || !out)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(scores) || !aligned16(vq) || !aligned16(vs_f16) || !aligned16(out))
        return fail(QUAROT_ERR_MISALIGNED, "scores, codes, scales and output must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    // tokens split over a cluster of S CTAs, at least 128 tokens each: the S
    // whose B * Hkv * S CTAs fill the resident slots best (CTAs / (waves x
    // resident CTAs)); on a tie the one with fewer waves (no tail wave that
    // runs on a few SMs only)
    const int smax = T >= 1024 ? 8 : T >= 512 ? 4 : T >= 256 ? 2 : 1;
    int split = smax;
    double best_eff = -1.0;
    int64_t best_waves = 0;
    for (int sp = smax; sp >= 1; sp /= 2) {
        int fit = 0;
        s = attend_resident_clusters((int)G, sp, dev, fit);
        if (s != QUAROT_OK)
            return s;
        const int64_t clusters = B * Hkv;
        const int64_t waves = fit > 0 ? (clusters + fit - 1) / fit : clusters;
        const double eff = fit > 0 ? (double)clusters / ((double)waves * fit) : 0.0;
        if (eff > best_eff + 1e-9 || (eff > best_eff - 1e-9 && waves < best_waves)) {
            best_eff = eff;
            best_waves = waves;
            split = sp;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)split, (unsigned)Hkv, (unsigned)B);
    cfg.blockDim = dim3(kAttThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const __half *vsh = static_cast<const __half *>(vs_f16);
    const int hkv = (int)Hkv;
    cudaError_t e;
    switch (G) {
    case 1: e = cudaLaunchKernelEx(&cfg, kv_attend_kernel<1>, scores, vq, vsh, T, hkv, out); break;
    case 2: e = cudaLaunchKernelEx(&cfg, kv_attend_kernel<2>, scores, vq, vsh, T, hkv, out); break;
    case 4: e = cudaLaunchKernelEx(&cfg, kv_attend_kernel<4>, scores, vq, vsh, T, hkv, out); break;
    case 8: e = cudaLaunchKernelEx(&cfg, kv_attend_kernel<8>, scores, vq, vsh, T, hkv, out); break;
    default: e = cudaLaunchKernelEx(&cfg, kv_attend_kernel<16>, scores, vq, vsh, T, hkv, out); break;
    }
    if (e != cudaSuccess)
        return cuda_fail(e, "kv_attend_kernel launch");
    return after_launch("kv_attend_kernel launch");
}

quarot_status_t quarot_probe_mma_i8(int64_t steps, int operands, int64_t *pairs, quarot_stream_t stream)
{
    if (steps < 1 || steps > (int64_t(1) << 22))
        return fail(QUAROT_ERR_INVALID_ARG, "steps must lie in [1, 2^22]");
    if (operands < 0 || operands > 2)
        return fail(QUAROT_ERR_INVALID_ARG, "operands must be 0 (zeros), 1 (random bytes) or 2 (random 4-bit codes)");
    if (!pairs)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    using S = MmaPeakShape;
    int per_sm = 0;
    s = kernel_occupancy(mma_peak_i8_kernel, dev, S::kThreads, S::kSmemBytes, per_sm);
    if (s != QUAROT_OK)
        return s;
    const int clusters = info->sm_count / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(S::kThreads);
    cfg.dynamicSmemBytes = S::kSmemBytes;
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, mma_peak_i8_kernel, steps, operands);
    if (e != cudaSuccess)
        return cuda_fail(e, "mma_peak_i8_kernel launch");
    *pairs = clusters;
    return after_launch("mma_peak_i8_kernel launch");
}

quarot_status_t quarot_test_wait_timeout(const void *v_f16, int64_t rows, uint8_t *q_packed, void *scales_f16,
                                         int64_t withheld_tile, uint64_t wait_limit_ns, quarot_stream_t stream)
{
    if (rows <= 0 || rows >= (int64_t(1) << 31) - kKvTileRows)
        return fail(QUAROT_ERR_INVALID_ARG, "rows must lie in [1, 2^31 - 128)");
    const int64_t tiles = (rows + kKvTileRows - 1) / kKvTileRows;
    if (withheld_tile < 0 || withheld_tile >= tiles)
        return fail(QUAROT_ERR_INVALID_ARG, "withheld_tile must name one of the tiles of 128 rows");
    if (wait_limit_ns < 100000ull || wait_limit_ns > kKvWaitLimitNs)
        return fail(QUAROT_ERR_INVALID_ARG, "wait_limit_ns must lie in [1e5, 2e9]");
    if (!v_f16 || !q_packed || !scales_f16)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(v_f16) || !aligned16(q_packed) || !aligned16(scales_f16))
        return fail(QUAROT_ERR_MISALIGNED, "rows, codes and scales must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    return launch_kv_tma<false>(v_f16, rows, 1, nullptr, q_packed, scales_f16, (float)(1.0 / 7.0), 1.0f,
                                (cudaStream_t)stream, dev, info->sm_count, wait_limit_ns, withheld_tile);
}

quarot_status_t quarot_kv_decode_attention(const void *q_f16, int64_t Hq, const int8_t *signs, const uint8_t *kq,
                                           const void *ks_f16, const uint8_t *vq, const void *vs_f16, int64_t B,
                                           int64_t T, int64_t Hkv, int64_t D, float *out, quarot_stream_t stream)
{
    if (B < 0 || T <= 0 || Hkv <= 0 || Hq <= 0)
        return fail(QUAROT_ERR_INVALID_ARG, "B must be >= 0; T, Hq, Hkv > 0");
    if (D != 128)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "head dimension must be 128");
    if (Hq % Hkv != 0)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "Hq must be a multiple of Hkv");
    const int64_t G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "Hq / Hkv must be 1, 2, 4, 8 or 16");
    if (Hkv > 65535 || B > 65535)
        return fail(QUAROT_ERR_UNSUPPORTED_SHAPE, "B and Hkv must be <= 65535");
    if (B == 0)
        return QUAROT_OK;
    if (!q_f16 || !signs || !kq || !ks_f16 || !vq || !vs_f16 || !out)
        return fail(QUAROT_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q_f16) || !aligned16(kq) || !aligned16(ks_f16) || !aligned16(vq) || !aligned16(vs_f16) ||
        !aligned16(out))
        return fail(QUAROT_ERR_MISALIGNED, "q, codes, scales and output must be 16-byte aligned");
    int dev;
    DeviceInfo *info;
    quarot_status_t s = current_device(dev, info);
    if (s != QUAROT_OK)
        return s;
    const __half *qh = static_cast<const __half *>(q_f16);
    const __half *ksh = static_cast<const __half *>(ks_f16);
    const __half *vsh = static_cast<const __half *>(vs_f16);
    cudaStream_t st = (cudaStream_t)stream;
    const int hkv = (int)Hkv;
    switch (G) {
    case 1: return launch_decode_tc<1>(qh, signs, kq, ksh, vq, vsh, B, T, hkv, out, st, dev);
    case 2: return launch_decode_tc<2>(qh, signs, kq, ksh, vq, vsh, B, T, hkv, out, st, dev);
    case 4: return launch_decode_tc<4>(qh, signs, kq, ksh, vq, vsh, B, T, hkv, out, st, dev);
    case 8: return launch_decode_tc<8>(qh, signs, kq, ksh, vq, vsh, B, T, hkv, out, st, dev);
    default: return launch_decode_tc<16>(qh, signs, kq, ksh, vq, vsh, B, T, hkv, out, st, dev);
    }
}

quarot_status_t quarot_get_device_status(quarot_stream_t stream)
{
    cudaError_t e = stream ? cudaStreamSynchronize((cudaStream_t)stream) : cudaDeviceSynchronize();
    if (e != cudaSuccess)
        return cuda_fail(e, stream ? "cudaStreamSynchronize" : "cudaDeviceSynchronize");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
    if (e != cudaSuccess)
        return cuda_fail(e, "read device status");
    if (v != kDevOk) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
        if (v & kDevBounds)
            return fail(QUAROT_ERR_DEVICE_BOUNDS, "a kernel skipped a store outside its output (bounds-checking build)");
        return fail(QUAROT_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait");
    }
    return QUAROT_OK;
}

int quarot_debug_bounds(void)
{
#ifdef QUAROT_DEBUG_BOUNDS
    return 1;
#else
    return 0;
#endif
}

const char *quarot_status_string(quarot_status_t status)
{
    switch (status) {
    case QUAROT_OK: return "QUAROT_OK";
    case QUAROT_ERR_INVALID_ARG: return "QUAROT_ERR_INVALID_ARG";
    case QUAROT_ERR_UNSUPPORTED_SHAPE: return "QUAROT_ERR_UNSUPPORTED_SHAPE";
    case QUAROT_ERR_MISALIGNED: return "QUAROT_ERR_MISALIGNED";
    case QUAROT_ERR_CUDA: return "QUAROT_ERR_CUDA";
    case QUAROT_ERR_DEVICE_TIMEOUT: return "QUAROT_ERR_DEVICE_TIMEOUT";
    case QUAROT_ERR_DEVICE_BOUNDS: return "QUAROT_ERR_DEVICE_BOUNDS";
    case QUAROT_ERR_NO_DEVICE: return "QUAROT_ERR_NO_DEVICE";
    }
    return "QUAROT_ERR_UNKNOWN";
}

const char *quarot_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
