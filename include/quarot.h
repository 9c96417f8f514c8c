/*
 * quarot.h -- C ABI of libquarot, the B200 (sm_100a) hot path of QuaRot
 * inference: online randomized Hadamard rotation + INT4 round-to-nearest
 * quantization, INT4 x INT4 linear layers with a dequantizing epilogue, and
 * an INT4 KV cache with a per-head Hadamard.
 *
 * Sources (page title, section):
 *  [QR-A] QuaRot: Outlier-free 4-bit inference in rotated LLMs -- ISTA research
 *         explorer record, abstract: weights, activations and KV cache in 4
 *         bits; rotations leave the output unchanged; all matrix
 *         multiplications in 4 bits.
 *  [QR-S] QuaRot: Outlier-Free 4-Bit Inference in Rotated LLMs -- Elamur
 *         Research summary, "Summary" (random orthogonal Hadamard matrices,
 *         most fused into the weights, a few applied at inference; products
 *         in integers) and "Key points" (activations quantized on the fly with
 *         round-to-nearest; group-wise variant with group size 128).
 *  [QR-R] The same summary, References, item 24: Sloane's library of Hadamard
 *         matrices, the source of factors whose order is not a power of two.
 *  [QR-N] QuaRot news article (onlyaistuff.com): randomized Hadamard
 *         transformations and computational invariance.
 *  [DQ-1], [DQ-2], [DQ-12] DuQuant (chapterpal) Knowl 1 (Y = XW =
 *         (XG)(G^-1 W)), Knowl 2 (block-diagonal rotations of 2^n channels),
 *         Knowl 12 (block size 128; a fixed +-1/sqrt(2^n) Hadamard on the
 *         query-key product with per-head quantization).
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE memory owned by the caller; the library
 *    allocates nothing and keeps no state beyond a per-device cache of kernel
 *    attributes and two device arrays compiled into it: the 288 KB Hadamard
 *    factor of the full Kronecker rotation (filled by that call's first use
 *    on a device) and the scratch of quarot_rotate_quant_linear_noalloc.
 *  - Every array pointer must be 16-byte aligned; arrays are dense row-major.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Argument errors are returned before any launch and
 *    leave every output untouched.  A launch failure returns
 *    QUAROT_ERR_CUDA; quarot_last_error() then gives the CUDA message.
 *  - fp16 is IEEE binary16.  INT4 codes are two's complement in [-8, 7],
 *    packed two per byte: element 2i in bits 0-3, element 2i+1 in bits 4-7.
 *  - No function throws; none blocks the host except
 *    quarot_get_device_status() (and the first quarot_rotate_quant_kron on a
 *    device, which copies its factor).
 */
#ifndef QUAROT_H
#define QUAROT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QUAROT_OK = 0,
    QUAROT_ERR_INVALID_ARG = 1,      /* null pointer, negative size, bad enum value */
    QUAROT_ERR_UNSUPPORTED_SHAPE = 2,/* a size outside the limits stated per call */
    QUAROT_ERR_MISALIGNED = 3,       /* a pointer not 16-byte aligned */
    QUAROT_ERR_CUDA = 4,             /* the CUDA runtime reported an error */
    QUAROT_ERR_DEVICE_TIMEOUT = 5,   /* a kernel gave up a bounded wait (see below) */
    QUAROT_ERR_NO_DEVICE = 6,        /* no sm_100 device is current */
    QUAROT_ERR_DEVICE_BOUNDS = 7     /* bounds-checking build only: a kernel skipped a store
                                        outside its output (see quarot_debug_bounds) */
} quarot_status_t;

/* A cudaStream_t passed as an opaque pointer. */
typedef void *quarot_stream_t;

/*
 * quarot_rotate_quant -- online rotation + INT4 RTN quantization + packing
 * of activations [QR-S Summary, Key points; QR-N; DQ-2; DQ-12].
 *
 *   x'  = (x * diag(signs)) * R,  R = H_K / sqrt(K)              (had_block == 0)
 *                                 R = I_{K/128} (x) H_128/sqrt(128) (had_block == 128)
 *   H is the Sylvester-ordered Hadamard matrix.
 *   group == 0:   s[m] = max_k |x'[m,k]| / 7, stored fp32;  q = rint(x'/s)
 *   group == 128: s[m,g] = fp16(max over the 128-group |x'| / 7); q = clamp(rint(x'/s16), -8, 7)
 *   (round half to even; a zero stored scale gives zero codes.)
 * The rotated values are kept in fp32 inside the kernel and never stored.
 * The same call prepares weights offline (rows of W are rows of x; group 0
 * then gives one fp32 scale per output channel) [QR-S Summary].
 *
 * x_f16     [M, K] fp16, read only.
 * signs     [K] int8, each +1 or -1 (any negative value counts as -1).
 * had_block 0 (K a power of two, 128 <= K <= 8192) or 128 (K % 128 == 0,
 *           128 <= K <= 65536).
 * group     0 or 128.
 * q_packed  [M, K/2] uint8 output.
 * scales    group 0: fp32 [M]; group 128: fp16 [M, K/128].  Output.
 * M         >= 0; M == 0 launches nothing and returns QUAROT_OK.
 */
quarot_status_t quarot_rotate_quant(const void *x_f16, int64_t M, int64_t K,
                                    const int8_t *signs, int had_block, int group,
                                    uint8_t *q_packed, void *scales, quarot_stream_t stream);

/*
 * quarot_rotate_quant_kron -- the full (not block-diagonal) rotation for
 * K = 11008, which is not a power of two, fused with INT4 RTN quantization
 * and packing [QR-S Summary, Key points; QR-R; DQ-1]:
 *
 *   x' = (x * diag(signs)) * (H_344 (x) H_32) / sqrt(11008),  element i = 32 a + b,
 *   (H_344 (x) H_32)[32a + b][32a' + b'] = H_344[a][a'] * H_32[b][b'],
 *
 * H_32 Sylvester-ordered; H_344 the library's Hadamard matrix of order 344
 * (Paley's first construction over GF(7^3) = GF(7)[x]/(x^3 + 2), elements
 * c0 + c1 x + c2 x^2 numbered c0 + 7 c1 + 49 c2; quarot_kron_factor returns
 * it).  Quantization exactly as quarot_rotate_quant (group 0: fp32 scale per
 * row; group 128: fp16 scale per 128 elements).  Every output element mixes
 * all 11008 inputs, unlike had_block == 128.
 *
 * x_f16 [M, 11008] fp16; signs [11008] int8 (+1 / -1); q_packed [M, 5504]
 * uint8 out; scales fp32 [M] (group 0) or fp16 [M, 86] (group 128) out.
 * K must be 11008 (else QUAROT_ERR_UNSUPPORTED_SHAPE).  The factor lives in
 * a 288 KB device array compiled into the library (nothing is allocated);
 * the first call on a device fills it with a synchronous host-to-device copy,
 * so make that first call outside any stream capture.
 */
quarot_status_t quarot_rotate_quant_kron(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                         int64_t group, uint8_t *q_packed, void *scales, quarot_stream_t stream);

/*
 * quarot_kron_factor -- writes the library's Hadamard factor of order m
 * (only m == 344) to HOST memory h_out[m * m] (int8 +1 / -1, row-major), for
 * rotating weights offline with the same matrix [QR-S Summary: the rotations
 * are folded into the weights].  H H^T = m I.  Needs no device.
 */
quarot_status_t quarot_kron_factor(int64_t m, int8_t *h_out);

/*
 * quarot_int4_linear -- INT4 x INT4 linear layer with int32 accumulation on
 * the tensor cores and a fused dequantizing epilogue [QR-A: all matrix
 * multiplications in 4 bits; QR-S Summary: integer products].
 *
 *   group == 0:   out[m,n] = fp16( acc[m,n] * s_a[m] * s_w[n] ),
 *                 acc[m,n] = sum_k qa[m,k] * qw[n,k]  (int32, exact)
 *   group == 128: out[m,n] = fp16( sum_g acc_g[m,n] * s_a[m,g] * s_w[n,g] ),
 *                 acc_g over k in [128g, 128g+128), sum in fp32
 *
 * qa   [M, K/2] packed INT4 activations (from quarot_rotate_quant).
 * s_a  group 0: fp32 [M]; group 128: fp16 [M, K/128].
 * qw   [N, K/2] packed INT4 weights, the rows rotated with the same signs and
 *      Hadamard as the activations (computational invariance [DQ-1]).
 * s_w  group 0: fp32 [N]; group 128: fp16 [N, K/128].
 * out  [M, N] fp16 output.
 * Limits: M >= 0 (0 launches nothing), N >= 1 with N % 8 == 0,
 *         K % 128 == 0 with 128 <= K <= 65536.
 */
quarot_status_t quarot_int4_linear(const uint8_t *qa, const void *s_a, int64_t M,
                                   const uint8_t *qw, const void *s_w, int64_t N, int64_t K,
                                   int group, void *out_f16, quarot_stream_t stream);

/*
 * quarot_int4_gemm_s32 -- the same integer product without the epilogue:
 * acc[m,n] = sum_k qa[m,k] * qw[n,k] written as int32 [M, N].  Exact for
 * every input (|acc| <= 64 K).  Same layouts and limits as
 * quarot_int4_linear (no scales).  For testing the integer path in
 * isolation [QR-S Summary: matrix multiplications in integers].
 */
quarot_status_t quarot_int4_gemm_s32(const uint8_t *qa, int64_t M, const uint8_t *qw,
                                     int64_t N, int64_t K, int32_t *acc,
                                     quarot_stream_t stream);

/*
 * quarot_rotate_quant_linear_workspace -- bytes of device workspace that
 * quarot_rotate_quant_linear needs for M tokens of K channels: the packed
 * INT4 activations and their scales, each at a 256-byte aligned offset.
 */
size_t quarot_rotate_quant_linear_workspace(int64_t M, int64_t K, int group);

/*
 * quarot_rotate_quant_linear -- the fused online path of one linear layer:
 * quarot_rotate_quant of x into `workspace`, then quarot_int4_linear against
 * the prepared weights, both on `stream`; the GEMM is launched as a
 * programmatic dependent of the quantizer so that its set-up overlaps the
 * quantizer's tail [QR-S Summary: a few rotations are performed online].
 *
 * Arguments as in the two calls above.  workspace: caller-owned device
 * memory of at least quarot_rotate_quant_linear_workspace(M, K, group) bytes,
 * 256-byte aligned; its contents are scratch (overwritten, no meaning after
 * the call).  ws_bytes: its size.
 */
quarot_status_t quarot_rotate_quant_linear(const void *x_f16, int64_t M, int64_t K,
                                           const int8_t *signs, int had_block, int group,
                                           const uint8_t *qw, const void *s_w, int64_t N,
                                           void *workspace, size_t ws_bytes, void *out_f16,
                                           quarot_stream_t stream);

/*
 * quarot_rotate_quant_linear_noalloc -- quarot_rotate_quant_linear for callers
 * that cannot give this library any device memory.  No passage of the pages
 * corresponds to this entry point; it exists for how the library is called,
 * not for the method.
 *
 * Who needs it: code that reaches the kernels only through this C interface
 * and has no device allocator of its own to draw a workspace from (a host
 * program or plug-in whose device memory belongs to another framework), and
 * serving loops whose device memory was budgeted up front and that must not
 * call cudaMalloc / cudaFree on the request path -- those calls can
 * synchronize the device and can fail under memory pressure in the middle of
 * a request.  This call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *
 * Instead of a caller workspace it uses a scratch array compiled into the
 * library: QUAROT_NOALLOC_SCRATCH_BYTES (16 MiB) of device memory that every
 * GPU which loads the library holds until the process exits.  Sizes whose
 * workspace, quarot_rotate_quant_linear_workspace(M, K, group), is larger
 * return QUAROT_ERR_UNSUPPORTED_SHAPE (with per-token scales, 16 MiB holds
 * up to 4092 tokens at K = 8192, or 8176 tokens at K = 4096).
 *
 * The first call on a device looks up the array's device address with that
 * device current (cudaGetSymbolAddress) and keeps it; make that first call
 * before any stream capture.  All calls share the one array, which keeps the
 * last call's contents; nothing in it has to start at zero, because the
 * quantizer writes every byte the GEMM then reads.  Calls that can overlap on
 * the GPU (other streams, or unordered host threads) race on the array: the
 * caller must serialize them.
 *
 * Arguments, layouts, limits and results are those of
 * quarot_rotate_quant_linear without `workspace` and `ws_bytes`; the output is
 * the same.
 */
#define QUAROT_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
quarot_status_t quarot_rotate_quant_linear_noalloc(const void *x_f16, int64_t M, int64_t K,
                                                   const int8_t *signs, int had_block, int group,
                                                   const uint8_t *qw, const void *s_w, int64_t N,
                                                   void *out_f16, quarot_stream_t stream);

/*
 * ---------------------------------------------------------------------------
 * The 8-bit variant of the same recipe: symmetric round-to-nearest codes of
 * one signed byte each, one scale per row [QR-A: 4-bit is the headline, the
 * same rotation makes higher widths lossless; QR-S Key points: round-to-
 * nearest without calibration].  The rotation is the one of
 * quarot_rotate_quant; only the code width changes:
 *
 *   s[m] = max_k |x'[m,k]| / 127 (fp32),  q = rint(x'/s)  (in [-127, 127];
 *   round half to even; a zero scale gives zero codes)
 *
 * INT8 codes are stored one per byte, two's complement, row-major [rows, K].
 * ---------------------------------------------------------------------------
 */

/*
 * quarot_rotate_quant_i8 -- online rotation + 8-bit RTN of activations (or,
 * offline, of weight rows).  x_f16, signs, had_block, M, K: as in
 * quarot_rotate_quant (same limits).  q: [M, K] int8 output.  scales: fp32
 * [M] output.  M == 0 launches nothing and returns QUAROT_OK.
 */
quarot_status_t quarot_rotate_quant_i8(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                       int had_block, int8_t *q, float *scales, quarot_stream_t stream);

/*
 * quarot_int8_linear -- INT8 x INT8 linear layer, int32 accumulation on the
 * tensor cores, fused dequantizing epilogue [QR-S Summary: products in
 * integers]:
 *   out[m,n] = fp16( acc[m,n] * s_a[m] * s_w[n] ),  acc = sum_k qa[m,k] qw[n,k]
 * (exact: |acc| <= 2^14 K < 2^31).
 * qa [M, K] int8, s_a fp32 [M]; qw [N, K] int8 (rows rotated with the same
 * signs and Hadamard [DQ-1]), s_w fp32 [N]; out [M, N] fp16.
 * Limits: M >= 0 (0 launches nothing), N >= 1 with N % 8 == 0,
 *         K % 128 == 0 with 128 <= K <= 65536.
 */
quarot_status_t quarot_int8_linear(const int8_t *qa, const float *s_a, int64_t M, const int8_t *qw,
                                   const float *s_w, int64_t N, int64_t K, void *out_f16,
                                   quarot_stream_t stream);

/*
 * quarot_int8_gemm_s32 -- the same integer product without the epilogue,
 * acc[m,n] written as int32 [M, N]; exact for every input.  Layouts and
 * limits as quarot_int8_linear (no scales).
 */
quarot_status_t quarot_int8_gemm_s32(const int8_t *qa, int64_t M, const int8_t *qw, int64_t N, int64_t K,
                                     int32_t *acc, quarot_stream_t stream);

/*
 * quarot_rotate_quant_linear_i8_workspace -- bytes of device workspace that
 * quarot_rotate_quant_linear_i8 needs: the INT8 activation codes [M, K] and
 * their fp32 scales, each at a 256-byte aligned offset.
 */
size_t quarot_rotate_quant_linear_i8_workspace(int64_t M, int64_t K);

/*
 * quarot_rotate_quant_linear_i8 -- the fused online path of one INT8 linear
 * layer: quarot_rotate_quant_i8 of x into `workspace`, then
 * quarot_int8_linear against the prepared weights, both on `stream` (the
 * GEMM launched as a programmatic dependent of the quantizer).  Arguments as
 * in those calls; workspace: caller-owned device memory of at least
 * quarot_rotate_quant_linear_i8_workspace(M, K) bytes, 256-byte aligned,
 * scratch; ws_bytes: its size.
 */
quarot_status_t quarot_rotate_quant_linear_i8(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                              int had_block, const int8_t *qw, const float *s_w, int64_t N,
                                              void *workspace, size_t ws_bytes, void *out_f16,
                                              quarot_stream_t stream);

/*
 * ---------------------------------------------------------------------------
 * The 6-bit variant [QR-S Key points: round-to-nearest is close to lossless
 * at 6 and 8 bits without calibration; QR-A: higher widths of the same
 * recipe].  The rotation is the one of quarot_rotate_quant; per row
 *
 *   s[m] = max_k |x'[m,k]| / 31 (fp32),  q = rint(x'/s)  (in [-31, 31];
 *   round half to even; a zero scale gives zero codes)
 *
 * Codes are stored one signed byte each, row-major [rows, K], so the INT8
 * linear layer (quarot_int8_linear, quarot_int8_gemm_s32) takes them as they
 * are: the tensor cores have no 6-bit integer kind, and a 6-bit code is an
 * 8-bit code that never leaves [-31, 31] (|acc| <= 961 K, exact).
 * ---------------------------------------------------------------------------
 */

/*
 * quarot_rotate_quant_i6 -- online rotation + 6-bit RTN of activations (or,
 * offline, of weight rows).  Arguments, limits and layouts as
 * quarot_rotate_quant_i8: q int8 [M, K] output (codes in [-31, 31]), scales
 * fp32 [M] output.
 */
quarot_status_t quarot_rotate_quant_i6(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                       int had_block, int8_t *q, float *scales, quarot_stream_t stream);

/*
 * quarot_rotate_quant_linear_i6 -- the fused online path of one 6-bit linear
 * layer: quarot_rotate_quant_i6 of x into `workspace`, then
 * quarot_int8_linear against weights prepared by quarot_rotate_quant_i6.
 * Arguments as quarot_rotate_quant_linear_i8; the workspace size is
 * quarot_rotate_quant_linear_i8_workspace(M, K).
 */
quarot_status_t quarot_rotate_quant_linear_i6(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                              int had_block, const int8_t *qw, const float *s_w, int64_t N,
                                              void *workspace, size_t ws_bytes, void *out_f16,
                                              quarot_stream_t stream);

/*
 * ---------------------------------------------------------------------------
 * Asymmetric INT4 with a clipping ratio [DQ-12: per-token asymmetric
 * quantization of activations, per-channel asymmetric quantization of
 * weights, clipping ratios on the extremes (0.9 for activations, 0.8 for
 * weights in its setup), step (gamma max - beta min) / (2^b - 1)]:
 *
 *   per row of x' (rotated as in quarot_rotate_quant, full Hadamard):
 *     lo = clip * min x', hi = clip * max x', d = (hi - lo) / 15 (fp32),
 *     z = rint(-lo / d) (int32 zero point), u = clamp(rint(x'/d) + z, 0, 15),
 *     reconstruction d * (u - z); a zero step gives zero codes and z = 0.
 *   Codes u are unsigned nibbles packed two per byte (element 2i in bits 0-3).
 *   The quantizer also returns the row's code sum r = sum_k u.
 * The linear layer:
 *   out[m,n] = fp16( d_a[m] d_w[n] (acc - z_w[n] r_a[m] - z_a[m] r_w[n] + K z_a[m] z_w[n]) ),
 *   acc = sum_k u_a[m,k] u_w[n,k]  (int32, exact; the bracket is formed in 64-bit integers).
 * ---------------------------------------------------------------------------
 */

/*
 * quarot_rotate_quant_asym -- rotation + asymmetric 4-bit RTN of activations
 * (per token) or, offline, of weight rows (per output channel).
 * x_f16, signs, M, K: as quarot_rotate_quant; had_block must be 0 and
 * 256 <= K <= 8192 (a power of two).  clip in (0, 1].
 * q_packed [M, K/2] uint8, scales fp32 [M] (the steps d), zeros int32 [M],
 * rowsums int32 [M]: outputs.  Valid while |z| < 2^22 (the clipped range
 * of a row does not sit more than 2^22 steps away from zero).
 */
quarot_status_t quarot_rotate_quant_asym(const void *x_f16, int64_t M, int64_t K, const int8_t *signs,
                                         int had_block, float clip, uint8_t *q_packed, float *scales,
                                         int32_t *zeros, int32_t *rowsums, quarot_stream_t stream);

/*
 * quarot_uint4_gemm_s32 -- acc[m,n] = sum_k u_a[m,k] u_w[n,k] of unsigned
 * nibble codes as int32 [M, N] (exact: acc <= 225 K).  Layouts and limits
 * as quarot_int4_gemm_s32.  For testing the integer path in isolation.
 */
quarot_status_t quarot_uint4_gemm_s32(const uint8_t *qa, int64_t M, const uint8_t *qw, int64_t N, int64_t K,
                                      int32_t *acc, quarot_stream_t stream);

/*
 * quarot_int4_linear_asym -- the asymmetric INT4 linear layer (formula
 * above).  qa [M, K/2], s_a fp32 [M], z_a int32 [M], r_a int32 [M] (from
 * quarot_rotate_quant_asym of the activations); qw [N, K/2], s_w, z_w, r_w
 * [N] (the same call on the weight rows); out [M, N] fp16.
 * Limits: as quarot_int4_linear with group 0.
 */
quarot_status_t quarot_int4_linear_asym(const uint8_t *qa, const float *s_a, const int32_t *z_a,
                                        const int32_t *r_a, int64_t M, const uint8_t *qw, const float *s_w,
                                        const int32_t *z_w, const int32_t *r_w, int64_t N, int64_t K,
                                        void *out_f16, quarot_stream_t stream);

/*
 * quarot_kv_quant -- INT4 KV-cache write [QR-A: the KV cache in 4 bits;
 * DQ-12: fixed Hadamard on the query-key product, per-head quantization].
 *
 *   key row k[b,t,h,:]:   k' = (k * diag(signs[h,:])) * H_D / sqrt(D), then
 *                         s = fp16(max|k'| / 7), q = clamp(rint(k'/s), -8, 7)
 *   value row v[b,t,h,:]: not rotated; same quantizer.
 *
 * k_f16, v_f16  [B, T, Hkv, D] fp16.       signs [Hkv, D] int8 (+-1).
 * kq, vq        [B, T, Hkv, D/2] uint8 packed codes (outputs).
 * ks_f16, vs_f16 [B, T, Hkv] fp16 scales (outputs).
 * Limits: D == 128; B, T >= 0; 1 <= Hkv <= 512.
 */
quarot_status_t quarot_kv_quant(const void *k_f16, const void *v_f16, int64_t B, int64_t T,
                                int64_t Hkv, int64_t D, const int8_t *signs, uint8_t *kq,
                                void *ks_f16, uint8_t *vq, void *vs_f16,
                                quarot_stream_t stream);

/*
 * quarot_kv_decode_scores -- one decode step of query-key scores against the
 * INT4 key cache [QR-A: aspects of the attention mechanism; DQ-12].
 *
 *   q'[b,hq,:] = (q[b,hq,:] * diag(signs[h,:])) * H_D / sqrt(D), fp32 (not
 *                quantized), h = hq / (Hq / Hkv)   (grouped-query attention)
 *   scores[b,hq,t] = sum_d q'[d] * kq[b,t,h,d] * ks[b,t,h]   (fp32; no 1/sqrt(D),
 *                no softmax)
 *
 * The products run on the tensor cores and are exact: the codes as fp16, the
 * fp32 query split into two fp16 parts that carry 22 of its bits; only the
 * fp32 sums over d round.
 *
 * q_f16   [B, Hq, D] fp16.   signs [Hkv, D] int8.
 * kq      [B, T, Hkv, D/2] packed codes, ks_f16 [B, T, Hkv] fp16 (from quarot_kv_quant).
 * scores  [B, Hq, T] fp32 output.
 * Limits: D == 128; Hq / Hkv in {1, 2, 4, 8, 16}; B, Hkv <= 65535; B, T >= 0
 * (B == 0 or T == 0 launches nothing).
 */
quarot_status_t quarot_kv_decode_scores(const void *q_f16, int64_t Hq, const int8_t *signs,
                                        const uint8_t *kq, const void *ks_f16, int64_t B,
                                        int64_t T, int64_t Hkv, int64_t D,
                                        float *scores, quarot_stream_t stream);

/*
 * quarot_kv_decode_attend -- the rest of one decode step of attention over
 * the INT4 value cache [QR-A: the KV cache in 4 bits; DQ-12: the attention
 * output x value product on quantized values, softmax outputs unquantized]:
 *
 *   p[b,hq,t]   = softmax over t of scores[b,hq,t] / sqrt(D)
 *   out[b,hq,d] = sum_t p[b,hq,t] * vs[b,t,h] * vcode[b,t,h,d],  h = hq / (Hq/Hkv)
 *
 * The value rows are not rotated (quarot_kv_quant), so no inverse rotation
 * follows.  scores: fp32 [B, Hq, T] (e.g. from quarot_kv_decode_scores);
 * vq [B, T, Hkv, D/2] packed value codes and vs_f16 [B, T, Hkv] fp16 value
 * scales (from quarot_kv_quant); out: fp32 [B, Hq, D].
 * Limits: D == 128; T >= 1; Hq / Hkv in {1, 2, 4, 8, 16}; B, Hkv <= 65535.
 */
quarot_status_t quarot_kv_decode_attend(const float *scores, int64_t B, int64_t Hq, const uint8_t *vq,
                                        const void *vs_f16, int64_t T, int64_t Hkv, int64_t D, float *out,
                                        quarot_stream_t stream);

/*
 * quarot_kv_decode_attention -- one whole decode step of attention over the
 * INT4 KV cache in one fused kernel [QR-A: the KV cache in 4 bits, the
 * rotation covering aspects of the attention mechanism; DQ-12: a fixed
 * Hadamard on the query-key product, per-head quantization, the attention
 * output x value product on quantized values]:
 *
 *   q'[b,hq,:]  = (q[b,hq,:] * diag(signs[h,:])) * H_D / sqrt(D)   (fp32, h = hq / (Hq/Hkv))
 *   s[b,hq,t]   = sum_d q'[d] * kq[b,t,h,d] * ks[b,t,h]
 *   p[b,hq,t]   = softmax over t of s[b,hq,t] / sqrt(D)
 *   out[b,hq,d] = sum_t p[b,hq,t] * vs[b,t,h] * vq[b,t,h,d]
 *
 * i.e. quarot_kv_decode_attend(quarot_kv_decode_scores(...)) without the
 * scores in memory: the key and value codes are read once.  Both contractions
 * run on the tensor cores with exact operands (codes in fp16; the fp32 query
 * and softmax weights as two fp16 parts each) and fp32 accumulation.
 * q_f16 [B, Hq, D] fp16; signs [Hkv, D] int8; kq, vq [B, T, Hkv, D/2] packed
 * codes and ks_f16, vs_f16 [B, T, Hkv] fp16 scales (from quarot_kv_quant);
 * out [B, Hq, D] fp32.  Limits: D == 128; T >= 1; Hq / Hkv in {1, 2, 4, 8,
 * 16}; B, Hkv <= 65535.  B == 0 launches nothing.
 */
quarot_status_t quarot_kv_decode_attention(const void *q_f16, int64_t Hq, const int8_t *signs,
                                           const uint8_t *kq, const void *ks_f16, const uint8_t *vq,
                                           const void *vs_f16, int64_t B, int64_t T, int64_t Hkv,
                                           int64_t D, float *out, quarot_stream_t stream);

/*
 * quarot_get_device_status -- synchronizes `stream` (the whole current device
 * when stream is NULL), then reports (and clears) the library's device-side
 * error word: QUAROT_ERR_DEVICE_BOUNDS if (bounds-checking build only) a
 * kernel skipped a store outside its output, else QUAROT_ERR_DEVICE_TIMEOUT if
 * any kernel since the last call gave up a bounded wait (every wait on a barrier, a copy or the tensor core
 * is bounded in time; on expiry the kernel records the fact, waits -- again
 * with a limit -- for the copies and tensor-core work it issued, frees its
 * tensor memory and exits), QUAROT_ERR_CUDA if the synchronization itself
 * failed, else QUAROT_OK.  The error word is one per device and process:
 * with a non-NULL stream, kernels still running on other streams may set it
 * after the read.
 */
quarot_status_t quarot_get_device_status(quarot_stream_t stream);

/*
 * quarot_probe_mma_i8 -- measures the denominator of the linear layers'
 * roofline (no passage of the pages corresponds to it: the pages time their
 * kernels on other hardware and give no peak).  On every pair of SMs, one CTA
 * pair issues `steps` groups of four tcgen05.mma.kind::i8 instructions of the
 * shape the INT4 and INT8 GEMMs use (M 256, N 256, K 32 each, int32
 * accumulation in tensor memory), on operands resident in shared memory, and
 * waits for them; nothing is copied or stored.  *pairs receives the number of
 * CTA pairs launched, so one call performs pairs * steps * 4 * 2 * 256 * 256
 * * 32 integer operations; timing the call on `stream` gives the dense INT8
 * tensor rate.  operands: 0 fills both operands with zeros, 1 with
 * pseudo-random bytes (the INT8 GEMMs' codes), 2 with pseudo-random 4-bit
 * codes in the high nibble of each byte (the form in which the INT4 GEMMs
 * hand their codes to the tensor core).  The work per clock is the same for
 * all three; nonzero operands draw the power that real data draws, so that a
 * run of them shows the rate the board's power limit allows.  Limits:
 * 1 <= steps <= 2^22; operands in {0, 1, 2}.
 */
quarot_status_t quarot_probe_mma_i8(int64_t steps, int operands, int64_t *pairs,
                                    quarot_stream_t stream);

/*
 * quarot_test_wait_timeout -- exercises the bounded-wait path of the kernels
 * (no passage of the pages corresponds to it: it tests the library's failure
 * reporting, not the method).  It runs the KV-cache value-row quantizer of
 * quarot_kv_quant (rows of 128 fp16, no rotation, fp16 scale per row) over
 * `rows` rows, but never issues the copy of tile `withheld_tile` (tiles are
 * 128 consecutive rows), and bounds every wait by `wait_limit_ns`.  The CTA
 * that owns the withheld tile gives up its wait after that time, records
 * QUAROT_ERR_DEVICE_TIMEOUT in the device error word, waits (with the same
 * bound) for the copies it did issue and exits; nothing is left in flight and
 * the context stays usable.  The other tiles are quantized as usual; rows of
 * the aborted CTA from the withheld tile on may be left unwritten.
 *
 * v_f16 [rows, 128] fp16; q_packed [rows, 64] uint8 and scales_f16 [rows]
 * fp16 outputs.  Limits: 1 <= rows < 2^31 - 128; 0 <= withheld_tile <
 * ceil(rows / 128); 1e5 <= wait_limit_ns <= 2e9.  Returns the launch status;
 * quarot_get_device_status() then reports the timeout.
 */
quarot_status_t quarot_test_wait_timeout(const void *v_f16, int64_t rows, uint8_t *q_packed, void *scales_f16,
                                         int64_t withheld_tile, uint64_t wait_limit_ns, quarot_stream_t stream);

/*
 * quarot_debug_bounds -- 1 for the bounds-checking build of the library
 * (libquarot_dbg.so, compiled with QUAROT_DEBUG_BOUNDS), 0 for the normal
 * one.  No passage of the pages corresponds to it: it is a test aid.  In the
 * bounds-checking build every kernel checks, before each global store of an
 * output, that the bytes it is about to write lie inside that output as the
 * call's sizes give it; a store that would not is skipped and recorded, and
 * quarot_get_device_status() then returns QUAROT_ERR_DEVICE_BOUNDS (before a
 * timeout, if both happened).  The normal build has no such checks.
 */
int quarot_debug_bounds(void);

/* Static, human-readable name of a status code. */
const char *quarot_status_string(quarot_status_t status);

/* Message of the last QUAROT_ERR_CUDA / argument error on this host thread. */
const char *quarot_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* QUAROT_H */
