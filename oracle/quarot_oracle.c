/*
 * quarot_oracle.c -- plain CPU oracle for the QuaRot online rotation + INT4 path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file.  Only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library: it is a second, independent statement of what the path
 * computes, written for reading, not for speed.
 *
 * Arithmetic: fp64 for every real number, int64 for every integer sum.
 * Parallelism: OpenMP over independent rows only; no blocking, no fusion and
 * no reordering of any sum beyond what each definition below states.
 *
 * What it follows:
 *  - QuaRot: Outlier-free 4-bit inference in rotated LLMs (ISTA research
 *    explorer record, abstract): weights, activations and the KV cache are
 *    quantized to 4 bits and all matrix products run in 4 bits; the rotation
 *    leaves the layer output unchanged (computational invariance).
 *  - QuaRot: Outlier-Free 4-Bit Inference in Rotated LLMs (Elamur Research
 *    summary), "Summary": the model is multiplied by random orthogonal
 *    Hadamard matrices, most folded into the weights, a few applied online;
 *    "Key points": activations are quantized on the fly with round-to-nearest,
 *    and a group-wise variant uses groups of 128.
 *  - Scientists from ETH Zurich, EPFL and Microsoft have presented QuaRot
 *    (onlyaistuff.com article): the rotations are randomized Hadamard
 *    transformations.
 *  - DuQuant: Distributing Outliers via Dual Transformation Makes Stronger
 *    Quantized LLMs (chapterpal), Knowl 1 (Y = XW = (XG)(G^-1 W)), Knowl 2
 *    (block-diagonal rotations of size 2^n; a normalized Hadamard has a
 *    uniform first row), Knowl 12 (block size 128; a fixed Hadamard with
 *    entries +-1/sqrt(2^n) on the attention path, per-head quantization).
 *  - The Elamur Research QuaRot summary, References, item 24: Sloane's
 *    library of Hadamard matrices, for factors whose order is not a power of
 *    two (here built by Paley's first construction, qo_paley, for the full
 *    rotation of K = 11008 = 344 * 32, qo_rotate_kron).
 *  - The rest of a decode attention step (qo_kv_attend): softmax of the
 *    scores scaled by 1/sqrt(D) over the tokens, then the product with the
 *    dequantized INT4 value cache (QuaRot abstract: the KV cache in 4 bits;
 *    DuQuant Knowl 12: softmax outputs are not quantized).
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes): Sylvester order for H_n, normalization 1/sqrt(n), signs applied
 * before the Hadamard (x * diag(s) * H), symmetric scale absmax/7, codes
 * clamp(rint(v/scale), -8, 7) with round-half-to-even, a zero stored scale
 * giving zero codes, group scales stored as fp16 and the stored fp16 value
 * used to quantize, nibble order low = even element.
 *
 * Parity pins: every function here is pinned by a CPU test against something
 * other than itself (textbook Sylvester matrices, scipy's Hadamard, closed
 * forms, numpy's fp16 conversion, brute-force integer loops, invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE binary16 <-> binary64, written from the format's definition.          */
/* ------------------------------------------------------------------------ */

/* Exact value of a binary16 bit pattern. */
double qo_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (exp == 0) {
        v = ldexp((double)man, -24);                 /* subnormal: man * 2^-24 */
    } else if (exp == 31) {
        v = man ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + man), exp - 25);   /* (1 + man/1024) * 2^(exp-15) */
    }
    return sign ? -v : v;
}

/* Nearest binary16 to x, ties to even; overflow to infinity. */
uint16_t qo_f64_to_f16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x))
        return 0x7e00;
    if (a >= 65520.0)                 /* halfway between 65504 and 2^16 rounds up */
        return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {        /* subnormal range: multiples of 2^-24 */
        double q = nearbyint(ldexp(a, 24));          /* default mode: ties to even */
        return sign | (uint16_t)q;    /* q == 1024 is the smallest normal, as bits */
    }
    int e2;
    double f = frexp(a, &e2);         /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;                   /* a = (2f) * 2^e, 2f in [1, 2) */
    double m = nearbyint((2.0 * f - 1.0) * 1024.0);
    if (m == 1024.0) {
        m = 0.0;
        e += 1;
    }
    if (e + 15 >= 31)
        return sign | 0x7c00;
    return sign | (uint16_t)(((e + 15) << 10) | (int)m);
}

void qo_f16_to_f64_array(const uint16_t *h, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = qo_f16_to_f64(h[i]);
}

void qo_f64_to_f16_array(const double *x, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = qo_f64_to_f16(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Hadamard matrices and the transform.                                       */
/* ------------------------------------------------------------------------ */

static int is_pow2(int64_t n) { return n >= 1 && (n & (n - 1)) == 0; }

/*
 * Sylvester construction: H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]].
 * Writes the n x n matrix row-major.  Returns 0, or -1 if n is not a power
 * of two.
 */
int qo_sylvester(int64_t n, int8_t *H)
{
    if (!is_pow2(n))
        return -1;
    H[0] = 1;
    for (int64_t m = 1; m < n; m *= 2) {
        for (int64_t i = 0; i < m; ++i) {
            for (int64_t j = 0; j < m; ++j) {
                int8_t h = H[i * n + j];
                H[i * n + (j + m)] = h;
                H[(i + m) * n + j] = h;
                H[(i + m) * n + (j + m)] = (int8_t)-h;
            }
        }
    }
    return 0;
}

/*
 * Unnormalized fast Walsh-Hadamard transform in place: v <- v * H_n, Sylvester
 * order (H_n is symmetric, so this is also H_n * v).  The textbook butterfly:
 * for each span h = 1, 2, 4, ..., n/2, replace every pair (a, b) that is h
 * apart inside a block of 2h by (a + b, a - b).
 */
int qo_fwht(double *v, int64_t n)
{
    if (!is_pow2(n))
        return -1;
    for (int64_t h = 1; h < n; h *= 2) {
        for (int64_t i = 0; i < n; i += 2 * h) {
            for (int64_t j = i; j < i + h; ++j) {
                double a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
        }
    }
    return 0;
}

/*
 * The online randomized rotation of the activations (QuaRot summary and
 * article: randomized Hadamard; DuQuant Knowl 2 and 12: block-diagonal
 * rotations of block 128).  For each row x of X (fp16 bits, M x K):
 *     x' = (x * diag(s)) * R,
 * where R = H_K / sqrt(K) when had_block == 0 (K a power of two), and
 * R = I_{K/b} (x) (H_b / sqrt(b)) when had_block == b (each b-wide block of
 * the row rotated on its own).  Output fp64, M x K.
 */
int qo_rotate(const uint16_t *x16, int64_t M, int64_t K, const int8_t *signs,
              int64_t had_block, double *out)
{
    int64_t n = had_block == 0 ? K : had_block;
    if (!is_pow2(n) || K % n != 0 || M < 0)
        return -1;
    double inv = 1.0 / sqrt((double)n);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        double *o = out + r * K;
        for (int64_t k = 0; k < K; ++k)
            o[k] = qo_f16_to_f64(x16[r * K + k]) * (double)signs[k];
        for (int64_t b0 = 0; b0 < K; b0 += n) {
            qo_fwht(o + b0, n);
            for (int64_t k = 0; k < n; ++k)
                o[b0 + k] *= inv;
        }
    }
    return 0;
}

/*
 * The same rotation as a dense product with the Sylvester matrix:
 * x'[k] = sum_l x[l] s[l] H[l][k] / sqrt(n), block by block.  O(n^2) per
 * block; used for small n and as a second route in the tests.
 */
int qo_rotate_dense(const uint16_t *x16, int64_t M, int64_t K, const int8_t *signs,
                    int64_t had_block, double *out)
{
    int64_t n = had_block == 0 ? K : had_block;
    if (!is_pow2(n) || K % n != 0 || M < 0 || n > 8192)
        return -1;
    int8_t *H = (int8_t *)malloc((size_t)(n * n));
    if (!H)
        return -2;
    qo_sylvester(n, H);
    double inv = 1.0 / sqrt((double)n);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t b0 = 0; b0 < K; b0 += n) {
            for (int64_t k = 0; k < n; ++k) {
                double acc = 0.0;
                for (int64_t l = 0; l < n; ++l)
                    acc += qo_f16_to_f64(x16[r * K + b0 + l]) * (double)signs[b0 + l] *
                           (double)H[l * n + k];
                out[r * K + b0 + k] = acc * inv;
            }
        }
    }
    free(H);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Symmetric round-to-nearest INT4 quantization (QuaRot key points: RTN).      */
/* ------------------------------------------------------------------------ */

/* q = clamp(rint(v / s), -8, 7); a zero scale gives a zero code. */
static int8_t rtn_code(double v, double s)
{
    if (s == 0.0)
        return 0;
    double q = nearbyint(v / s);      /* ties to even */
    if (q < -8.0)
        q = -8.0;
    if (q > 7.0)
        q = 7.0;
    return (int8_t)q;
}

/*
 * Quantize the rotated values xr (M x K, fp64).
 *  group == 0:   one scale per row, s = max|row| / 7, kept in fp64 (scale64[M]).
 *  group == g>0: one scale per (row, g-wide group), s16 = fp16(max|group| / 7)
 *                stored in scale16[M, K/g]; the codes use the stored fp16 value.
 * Codes are written unpacked, one int8 per element.
 */
int qo_quantize(const double *xr, int64_t M, int64_t K, int64_t group, int8_t *codes,
                double *scale64, uint16_t *scale16)
{
    if (M < 0 || K <= 0 || group < 0 || (group > 0 && K % group != 0))
        return -1;
    int64_t G = group == 0 ? 1 : K / group;
    int64_t w = group == 0 ? K : group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            const double *v = xr + r * K + g * w;
            double amax = 0.0;
            for (int64_t k = 0; k < w; ++k)
                if (fabs(v[k]) > amax)
                    amax = fabs(v[k]);
            double s;
            if (group == 0) {
                s = amax / 7.0;
                scale64[r] = s;
            } else {
                uint16_t h = qo_f64_to_f16(amax / 7.0);
                scale16[r * G + g] = h;
                s = qo_f16_to_f64(h);
            }
            for (int64_t k = 0; k < w; ++k)
                codes[r * K + g * w + k] = rtn_code(v[k], s);
        }
    }
    return 0;
}

/*
 * The RTN step alone with scales supplied by the caller (one per row when
 * group == 0, else one per group): q = clamp(rint(v/s), -8, 7), zero scale ->
 * zero code.  Used to state the expected codes once a scale has been checked.
 */
int qo_quantize_with_scales(const double *xr, int64_t M, int64_t K, int64_t group,
                            const double *scales, int8_t *codes)
{
    if (M < 0 || K <= 0 || group < 0 || (group > 0 && K % group != 0))
        return -1;
    int64_t G = group == 0 ? 1 : K / group;
    int64_t w = group == 0 ? K : group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r)
        for (int64_t g = 0; g < G; ++g)
            for (int64_t k = 0; k < w; ++k)
                codes[r * K + g * w + k] = rtn_code(xr[r * K + g * w + k], scales[r * G + g]);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The same symmetric RTN at other code widths (QuaRot abstract: 4-bit is the */
/* headline, higher widths are the lossless end of the same recipe; QuaRot    */
/* summary, "Key points": round-to-nearest without calibration).              */
/* ------------------------------------------------------------------------ */

/* q = clamp(rint(v / s), -2^(bits-1), 2^(bits-1) - 1); zero scale -> zero. */
static int32_t rtn_code_bits(double v, double s, int bits)
{
    const double qmax = (double)((1 << (bits - 1)) - 1);
    if (s == 0.0)
        return 0;
    double q = nearbyint(v / s);      /* ties to even */
    if (q < -qmax - 1.0)
        q = -qmax - 1.0;
    if (q > qmax)
        q = qmax;
    return (int32_t)q;
}

/*
 * Per-row symmetric RTN at `bits` (2..8) bits: s = max|row| / (2^(bits-1) - 1)
 * kept in fp64 (scale64[M]), codes as above, one int8 per element.
 */
int qo_quantize_bits(const double *xr, int64_t M, int64_t K, int bits, int8_t *codes, double *scale64)
{
    if (M < 0 || K <= 0 || bits < 2 || bits > 8)
        return -1;
    const double qmax = (double)((1 << (bits - 1)) - 1);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        const double *v = xr + r * K;
        double amax = 0.0;
        for (int64_t k = 0; k < K; ++k)
            if (fabs(v[k]) > amax)
                amax = fabs(v[k]);
        const double s = amax / qmax;
        scale64[r] = s;
        for (int64_t k = 0; k < K; ++k)
            codes[r * K + k] = (int8_t)rtn_code_bits(v[k], s, bits);
    }
    return 0;
}

/* The RTN step alone at `bits` bits with one caller-supplied scale per row. */
int qo_quantize_bits_with_scales(const double *xr, int64_t M, int64_t K, int bits, const double *scales,
                                 int8_t *codes)
{
    if (M < 0 || K <= 0 || bits < 2 || bits > 8)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k)
            codes[r * K + k] = (int8_t)rtn_code_bits(xr[r * K + k], scales[r], bits);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Asymmetric RTN with a clipping ratio (DuQuant, Knowl 12: per-token         */
/* asymmetric activations, per-channel asymmetric weights, clipping ratios    */
/* 0.9 / 0.8 on the extremes; the step of its clipped range is                */
/* (gamma max - beta min) / (2^b - 1), here gamma = beta = the ratio).        */
/* ------------------------------------------------------------------------ */

/*
 * Per row: lo = clip * min, hi = clip * max, step d = (hi - lo) / (2^bits - 1),
 * zero point z = rint(-lo / d), codes u = clamp(rint(v / d) + z, 0, 2^bits - 1)
 * (ties to even), so that v is reconstructed as d * (u - z).  A zero step
 * gives zero codes and zero point.  Outputs: codes (one per int8, values
 * 0 .. 2^bits - 1), step (fp64), zero point and the row's code sum (int64).
 */
int qo_quantize_asym(const double *xr, int64_t M, int64_t K, int bits, double clip, int8_t *codes,
                     double *step, int64_t *zero, int64_t *rowsum)
{
    if (M < 0 || K <= 0 || bits < 2 || bits > 8 || !(clip > 0.0) || clip > 1.0)
        return -1;
    const double qmax = (double)((1 << bits) - 1);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        const double *v = xr + r * K;
        double mn = v[0], mx = v[0];
        for (int64_t k = 1; k < K; ++k) {
            if (v[k] < mn)
                mn = v[k];
            if (v[k] > mx)
                mx = v[k];
        }
        const double lo = clip * mn, hi = clip * mx;
        const double d = (hi - lo) / qmax;
        int64_t z = 0, sum = 0;
        if (d > 0.0)
            z = (int64_t)nearbyint(-lo / d);
        for (int64_t k = 0; k < K; ++k) {
            int64_t u = 0;
            if (d > 0.0) {
                double q = nearbyint(v[k] / d) + (double)z;
                if (q < 0.0)
                    q = 0.0;
                if (q > qmax)
                    q = qmax;
                u = (int64_t)q;
            }
            codes[r * K + k] = (int8_t)u;
            sum += u;
        }
        step[r] = d;
        zero[r] = z;
        rowsum[r] = sum;
    }
    return 0;
}

/* The asymmetric RTN step alone under a caller-supplied step and zero point
 * per row: u = clamp(rint(v / d) + z, 0, 2^bits - 1), zero step -> zero code. */
int qo_quantize_asym_with(const double *xr, int64_t M, int64_t K, int bits, const double *step, const int64_t *zero,
                          int8_t *codes)
{
    if (M < 0 || K <= 0 || bits < 2 || bits > 8)
        return -1;
    const double qmax = (double)((1 << bits) - 1);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            double q = 0.0;
            if (step[r] > 0.0) {
                q = nearbyint(xr[r * K + k] / step[r]) + (double)zero[r];
                if (q < 0.0)
                    q = 0.0;
                if (q > qmax)
                    q = qmax;
            }
            codes[r * K + k] = (int8_t)q;
        }
    return 0;
}

/*
 * The dequantized product of asymmetric codes:
 *   y[m, n] = da[m] dw[n] sum_k (ua[m,k] - za[m]) (uw[n,k] - zw[n])
 *           = da[m] dw[n] (acc[m,n] - zw[n] ra[m] - za[m] rw[n] + K za[m] zw[n])
 * with acc = sum_k ua uw (int64) and ra, rw the row code sums; the integer
 * bracket is formed exactly, then scaled in fp64.
 */
int qo_dequant_asym(const int64_t *acc, int64_t M, int64_t N, int64_t K, const double *da, const int64_t *za,
                    const int64_t *ra, const double *dw, const int64_t *zw, const int64_t *rw, double *y64,
                    uint16_t *y16)
{
    if (M < 0 || N < 0 || K <= 0)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            const int64_t b = acc[m * N + n] - zw[n] * ra[m] - za[m] * rw[n] + K * za[m] * zw[n];
            const double y = (double)b * da[m] * dw[n];
            y64[m * N + n] = y;
            if (y16)
                y16[m * N + n] = qo_f64_to_f16(y);
        }
    return 0;
}

/* Nibble packing: byte i = code[2i] in bits 0-3, code[2i+1] in bits 4-7. */
int qo_pack(const int8_t *codes, int64_t n, uint8_t *packed)
{
    if (n % 2 != 0)
        return -1;
    for (int64_t i = 0; i < n / 2; ++i)
        packed[i] = (uint8_t)((codes[2 * i] & 0x0f) | ((codes[2 * i + 1] & 0x0f) << 4));
    return 0;
}

/* Inverse of qo_pack: each nibble read as a 4-bit two's-complement number. */
int qo_unpack(const uint8_t *packed, int64_t n, int8_t *codes)
{
    if (n % 2 != 0)
        return -1;
    for (int64_t i = 0; i < n / 2; ++i) {
        int lo = packed[i] & 0x0f, hi = (packed[i] >> 4) & 0x0f;
        codes[2 * i] = (int8_t)(lo >= 8 ? lo - 16 : lo);
        codes[2 * i + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Integer matrix product and dequantization (QuaRot: all matrix products in  */
/* 4 bits, in integers).                                                      */
/* ------------------------------------------------------------------------ */

/*
 * acc[m, n, g] = sum over k in group g of qa[m, k] * qw[n, k], int64.
 * group == 0 means one group spanning all of K (acc is M x N).
 */
int qo_int_gemm(const int8_t *qa, const int8_t *qw, int64_t M, int64_t N, int64_t K,
                int64_t group, int64_t *acc)
{
    if (M < 0 || N < 0 || K <= 0 || group < 0 || (group > 0 && K % group != 0))
        return -1;
    int64_t G = group == 0 ? 1 : K / group;
    int64_t w = group == 0 ? K : group;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t g = 0; g < G; ++g) {
                int64_t s = 0;
                for (int64_t k = g * w; k < (g + 1) * w; ++k)
                    s += (int64_t)qa[m * K + k] * (int64_t)qw[n * K + k];
                acc[(m * N + n) * G + g] = s;
            }
        }
    }
    return 0;
}

/*
 * Dequantized output.  group == 0: y[m, n] = acc[m, n] * sa[m] * sw[n].
 * group > 0 (G groups): y[m, n] = sum_g acc[m, n, g] * sa[m, g] * sw[n, g].
 * y64 gets the fp64 value, y16 (if not NULL) its nearest fp16.
 */
int qo_dequant_linear(const int64_t *acc, int64_t M, int64_t N, int64_t G, const double *sa,
                      const double *sw, double *y64, uint16_t *y16)
{
    if (M < 0 || N < 0 || G <= 0)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double y = 0.0;
            for (int64_t g = 0; g < G; ++g)
                y += (double)acc[(m * N + n) * G + g] * sa[m * G + g] * sw[n * G + g];
            y64[m * N + n] = y;
            if (y16)
                y16[m * N + n] = qo_f64_to_f16(y);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* INT4 KV cache (QuaRot abstract: the KV cache in 4 bits; DuQuant Knowl 12:  */
/* fixed Hadamard rotation on the query-key product with per-head quantization). */
/* ------------------------------------------------------------------------ */

/*
 * K, V: fp16 [B, T, H, D].  signs: [H, D].  Each key row k[b, t, h, :] becomes
 * (k * diag(signs[h])) * H_D / sqrt(D); keys and values are then quantized
 * with one fp16 scale per (b, t, h) over the D channels.  Values are not
 * rotated.  Codes unpacked, int8 [B, T, H, D]; scales fp16 [B, T, H].
 */
int qo_kv_quant(const uint16_t *k16, const uint16_t *v16, int64_t B, int64_t T, int64_t H,
                int64_t D, const int8_t *signs, int8_t *kcodes, uint16_t *kscale16,
                int8_t *vcodes, uint16_t *vscale16)
{
    if (!is_pow2(D) || B < 0 || T < 0 || H <= 0)
        return -1;
    int64_t rows = B * T;
    int64_t W = H * D;
    double *tmp = (double *)malloc((size_t)(rows * W) * sizeof(double));
    if (!tmp && rows > 0)
        return -2;
    /* keys: the row of H heads is rotated block-wise, block D, with the
       concatenated per-head sign vectors; the scale groups are the heads */
    int rc = qo_rotate(k16, rows, W, signs, D, tmp);
    if (rc == 0)
        rc = qo_quantize(tmp, rows, W, D, kcodes, NULL, kscale16);
    /* values: no rotation */
    if (rc == 0) {
        for (int64_t i = 0; i < rows * W; ++i)
            tmp[i] = qo_f16_to_f64(v16[i]);
        rc = qo_quantize(tmp, rows, W, D, vcodes, NULL, vscale16);
    }
    free(tmp);
    return rc;
}

/*
 * One decode step of query-key scores over the INT4 key cache.
 * q: fp16 [B, Hq, D]; query head hq uses KV head hq / (Hq / H).
 * q' = (q * diag(signs[h])) * H_D / sqrt(D), kept in fp64 (not quantized);
 * scores[b, hq, t] = sum_d q'[d] * kcodes[b, t, h, d] * kscale[b, t, h].
 */
int qo_kv_scores(const uint16_t *q16, int64_t B, int64_t Hq, int64_t H, int64_t D, int64_t T,
                 const int8_t *signs, const int8_t *kcodes, const double *kscale,
                 double *scores)
{
    if (!is_pow2(D) || H <= 0 || Hq % H != 0 || B < 0 || T < 0)
        return -1;
    int64_t grp = Hq / H;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < B * Hq; ++bh) {
        int64_t b = bh / Hq, hq = bh % Hq, h = hq / grp;
        double *qr = (double *)malloc((size_t)D * sizeof(double));
        for (int64_t d = 0; d < D; ++d)
            qr[d] = qo_f16_to_f64(q16[(b * Hq + hq) * D + d]) * (double)signs[h * D + d];
        qo_fwht(qr, D);
        double inv = 1.0 / sqrt((double)D);
        for (int64_t d = 0; d < D; ++d)
            qr[d] *= inv;
        for (int64_t t = 0; t < T; ++t) {
            const int8_t *kc = kcodes + ((b * T + t) * H + h) * D;
            double s = 0.0;
            for (int64_t d = 0; d < D; ++d)
                s += qr[d] * (double)kc[d];
            scores[(b * Hq + hq) * T + t] = s * kscale[(b * T + t) * H + h];
        }
        free(qr);
    }
    return 0;
}

/*
 * The rest of one decode step of attention over the INT4 value cache
 * (QuaRot abstract: the KV cache in 4 bits, the attention path rotated too;
 * DuQuant Knowl 12: the attention output x value product runs on quantized
 * values while the softmax outputs stay unquantized):
 *   p[b,hq,t] = softmax over t of scores[b,hq,t] / sqrt(D),
 *   out[b,hq,d] = sum_t p[b,hq,t] * vscale[b,t,h] * vcode[b,t,h,d],  h = hq / (Hq/H).
 * The value rows were not rotated, so no inverse rotation follows.  The
 * softmax subtracts the row maximum before exponentiating (the same
 * function, evaluated without overflow).
 */
int qo_kv_attend(const double *scores, int64_t B, int64_t Hq, int64_t H, int64_t D, int64_t T,
                 const int8_t *vcodes, const double *vscale, double *out)
{
    if (D <= 0 || H <= 0 || Hq % H != 0 || B < 0 || T <= 0)
        return -1;
    int64_t grp = Hq / H;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < B * Hq; ++bh) {
        int64_t b = bh / Hq, hq = bh % Hq, h = hq / grp;
        const double *sr = scores + (b * Hq + hq) * T;
        const double inv = 1.0 / sqrt((double)D);
        double mx = sr[0] * inv;
        for (int64_t t = 1; t < T; ++t)
            if (sr[t] * inv > mx)
                mx = sr[t] * inv;
        double z = 0.0;
        for (int64_t t = 0; t < T; ++t)
            z += exp(sr[t] * inv - mx);
        double *o = out + (b * Hq + hq) * D;
        for (int64_t d = 0; d < D; ++d)
            o[d] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            const double w = exp(sr[t] * inv - mx) / z * vscale[(b * T + t) * H + h];
            const int8_t *vc = vcodes + ((b * T + t) * H + h) * D;
            for (int64_t d = 0; d < D; ++d)
                o[d] += w * (double)vc[d];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Full rotation for sizes that are not a power of two: K = m * n with n a    */
/* power of two and m = q + 1 the order of a Paley Hadamard matrix.           */
/* (QuaRot summary, Elamur Research: the references name Sloane's library of  */
/* Hadamard matrices as the source of the non-power-of-two factors.  That     */
/* library is not available here; Paley's first construction gives a         */
/* Hadamard matrix of every order q + 1 with q a prime power, q = 3 mod 4 --  */
/* for K = 11008 = 344 * 32, q = 343 = 7^3.  Any Hadamard factor gives an     */
/* orthogonal rotation with entries +-1/sqrt(K); this one is the reading.)    */
/* ------------------------------------------------------------------------ */

/* GF(p^e), e <= 3: element c0 + c1 x + c2 x^2 (c_i in Z_p) has index
 * c0 + c1 p + c2 p^2.  The modulus is the first monic f(x) = x^e + f[e-1]
 * x^(e-1) + ... + f[0] (in the order of the index of (f[0], .., f[e-1]))
 * with no root in Z_p; for e <= 3 that is irreducibility. */
typedef struct {
    int p, e, q;
    int f[3];
} qo_gf;

static int gf_digits(const qo_gf *F, int a, int *c)
{
    for (int i = 0; i < F->e; ++i) {
        c[i] = a % F->p;
        a /= F->p;
    }
    return 0;
}

static int gf_index(const qo_gf *F, const int *c)
{
    int a = 0;
    for (int i = F->e - 1; i >= 0; --i)
        a = a * F->p + c[i];
    return a;
}

static int gf_sub(const qo_gf *F, int a, int b)
{
    int ca[3], cb[3], cd[3];
    gf_digits(F, a, ca);
    gf_digits(F, b, cb);
    for (int i = 0; i < F->e; ++i)
        cd[i] = ((ca[i] - cb[i]) % F->p + F->p) % F->p;
    return gf_index(F, cd);
}

/* Product of polynomials, then x^k (k >= e) replaced by x^(k-e) * (-f(x) + x^e). */
static int gf_mul(const qo_gf *F, int a, int b)
{
    int ca[3], cb[3];
    long prod[5] = {0, 0, 0, 0, 0};
    gf_digits(F, a, ca);
    gf_digits(F, b, cb);
    for (int i = 0; i < F->e; ++i)
        for (int j = 0; j < F->e; ++j)
            prod[i + j] += (long)ca[i] * cb[j];
    for (int k = 2 * F->e - 2; k >= F->e; --k) {
        long t = prod[k] % F->p;
        prod[k] = 0;
        for (int i = 0; i < F->e; ++i)
            prod[k - F->e + i] -= t * F->f[i];
    }
    int c[3];
    for (int i = 0; i < F->e; ++i)
        c[i] = (int)(((prod[i] % F->p) + F->p) % F->p);
    return gf_index(F, c);
}

/* Quadratic character: 0 at 0, +1 on nonzero squares, -1 otherwise, as
 * a^((q-1)/2) (Euler's criterion; the power is 1 or -1 in the field). */
static int gf_chi(const qo_gf *F, int a)
{
    if (a == 0)
        return 0;
    int r = 1, base = a, k = (F->q - 1) / 2;
    while (k > 0) {
        if (k & 1)
            r = gf_mul(F, r, base);
        base = gf_mul(F, base, base);
        k >>= 1;
    }
    return r == 1 ? 1 : -1;
}

static int is_prime(int p)
{
    if (p < 2)
        return 0;
    for (int d = 2; d * d <= p; ++d)
        if (p % d == 0)
            return 0;
    return 1;
}

static int gf_init(qo_gf *F, int p, int e)
{
    if (!is_prime(p) || e < 1 || e > 3)
        return -1;
    F->p = p;
    F->e = e;
    F->q = 1;
    for (int i = 0; i < e; ++i)
        F->q *= p;
    F->f[0] = F->f[1] = F->f[2] = 0;
    if (e == 1)
        return 0;
    int nf = 1;
    for (int i = 0; i < e; ++i)
        nf *= p;
    for (int idx = 0; idx < nf; ++idx) {
        int t = idx;
        for (int i = 0; i < e; ++i) {
            F->f[i] = t % p;
            t /= p;
        }
        int has_root = 0;
        for (int x = 0; x < p && !has_root; ++x) {
            long v = 1;                       /* x^e */
            for (int i = 0; i < e; ++i)
                v = v * x % p;
            long xp = 1;
            for (int i = 0; i < e; ++i) {
                v += (long)F->f[i] * xp;
                xp = xp * x % p;
            }
            has_root = (v % p) == 0;
        }
        if (!has_root)
            return 0;
    }
    return -1;
}

/*
 * Paley's first construction, q = p^e = 3 mod 4, order n = q + 1:
 *   Q[i][j] = chi(a_i - a_j)  over the field elements a_0 .. a_{q-1} (index order),
 *   S = [[0, 1^T], [-1, Q]],  H = I + S.
 * chi(-1) = -1 when q = 3 mod 4, so Q and S are skew-symmetric, Q Q^T = q I - J
 * and Q J = 0, hence S S^T = q I and H H^T = (q + 1) I.
 * Writes H row-major (n x n, +-1).  Returns 0, or -1 for an unsupported (p, e).
 */
int qo_paley(int p, int e, int8_t *H)
{
    qo_gf F;
    if (gf_init(&F, p, e) != 0 || F.q % 4 != 3)
        return -1;
    const int n = F.q + 1;
    int8_t *chi = (int8_t *)malloc((size_t)F.q);
    if (!chi)
        return -2;
    for (int a = 0; a < F.q; ++a)
        chi[a] = (int8_t)gf_chi(&F, a);
    H[0] = 1;
    for (int j = 1; j < n; ++j) {
        H[j] = 1;
        H[(int64_t)j * n] = -1;
    }
    for (int i = 1; i < n; ++i)
        for (int j = 1; j < n; ++j)
            H[(int64_t)i * n + j] = i == j ? 1 : chi[gf_sub(&F, i - 1, j - 1)];
    free(chi);
    return 0;
}

/*
 * The full rotation for K = m * n, m = p^e + 1 (Paley factor), n = K / m a
 * power of two (Sylvester factor):
 *     x' = (x * diag(s)) * (H_m (x) H_n) / sqrt(K),
 * with element index i = a * n + b and (A (x) B)[(a,b)][(a',b')] = A[a][a'] B[b][b'].
 * The Kronecker product is applied through its two factors: with X the
 * m x n matrix of x * s, X' = H_m^T X H_n / sqrt(K), both products written out.
 */
int qo_rotate_kron(const uint16_t *x16, int64_t M, int64_t K, const int8_t *signs, int p, int e,
                   double *out)
{
    if (M < 0 || p < 2 || e < 1 || e > 3)
        return -1;
    int64_t q = 1;
    for (int i = 0; i < e; ++i)
        q *= p;
    const int64_t m = q + 1;
    if (K % m != 0 || !is_pow2(K / m))
        return -1;
    const int64_t n = K / m;
    int8_t *Hm = (int8_t *)malloc((size_t)(m * m));
    int8_t *Hn = (int8_t *)malloc((size_t)(n * n));
    if (!Hm || !Hn) {
        free(Hm);
        free(Hn);
        return -2;
    }
    if (qo_paley(p, e, Hm) != 0 || qo_sylvester(n, Hn) != 0) {
        free(Hm);
        free(Hn);
        return -1;
    }
    const double inv = 1.0 / sqrt((double)K);
    int err = 0;
#pragma omp parallel for schedule(dynamic)
    for (int64_t r = 0; r < M; ++r) {
        double *X = (double *)malloc(sizeof(double) * (size_t)K);
        double *T = (double *)malloc(sizeof(double) * (size_t)K);
        if (!X || !T) {
            free(X);
            free(T);
#pragma omp atomic write
            err = -2;
            continue;
        }
        for (int64_t i = 0; i < K; ++i)
            X[i] = qo_f16_to_f64(x16[r * K + i]) * (double)signs[i];
        /* T = H_m^T X: T[a'][b] = sum_a H_m[a][a'] X[a][b] */
        for (int64_t a2 = 0; a2 < m; ++a2)
            for (int64_t b = 0; b < n; ++b) {
                double acc = 0.0;
                for (int64_t a = 0; a < m; ++a)
                    acc += (double)Hm[a * m + a2] * X[a * n + b];
                T[a2 * n + b] = acc;
            }
        /* X' = T H_n / sqrt(K): X'[a'][b'] = sum_b T[a'][b] H_n[b][b'] */
        for (int64_t a2 = 0; a2 < m; ++a2)
            for (int64_t b2 = 0; b2 < n; ++b2) {
                double acc = 0.0;
                for (int64_t b = 0; b < n; ++b)
                    acc += T[a2 * n + b] * (double)Hn[b * n + b2];
                out[r * K + a2 * n + b2] = acc * inv;
            }
        free(X);
        free(T);
    }
    free(Hm);
    free(Hn);
    return err;
}

int qo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
