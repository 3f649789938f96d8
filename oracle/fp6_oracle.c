/*
 * fp6_oracle.c -- plain, slow CPU reference for the FP6 (e3m2) weight-only
 * linear layer.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg are the only callers.  The CUDA library never
 * links, includes or calls this file, and this file shares no code, header or
 * table with it.
 *
 * Sources (web pages on the method):
 *   - "FP6-LLM: Efficiently Serving Large Language Models Through FP6-Centric
 *     Algorithm-System Co-Design", abstract: weights quantized to 6-bit floats,
 *     activations stay FP16 (W6A16).
 *   - duicuo.cn news article on TC-FPx, section "kernel solution redesign":
 *     dequantization turns FP6 into FP16 before the tensor-core product; weights
 *     are pre-packed offline and each 6-bit weight is split into a 2-bit and a
 *     4-bit piece stored in aligned 32-bit words.
 * The pages fix neither the bit format nor the scale; the format used here is
 * e3m2 with exponent bias 3, no inf/NaN, maximum magnitude 28, and one FP16
 * scale per output row (the layer's stated specification).
 *
 * Every floating-point step is done in IEEE binary64 unless stated.
 *
 * Parity status of each function (what pins it, all in tests/):
 *   decode table        pinned: closed form over all 64 codes + golden file
 *   f16 rounding        pinned: numpy float16 conversion (library routine)
 *   quantize            pinned: exact brute-force argmin, round trip, error
 *                       bound, CUDA's own fp6 conversion routine
 *   prepack / unpack    pinned: a numpy reading of the packed words (byte
 *                       containers plus gathered top bits) gives the
 *                       closed-form fp16 pattern; one-hot probe; round trip
 *   dequant             pinned: closed form of decode*scale rounded by numpy
 *   linear              pinned: exact rational dot products (tiny shapes),
 *                       one-hot and constant-code special cases
 *   fpx_* (FP6 e2m3, FP4 e2m1, FP5 e2m2)
 *                       pinned: closed-form tables over every code, brute-force
 *                       rounding in exact rationals and CUDA's own host
 *                       conversions (e2m3, e2m1; e2m2 through its values being
 *                       e2m3 values), round trips, independent readers of the
 *                       FP4 and FP5 layouts, one-hot probes, exact rational dot
 *                       products
 *   s24_* (2:4 sparse INT4)
 *                       pinned: properties that fix the kept pair uniquely,
 *                       brute-force rounding and exact ties, representable
 *                       round trips, an independent layout reader, one-hot
 *                       probes, dense dequant, exact rational dot products
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>

#define ORC_OK 0
#define ORC_ERR_INVALID_ARG 1
#define ORC_ERR_UNSUPPORTED_SHAPE 2
#define ORC_ERR_NONFINITE 4
#define ORC_ERR_SCALE_RANGE 5

/* ------------------------------------------------------------------------ */
/* FP16 <-> binary64                                                         */
/* ------------------------------------------------------------------------ */

/* Value of an IEEE binary16 bit pattern, exactly. */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);               /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25);   /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round a binary64 value to the nearest binary16, ties to even.
 * Magnitudes at or above 65520 (the midpoint past 65504) become infinity. */
uint16_t oracle_f64_to_f16_rne(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (isnan(v)) return 0x7E00u;
    if (isinf(a)) return sign | 0x7C00u;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: count in units of 2^-24 (exact scaling) */
        double q = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)q;   /* q == 1024 is the smallest normal */
    }
    int ex;
    frexp(a, &ex);          /* a = f * 2^ex with f in [0.5, 1) */
    int e = ex - 1;         /* a in [2^e, 2^(e+1)) */
    double q = nearbyint(ldexp(a, 10 - e));      /* in [1024, 2048] */
    int biased = e + 15;
    if (biased >= 31) return sign | 0x7C00u;
    uint32_t bits = ((uint32_t)biased << 10) + ((uint32_t)q - 1024u);
    if (bits >= 0x7C00u) return sign | 0x7C00u; /* rounded past 65504 */
    return sign | (uint16_t)bits;
}

/* ------------------------------------------------------------------------ */
/* FP6 e3m2 decode (table-driven)                                            */
/* ------------------------------------------------------------------------ */

/* Code bits, low 6 bits of a byte: b5 = sign, b4..b2 = exponent e, b1..b0 =
 * mantissa m.  e > 0: (-1)^s * 2^(e-3) * (1 + m/4);  e == 0: (-1)^s * 2^-2 * m/4. */
static double g_decode[64];
static int g_decode_ready = 0;

static void build_decode_table(void)
{
    for (int c = 0; c < 64; ++c) {
        int s = (c >> 5) & 1, e = (c >> 2) & 7, m = c & 3;
        double mag = (e > 0) ? ldexp(1.0 + m / 4.0, e - 3) : ldexp(m / 4.0, -2);
        g_decode[c] = s ? -mag : mag;
    }
    g_decode_ready = 1;
}

static inline double decode(uint8_t c)
{
    return g_decode[c & 0x3F];
}

void oracle_decode_table(double *out64)
{
    if (!g_decode_ready) build_decode_table();
    for (int c = 0; c < 64; ++c) out64[c] = g_decode[c];
}

/* Round v to the nearest e3m2 value, ties to the even mantissa, saturating to
 * +-28 (there is no infinity code).  The sign bit of v is kept, so negative
 * values that round to zero give the code 0x20.  Steps: find the binade of
 * |v| (or the subnormal range), scale |v| to units of that binade's spacing,
 * round to an integer with ties to even, and rebuild the code; a carry out of
 * the mantissa lands on the next binade's first code. */
uint8_t oracle_round_e3m2(double v)
{
    uint8_t sign = signbit(v) ? 0x20u : 0u;
    double a = fabs(v);
    int code;
    if (a < 0.25) {
        /* subnormal spacing 2^-4; the quotient 4 is the code of 0.25 */
        code = (int)nearbyint(ldexp(a, 4));
    } else {
        int ex;
        frexp(a, &ex);
        int e = ex - 1;                       /* a in [2^e, 2^(e+1)) */
        if (e > 4) {
            code = 32;                        /* beyond the top binade */
        } else {
            double q = nearbyint(ldexp(a, 2 - e));   /* in [4, 8] */
            code = ((e + 3) << 2) + ((int)q - 4);
        }
    }
    if (code > 31) code = 31;                 /* saturate at 28 */
    return sign | (uint8_t)code;
}

/* ------------------------------------------------------------------------ */
/* Quantize: one fp16 scale per output row, then RNE e3m2 codes              */
/* ------------------------------------------------------------------------ */

/* Per row n:  amax = max_k |W[n,k]|;  s = fp16_rne(fp32(amax / 28));
 * code[n,k] = round_e3m2(W[n,k] / s)  (binary64 division, correctly rounded).
 * A row of zeros gets s = 0 and codes 0.  Any non-finite weight is an error;
 * a scale that overflows or underflows fp16 is an error. */
int oracle_quantize(const float *W, int64_t N, int64_t K, uint8_t *codes, uint16_t *scales)
{
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (!g_decode_ready) build_decode_table();
    for (int64_t n = 0; n < N; ++n) {
        const float *row = W + n * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (!isfinite(row[k])) return ORC_ERR_NONFINITE;
            float a = fabsf(row[k]);
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            scales[n] = 0;
            memset(codes + n * K, 0, (size_t)K);
            continue;
        }
        volatile float s32 = amax / 28.0f;                 /* IEEE fp32 division */
        uint16_t s16 = oracle_f64_to_f16_rne((double)s32);
        if ((s16 & 0x7FFFu) >= 0x7C00u || (s16 & 0x7FFFu) == 0) return ORC_ERR_SCALE_RANGE;
        scales[n] = s16;
        double s = oracle_f16_to_f64(s16);
        for (int64_t k = 0; k < K; ++k) {
            double v = (double)row[k] / s;
            codes[n * K + k] = oracle_round_e3m2(v);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Prepack / unpack: bit split into 32-bit-aligned fragment words            */
/* ------------------------------------------------------------------------ */

/* Packed layout (version 2).  The pages cut each 6-bit weight into pieces held
 * in aligned 32-bit words so that registers rebuild many weights per
 * operation; the cut and the order are left open.  This layout is cut for a
 * converter that turns two bytes, each holding one code in its low six bits,
 * into two fp16 values and ignores each byte's top two bits: twelve of every
 * sixteen codes stay whole in the low six bits of a byte, and the other four
 * are cut into three 2-bit pieces stored in those bytes' top two bits.
 *
 * W is cut into tiles of 128 rows x 64 columns, stored tile after tile with
 * the column-tile index fastest:
 *     tile (nt, kt) at byte (nt * (K/64) + kt) * 6144.
 * Inside a tile, row r (0..127) owns twelve 32-bit words F_w, w = 0..11,
 *     F_w at byte (w/4)*2048 + r*16 + (w%4)*4.
 * Column kk (0..63) of the tile belongs to group g = kk/16 (words F_{3g},
 * F_{3g+1}, F_{3g+2}), position i = kk%16 in the group:
 *     i < 12: the whole code in bits 8b..8b+5 of F_{3g + i/4}, b = i%4;
 *     i >= 12: b = i - 12; code bits 2j and 2j+1 (j = 0, 1, 2) in bits 8b+6
 *              and 8b+7 of F_{3g + j}.
 * Byte order is little-endian (bit t of a word is bit t%8 of byte t/8). */
static inline int64_t tile_base(int64_t n, int64_t k, int64_t K)
{
    return ((n / 128) * (K / 64) + (k / 64)) * 6144;
}

static inline int64_t word_byte(int64_t base, int r, int w)
{
    return base + (w / 4) * 2048 + r * 16 + (w % 4) * 4;
}

static inline void put_bit(uint8_t *buf, int64_t wbyte, int bit, int value)
{
    if (value) buf[wbyte + bit / 8] |= (uint8_t)(1u << (bit % 8));
}

static inline int get_bit(const uint8_t *buf, int64_t wbyte, int bit)
{
    return (buf[wbyte + bit / 8] >> (bit % 8)) & 1;
}

/* Where bit t (0..5) of the code at tile row r, tile column kk lives:
 * the word's byte offset and the bit within that word. */
static inline void code_bit_place(int64_t base, int r, int kk, int t, int64_t *wbyte, int *bit)
{
    int g = kk / 16, i = kk % 16;
    if (i < 12) {
        *wbyte = word_byte(base, r, 3 * g + i / 4);
        *bit = 8 * (i % 4) + t;
    } else {
        *wbyte = word_byte(base, r, 3 * g + t / 2);
        *bit = 8 * (i - 12) + 6 + t % 2;
    }
}

int oracle_prepack(const uint8_t *codes, int64_t N, int64_t K, uint8_t *packed)
{
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    memset(packed, 0, (size_t)(N * K / 4 * 3));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t c = codes[n * K + k] & 0x3F;
            int64_t base = tile_base(n, k, K);
            for (int t = 0; t < 6; ++t) {
                int64_t wb;
                int bit;
                code_bit_place(base, (int)(n % 128), (int)(k % 64), t, &wb, &bit);
                put_bit(packed, wb, bit, (c >> t) & 1);
            }
        }
    }
    return ORC_OK;
}

int oracle_unpack(const uint8_t *packed, int64_t N, int64_t K, uint8_t *codes)
{
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t base = tile_base(n, k, K);
            uint8_t c = 0;
            for (int t = 0; t < 6; ++t) {
                int64_t wb;
                int bit;
                code_bit_place(base, (int)(n % 128), (int)(k % 64), t, &wb, &bit);
                c |= (uint8_t)(get_bit(packed, wb, bit) << t);
            }
            codes[n * K + k] = c;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Dequant: W16[n,k] = fp16(decode(c)) or fp16_rne(decode(c) * s[n])          */
/* ------------------------------------------------------------------------ */

int oracle_dequant(const uint8_t *packed, const uint16_t *scales, int64_t N, int64_t K, uint16_t *W16)
{
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    if (!g_decode_ready) build_decode_table();
    uint8_t *codes = (uint8_t *)malloc((size_t)(N * K) + 1);
    if (!codes) return ORC_ERR_INVALID_ARG;
    oracle_unpack(packed, N, K, codes);
    for (int64_t n = 0; n < N; ++n) {
        double s = scales ? oracle_f16_to_f64(scales[n]) : 1.0;
        for (int64_t k = 0; k < K; ++k)
            W16[n * K + k] = oracle_f64_to_f16_rne(decode(codes[n * K + k]) * s);
    }
    free(codes);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Linear: y[m,n] = fp16_rne( sum_k x[m,k] * (s[n] * decode(C[n,k])) )        */
/* ------------------------------------------------------------------------ */

/* The plain definition of the layer: weights reconstructed as s[n]*decode,
 * multiplied with the fp16 activations; each product is exact in binary64
 * (at most 25 significant bits) and the sum runs over k in ascending order.
 * One rounding to fp16 at the end. */
typedef struct {
    const uint16_t *x; const uint8_t *codes; const uint16_t *scales;
    int64_t M, N, K, n0, n1; uint16_t *y;
} linear_job;

static void *linear_rows(void *arg)
{
    linear_job *jb = (linear_job *)arg;
    double *xr = (double *)malloc(sizeof(double) * (size_t)(jb->K > 0 ? jb->K : 1));
    for (int64_t m = 0; m < jb->M; ++m) {
        for (int64_t k = 0; k < jb->K; ++k) xr[k] = oracle_f16_to_f64(jb->x[m * jb->K + k]);
        for (int64_t n = jb->n0; n < jb->n1; ++n) {
            double s = oracle_f16_to_f64(jb->scales[n]);
            const uint8_t *c = jb->codes + n * jb->K;
            double acc = 0.0;
            for (int64_t k = 0; k < jb->K; ++k) acc += xr[k] * (s * decode(c[k]));
            jb->y[m * jb->N + n] = oracle_f64_to_f16_rne(acc);
        }
    }
    free(xr);
    return NULL;
}

int oracle_linear(const uint16_t *x, const uint8_t *codes, const uint16_t *scales,
                  int64_t M, int64_t N, int64_t K, uint16_t *y, int nthreads)
{
    if (M < 0 || N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (!g_decode_ready) build_decode_table();
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > N) nthreads = (int)(N > 0 ? N : 1);
    pthread_t th[256];
    linear_job jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = (linear_job){x, codes, scales, M, N, K,
                               N * t / nthreads, N * (t + 1) / nthreads, y};
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, linear_rows, &jobs[t]);
    linear_rows(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    return ORC_OK;
}

/* ======================================================================== */
/* Other FPx formats (the pages: one design for floats of several widths)    */
/* ======================================================================== */
/*
 * The FP6-LLM abstract and the TC-FPx article present the kernel design as
 * covering float weights of several bit widths ("FPx"), and name none of
 * their bit formats.  Two more formats are taken here, each with one fp16
 * scale per output row like e3m2 (same readings as for e3m2):
 *   fmt 1, FP6 e2m3: s = bit 5, e = bits 4..3 (bias 1), m = bits 2..0;
 *                    e > 0: (-1)^s 2^(e-1) (1 + m/8), e = 0: (-1)^s m/8;
 *                    largest magnitude 7.5.
 *   fmt 2, FP4 e2m1: s = bit 3, e = bits 2..1 (bias 1), m = bit 0;
 *                    e > 0: (-1)^s 2^(e-1) (1 + m/2), e = 0: (-1)^s m/2;
 *                    largest magnitude 6.
 *   fmt 3, FP5 e2m2: s = bit 4, e = bits 3..2 (bias 1), m = bits 1..0;
 *                    e > 0: (-1)^s 2^(e-1) (1 + m/4), e = 0: (-1)^s m/4;
 *                    largest magnitude 7.
 * fmt 0 is e3m2 (the functions above).  No format has inf or NaN codes.
 */

typedef struct { int ebits, mbits, bias; double maxmag; float maxf; } fpx_fmt;

static int fpx_get(int fmt, fpx_fmt *f)
{
    switch (fmt) {
        case 0: *f = (fpx_fmt){3, 2, 3, 28.0, 28.0f}; return 1;
        case 1: *f = (fpx_fmt){2, 3, 1, 7.5, 7.5f}; return 1;
        case 2: *f = (fpx_fmt){2, 1, 1, 6.0, 6.0f}; return 1;
        case 3: *f = (fpx_fmt){2, 2, 1, 7.0, 7.0f}; return 1;
        default: return 0;
    }
}

/* Number of codes of the format (2^(1 + e + m)), 0 for an unknown format. */
int oracle_fpx_codes(int fmt)
{
    fpx_fmt f;
    if (!fpx_get(fmt, &f)) return 0;
    return 1 << (1 + f.ebits + f.mbits);
}

/* Value of code c, from the format's definition. */
static double fpx_decode_one(const fpx_fmt *f, int c)
{
    int mb = f->mbits, eb = f->ebits;
    int s = (c >> (eb + mb)) & 1;
    int e = (c >> mb) & ((1 << eb) - 1);
    int m = c & ((1 << mb) - 1);
    double frac = (double)m / (double)(1 << mb);
    double mag = (e > 0) ? ldexp(1.0 + frac, e - f->bias) : ldexp(frac, 1 - f->bias);
    return s ? -mag : mag;
}

int oracle_fpx_decode_table(int fmt, double *out)
{
    fpx_fmt f;
    if (!fpx_get(fmt, &f)) return ORC_ERR_INVALID_ARG;
    int n = oracle_fpx_codes(fmt);
    for (int c = 0; c < n; ++c) out[c] = fpx_decode_one(&f, c);
    return ORC_OK;
}

/* Round v to the nearest value of the format, ties to the even mantissa,
 * saturating at the largest magnitude; the sign of v is kept.  The same steps
 * as oracle_round_e3m2: subnormal range in units of its spacing, otherwise
 * the binade of |v| in units of that binade's spacing, round to an integer
 * with ties to even, rebuild the code (a mantissa carry lands on the next
 * binade's first code). */
int oracle_fpx_round(int fmt, double v)
{
    fpx_fmt f;
    if (!fpx_get(fmt, &f)) return -1;
    int mb = f.mbits, eb = f.ebits;
    int sign = signbit(v) ? (1 << (eb + mb)) : 0;
    int maxcode = (1 << (eb + mb)) - 1;
    double a = fabs(v);
    int code;
    if (a < ldexp(1.0, 1 - f.bias)) {
        code = (int)nearbyint(ldexp(a, f.bias - 1 + mb));   /* subnormal spacing 2^(1-bias-m) */
    } else {
        int ex;
        frexp(a, &ex);
        int e = ex - 1;                                      /* a in [2^e, 2^(e+1)) */
        int emax = (1 << eb) - 1 - f.bias;
        if (e > emax) {
            code = maxcode + 1;
        } else {
            double q = nearbyint(ldexp(a, mb - e));          /* in [2^m, 2^(m+1)] */
            code = ((e + f.bias) << mb) + ((int)q - (1 << mb));
        }
    }
    if (code > maxcode) code = maxcode;
    return sign | code;
}

/* Per row: s = fp16_rne(fp32(amax / maxmag)), code = round(w / s). */
int oracle_fpx_quantize(int fmt, const float *W, int64_t N, int64_t K, uint8_t *codes, uint16_t *scales)
{
    fpx_fmt f;
    if (!fpx_get(fmt, &f)) return ORC_ERR_INVALID_ARG;
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    for (int64_t n = 0; n < N; ++n) {
        const float *row = W + n * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (!isfinite(row[k])) return ORC_ERR_NONFINITE;
            float a = fabsf(row[k]);
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            scales[n] = 0;
            memset(codes + n * K, 0, (size_t)K);
            continue;
        }
        volatile float s32 = amax / f.maxf;                  /* IEEE fp32 division */
        uint16_t s16 = oracle_f64_to_f16_rne((double)s32);
        if ((s16 & 0x7FFFu) >= 0x7C00u || (s16 & 0x7FFFu) == 0) return ORC_ERR_SCALE_RANGE;
        scales[n] = s16;
        double s = oracle_f16_to_f64(s16);
        for (int64_t k = 0; k < K; ++k) codes[n * K + k] = (uint8_t)oracle_fpx_round(fmt, (double)row[k] / s);
    }
    return ORC_OK;
}

/* Packed size in bytes: 3/4 byte per weight for the 6-bit formats, 1/2 for
 * FP4, 5/8 for FP5. */
int64_t oracle_fpx_packed_bytes(int fmt, int64_t N, int64_t K)
{
    if (fmt == 0 || fmt == 1) return N * K / 4 * 3;
    if (fmt == 2) return N * K / 2;
    if (fmt == 3) return N * K / 8 * 5;
    return -1;
}

/* FP5 packed layout (the "4+1" cut of a 5-bit weight: a 4-bit piece and a
 * 1-bit piece, each kind in its own aligned 32-bit words): tiles of 128 rows x
 * 64 columns, 5120 bytes each, stored like the other tiles.  Row r of a tile
 * owns eight words P_w of 4-bit pieces at byte (w/4)*2048 + r*16 + (w%4)*4 and
 * two words Q_q of 1-bit pieces at byte 4096 + r*8 + q*4.  Column kk is
 * position i = kk%32 of half q = kk/32; with v = i/8, h = (i%8)/4, b = i%4:
 *   the code's top four bits (code >> 1) sit at bits 8b+4h .. 8b+4h+3 of
 *   P_{4q+v}, and its lowest bit (code & 1) at bit 8b+2v+h of Q_q.
 * (So each byte of a P word holds the pieces of codes b and b+4 of its group of
 * eight, and the eight bits that complete one P word's codes sit at
 * positions 8b+2v and 8b+2v+1 of Q.) */
static inline void fp5_positions(int64_t n, int64_t k, int64_t K, int64_t *pbyte, int *pshift,
                                 int64_t *qbyte, int *qshift)
{
    int64_t base = ((n / 128) * (K / 64) + (k / 64)) * 5120;
    int r = (int)(n % 128), kk = (int)(k % 64);
    int q = kk / 32, i = kk % 32, v = i / 8, h = (i % 8) / 4, b = i % 4;
    int w = 4 * q + v;
    int pbit = 8 * b + 4 * h;                                /* bit within P_w */
    int qbit = 8 * b + 2 * v + h;                            /* bit within Q_q */
    *pbyte = base + (w / 4) * 2048 + r * 16 + (w % 4) * 4 + pbit / 8;
    *pshift = pbit % 8;
    *qbyte = base + 4096 + r * 8 + q * 4 + qbit / 8;
    *qshift = qbit % 8;
}

/* FP4 packed layout: tiles of 128 rows x 64 columns, 4096 bytes each, stored
 * like the 6-bit tiles (column-tile index fastest).  Row r of a tile owns
 * eight 32-bit words F_w at byte (w/4)*2048 + r*16 + (w%4)*4; column kk is in
 * word kk/8, byte (kk%8)/2, low nibble for even kk and high nibble for odd kk
 * (each byte holds the pair of codes one conversion instruction turns into an
 * fp16 pair).  The 6-bit formats use the 6-bit layout above. */
static inline int64_t fp4_nibble_byte(int64_t n, int64_t k, int64_t K, int *shift)
{
    int64_t base = ((n / 128) * (K / 64) + (k / 64)) * 4096;
    int r = (int)(n % 128), kk = (int)(k % 64), w = kk / 8;
    *shift = 4 * (kk % 2);
    return base + (w / 4) * 2048 + r * 16 + (w % 4) * 4 + (kk % 8) / 2;
}

int oracle_fpx_prepack(int fmt, const uint8_t *codes, int64_t N, int64_t K, uint8_t *packed)
{
    if (fmt == 0 || fmt == 1) return oracle_prepack(codes, N, K, packed);
    if (fmt != 2 && fmt != 3) return ORC_ERR_INVALID_ARG;
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    if (fmt == 3) {
        memset(packed, 0, (size_t)(N * K / 8 * 5));
        for (int64_t n = 0; n < N; ++n)
            for (int64_t k = 0; k < K; ++k) {
                int64_t pb, qb;
                int ps, qs;
                fp5_positions(n, k, K, &pb, &ps, &qb, &qs);
                uint8_t c = codes[n * K + k] & 0x1F;
                packed[pb] |= (uint8_t)((c >> 1) << ps);
                packed[qb] |= (uint8_t)((c & 1) << qs);
            }
        return ORC_OK;
    }
    memset(packed, 0, (size_t)(N * K / 2));
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int sh;
            int64_t b = fp4_nibble_byte(n, k, K, &sh);
            packed[b] |= (uint8_t)((codes[n * K + k] & 0xF) << sh);
        }
    return ORC_OK;
}

int oracle_fpx_unpack(int fmt, const uint8_t *packed, int64_t N, int64_t K, uint8_t *codes)
{
    if (fmt == 0 || fmt == 1) return oracle_unpack(packed, N, K, codes);
    if (fmt != 2 && fmt != 3) return ORC_ERR_INVALID_ARG;
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    if (fmt == 3) {
        for (int64_t n = 0; n < N; ++n)
            for (int64_t k = 0; k < K; ++k) {
                int64_t pb, qb;
                int ps, qs;
                fp5_positions(n, k, K, &pb, &ps, &qb, &qs);
                codes[n * K + k] = (uint8_t)((((packed[pb] >> ps) & 0xF) << 1) | ((packed[qb] >> qs) & 1));
            }
        return ORC_OK;
    }
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int sh;
            int64_t b = fp4_nibble_byte(n, k, K, &sh);
            codes[n * K + k] = (uint8_t)((packed[b] >> sh) & 0xF);
        }
    return ORC_OK;
}

int oracle_fpx_dequant(int fmt, const uint8_t *packed, const uint16_t *scales, int64_t N, int64_t K, uint16_t *W16)
{
    fpx_fmt f;
    if (!fpx_get(fmt, &f)) return ORC_ERR_INVALID_ARG;
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    uint8_t *codes = (uint8_t *)malloc((size_t)(N * K) + 1);
    if (!codes) return ORC_ERR_INVALID_ARG;
    oracle_fpx_unpack(fmt, packed, N, K, codes);
    for (int64_t n = 0; n < N; ++n) {
        double s = scales ? oracle_f16_to_f64(scales[n]) : 1.0;
        for (int64_t k = 0; k < K; ++k)
            W16[n * K + k] = oracle_f64_to_f16_rne(fpx_decode_one(&f, codes[n * K + k]) * s);
    }
    free(codes);
    return ORC_OK;
}

/* The plain definition again, with the format's decode table. */
int oracle_fpx_linear(int fmt, const uint16_t *x, const uint8_t *codes, const uint16_t *scales,
                      int64_t M, int64_t N, int64_t K, uint16_t *y)
{
    fpx_fmt f;
    if (!fpx_get(fmt, &f)) return ORC_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    double table[64];
    oracle_fpx_decode_table(fmt, table);
    int mask = oracle_fpx_codes(fmt) - 1;
    double *xr = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    if (!xr) return ORC_ERR_INVALID_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) xr[k] = oracle_f16_to_f64(x[m * K + k]);
        for (int64_t n = 0; n < N; ++n) {
            double s = oracle_f16_to_f64(scales[n]);
            const uint8_t *c = codes + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += xr[k] * (s * table[c[k] & mask]);
            y[m * N + n] = oracle_f64_to_f16_rne(acc);
        }
    }
    free(xr);
    return ORC_OK;
}

/* ---- 2:4 sparse INT4 weights (Sparse-Marlin) --------------------------------
 * The Sparse-Marlin post (INT4 x FP16 kernel with 2:4 sparsity) names the
 * pieces: 4-bit weights, 2:4 sparsity with metadata giving the positions of
 * the kept weights, quantization statistics, sparse tensor cores.  It fixes
 * none of their details; the readings taken here are the plain ones:
 *   pruning  in each group of 4 consecutive weights of a row (k = 4j..4j+3)
 *            the two with the largest |w| are kept, ties going to the lower
 *            position; the other two become zero;
 *   scale    one fp16 scale per output row, s = fp16_rne(fp32(max|w| / 7));
 *   codes    q = round-half-even(w / s), clamped to [-8, 7] (signed 4-bit);
 *   value    s * q at the kept positions, 0 elsewhere.
 * Per group the two kept codes are stored in position order with their
 * positions i0 < i1 (2 bits each).
 */

/* Positions kept in one group of four (i0 < i1). */
static void s24_keep(const float *w, int *i0, int *i1)
{
    int best = 0;
    for (int i = 1; i < 4; ++i)
        if (fabsf(w[i]) > fabsf(w[best])) best = i;          /* strict: ties keep the lower */
    int second = -1;
    for (int i = 0; i < 4; ++i) {
        if (i == best) continue;
        if (second < 0 || fabsf(w[i]) > fabsf(w[second])) second = i;
    }
    *i0 = best < second ? best : second;
    *i1 = best < second ? second : best;
}

/* Round-half-even of v (binary64) to an integer, clamped to [-8, 7]. */
static int s24_round(double v)
{
    double r = nearbyint(v);                                 /* default rounding: to nearest, ties to even */
    if (r > 7.0) r = 7.0;
    if (r < -8.0) r = -8.0;
    return (int)r;
}

/* W [N,K] fp32 -> q [N,K/2] (int8, kept codes in position order),
 * pos [N,K/2] (their positions 0..3 within the group), scales [N] (fp16 bits).
 * K must be a multiple of 4. */
int oracle_s24_quantize(const float *W, int64_t N, int64_t K, int8_t *q, uint8_t *pos, uint16_t *scales)
{
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (K % 4) return ORC_ERR_UNSUPPORTED_SHAPE;
    for (int64_t n = 0; n < N; ++n) {
        const float *row = W + n * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (!isfinite(row[k])) return ORC_ERR_NONFINITE;
            float a = fabsf(row[k]);
            if (a > amax) amax = a;
        }
        double s = 0.0;
        if (amax == 0.0f) {
            scales[n] = 0;
        } else {
            volatile float s32 = amax / 7.0f;                /* IEEE fp32 division */
            uint16_t s16 = oracle_f64_to_f16_rne((double)s32);
            if ((s16 & 0x7FFFu) >= 0x7C00u || (s16 & 0x7FFFu) == 0) return ORC_ERR_SCALE_RANGE;
            scales[n] = s16;
            s = oracle_f16_to_f64(s16);
        }
        for (int64_t j = 0; j < K / 4; ++j) {
            int i0, i1;
            s24_keep(row + 4 * j, &i0, &i1);
            int64_t o = n * (K / 2) + 2 * j;
            pos[o] = (uint8_t)i0;
            pos[o + 1] = (uint8_t)i1;
            q[o] = (int8_t)(s > 0.0 ? s24_round((double)row[4 * j + i0] / s) : 0);
            q[o + 1] = (int8_t)(s > 0.0 ? s24_round((double)row[4 * j + i1] / s) : 0);
        }
    }
    return ORC_OK;
}

/* Packed size: 3/8 byte per weight (two 4-bit codes and two 2-bit positions
 * per four weights). */
int64_t oracle_s24_packed_bytes(int64_t N, int64_t K)
{
    return N * K / 8 * 3;
}

/* Packed layout: tiles of 128 rows x 64 columns, 3072 bytes each, stored
 * like the other formats' tiles (column-tile index fastest).  Row r of a tile
 * owns four code words V_w at byte r*16 + 4w and two position words P_h at
 * byte 2048 + r*8 + 4h.  Group j (0..15) of the tile row: its codes in byte
 * j%4 of V_{j/4} (first kept code in the low nibble, second in the high
 * nibble, 4-bit two's complement), its positions in bits 4(j%8)..4(j%8)+3 of
 * P_{j/8} (i0 in the low two bits, i1 in the next two).  Words are
 * little-endian. */
static inline int64_t s24_tile_base(int64_t n, int64_t k, int64_t K)
{
    return ((n / 128) * (K / 64) + (k / 64)) * 3072;
}

int oracle_s24_prepack(const int8_t *q, const uint8_t *pos, int64_t N, int64_t K, uint8_t *packed)
{
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    memset(packed, 0, (size_t)(N * K / 8 * 3));
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < K / 4; ++g) {                /* group g of the row: columns 4g..4g+3 */
            int64_t base = s24_tile_base(n, 4 * g, K);
            int r = (int)(n % 128), j = (int)(g % 16);
            int64_t o = n * (K / 2) + 2 * g;
            uint8_t codes = (uint8_t)((q[o] & 0xF) | ((q[o + 1] & 0xF) << 4));
            packed[base + r * 16 + 4 * (j / 4) + (j % 4)] = codes;
            uint8_t meta = (uint8_t)((pos[o] & 3) | ((pos[o + 1] & 3) << 2));
            int bit = 4 * (j % 8);
            packed[base + 2048 + r * 8 + 4 * (j / 8) + bit / 8] |= (uint8_t)(meta << (bit % 8));
        }
    return ORC_OK;
}

int oracle_s24_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *q, uint8_t *pos)
{
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < K / 4; ++g) {
            int64_t base = s24_tile_base(n, 4 * g, K);
            int r = (int)(n % 128), j = (int)(g % 16);
            int64_t o = n * (K / 2) + 2 * g;
            uint8_t codes = packed[base + r * 16 + 4 * (j / 4) + (j % 4)];
            int lo = codes & 0xF, hi = codes >> 4;
            q[o] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            q[o + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
            int bit = 4 * (j % 8);
            uint8_t meta = (uint8_t)((packed[base + 2048 + r * 8 + 4 * (j / 8) + bit / 8] >> (bit % 8)) & 0xF);
            pos[o] = (uint8_t)(meta & 3);
            pos[o + 1] = (uint8_t)(meta >> 2);
        }
    return ORC_OK;
}

/* Dense fp16 weights: fp16_rne(s * q) at the kept positions (fp16(q) without
 * scales), +0 elsewhere. */
int oracle_s24_dequant(const uint8_t *packed, const uint16_t *scales, int64_t N, int64_t K, uint16_t *W16)
{
    if (N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (N % 128 || K % 64) return ORC_ERR_UNSUPPORTED_SHAPE;
    int8_t *q = (int8_t *)malloc((size_t)(N * K / 2) + 1);
    uint8_t *pos = (uint8_t *)malloc((size_t)(N * K / 2) + 1);
    if (!q || !pos) {
        free(q);
        free(pos);
        return ORC_ERR_INVALID_ARG;
    }
    oracle_s24_unpack(packed, N, K, q, pos);
    memset(W16, 0, sizeof(uint16_t) * (size_t)(N * K));
    for (int64_t n = 0; n < N; ++n) {
        double s = scales ? oracle_f16_to_f64(scales[n]) : 1.0;
        for (int64_t g = 0; g < K / 4; ++g)
            for (int a = 0; a < 2; ++a) {
                int64_t o = n * (K / 2) + 2 * g + a;
                W16[n * K + 4 * g + pos[o]] = oracle_f64_to_f16_rne(s * (double)q[o]);
            }
    }
    free(q);
    free(pos);
    return ORC_OK;
}

/* y[M,N] = fp16_rne( sum_k x[m,k] * s_n * v[n,k] ), v the dense code values
 * (q at kept positions, 0 elsewhere), summed in binary64. */
int oracle_s24_linear(const uint16_t *x, const int8_t *q, const uint8_t *pos, const uint16_t *scales,
                      int64_t M, int64_t N, int64_t K, uint16_t *y)
{
    if (M < 0 || N < 0 || K < 0) return ORC_ERR_INVALID_ARG;
    if (K % 4) return ORC_ERR_UNSUPPORTED_SHAPE;
    double *xr = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    if (!xr) return ORC_ERR_INVALID_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) xr[k] = oracle_f16_to_f64(x[m * K + k]);
        for (int64_t n = 0; n < N; ++n) {
            double s = oracle_f16_to_f64(scales[n]);
            double acc = 0.0;
            for (int64_t g = 0; g < K / 4; ++g)
                for (int a = 0; a < 2; ++a) {
                    int64_t o = n * (K / 2) + 2 * g + a;
                    acc += xr[4 * g + pos[o]] * (s * (double)q[o]);
                }
            y[m * N + n] = oracle_f64_to_f16_rne(acc);
        }
    }
    free(xr);
    return ORC_OK;
}
