/*
 * mx_oracle.c -- plain, slow, obviously-correct CPU oracle for microscaling
 * quantization (MXFP8 E4M3/E5M2, MXFP6 E3M2, MXFP4, NVFP4) and the
 * block-scaled GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA implementation.
 *
 * Every decision is made in fp64 on exactly-representable values, element by
 * element, in the order the pages describe.  Sources (page title, section):
 *
 *   [MXFP4-page]  "Microscaling MXFP4/NVFP4 on Blackwell for reasoning LLMs"
 *                 (produtoramaxvision.com.br blog).  Sections "Fundamentos
 *                 matemáticos do formato MXFP4 e E8M0" (E2M1 value set, E8M0
 *                 formula, dequantization by multiplication, 4.25 bits/element,
 *                 format table with the E4M3 range [-448, 448]) and the FAQ entry
 *                 on how E8M0 computes the block's shared exponent (the ceil
 *                 scale rule).  The same page's format table lists MXFP6 as
 *                 E3M2 elements with an E8M0 scale per 32-element block,
 *                 6.25 bits/element.
 *   [NVFP4-news]  "NVIDIA's FP4 format delivers 1.68x speedup" (zubnet.ai):
 *                 NVFP4 = E2M1 elements in 16-element blocks; MXFP8 = E4M3/E5M2
 *                 elements in 32-element blocks (OCP standard).
 *   [OAS/MBS]     "Unveiling the Potential of Quantization with MXFP4:
 *                 Strategies for Quantization Error Reduction" (gist.science),
 *                 section "Metodologia e Propostas" A: the standard MX mapping
 *                 puts the block maximum into (3, 6] of the E2M1 range.
 *
 * Readings taken where the pages are silent:
 *   R1  rounding of elements is round-to-nearest, ties to the even code, and
 *       saturating ("satfinite") at the format's largest finite magnitude;
 *   R2  the sign of a value that rounds to zero is kept (-0 -> 0x8 / 0x80);
 *   R3  an all-zero MX block gets E8M0 byte 0 (the ceil rule's limit, clamped);
 *       E8M0 0xFF is NaN and never produced;
 *   R4  NVFP4 global scale g = amax_t / (6 * 448) rounded UP to fp32
 *       (amax_t == 0 -> g = 1); g is a decode multiplier like the E8M0 scale;
 *   R5  NVFP4 block scale s = the smallest positive finite E4M3 value with
 *       amax_b <= 6 * g * s (the ceil rule carried to an E4M3 scale); an
 *       all-zero block gets s = 0 (code 0x00) and all-zero codes;
 *   R6  FP4 packing: byte j of a row = code[2j] | code[2j+1] << 4;
 *   R7  block-scale byte (r, c) of an [R x C] scale matrix lives at
 *       ((r/128) * ceil(C/4) + c/4) * 512 + (r%32)*16 + ((r%128)/32)*4 + c%4,
 *       padding bytes are 0;
 *   R18 E3M2 is the OCP 6-bit layout (sign, 3 exponent bits with bias 3, 2
 *       mantissa bits, no infinities or NaN, largest magnitude 28); MXFP6
 *       packing: code k of a row occupies bits 6k .. 6k+5 of the row read as
 *       one little-endian bit string (16 codes in 12 bytes).
 *   R20 MXFP4 with static macro-block scaling [OAS/MBS page, section B]: E2M1
 *       elements in 1x16 base blocks with E8M0 scales (tiled as NVFP4's), and
 *       per 1x128 macro block a factor 1 + m/256 (m one byte, 8 mantissa
 *       bits) chosen from the macro block's max alpha so that alpha / (1 +
 *       m/256) lands at or just below 6 * 2^e, e = floor(log2(alpha / 6)):
 *       m = the smallest integer in [0, 255] with alpha <= 6 (256 + m) 2^(e-8)
 *       (0 if alpha == 0 or none suffices).  Each base block then takes the MX
 *       rule on x / (1 + m/256) and RNE elements of that quotient.  The
 *       macro bytes are stored after the scale tiles, row-major [rows][K/128].
 *   R21 MXFP4 with dynamic macro-block scaling [OAS/MBS page, section B, the
 *       variant whose macro factor minimises the squared error]: the same
 *       storage and per-m quantization as R20, with m = the byte in [0, 255]
 *       whose quantization of the macro block has the smallest sum of squared
 *       errors sum_i (x_i - xhat_i)^2, the terms (each exact in fp64) added in
 *       element order in fp64; ties go to the smallest m.  (The page names a
 *       lookup table computed to minimise the error; an exhaustive search is
 *       the error-minimising choice that table stands for.)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <float.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_MXFP8_E4M3 = 0, ORC_MXFP8_E5M2 = 1, ORC_MXFP4 = 2, ORC_NVFP4 = 3, ORC_MXFP6_E3M2 = 4, ORC_MXFP4_MBS = 5 };
enum { ORC_OK = 0, ORC_EINVAL = 1, ORC_ENONFINITE = 2 };

/* ------------------------------------------------------------------------- */
/* threads                                                                   */
/* ------------------------------------------------------------------------- */
void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* bf16                                                                      */
/* ------------------------------------------------------------------------- */

/* bf16 is the top half of an IEEE binary32. */
double orc_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round an fp64 value to bf16 with round-to-nearest-even, in one rounding.
 * Finite values at or above the midpoint between the largest finite bf16 and
 * 2^128 go to infinity, as IEEE RNE overflow does. */
uint16_t orc_double_to_bf16_rne(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    const double overflow_mid = ldexp(2.0 - ldexp(1.0, -8), 127);
    if (a >= overflow_mid) return sign | 0x7F80;
    int ex;
    frexp(a, &ex);              /* a = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;             /* a in [2^e, 2^(e+1)) */
    if (e < -126) e = -126;     /* subnormal range has the quantum of 2^-126 * 2^-7 */
    double quantum = ldexp(1.0, e - 7);
    double n = a / quantum;     /* exact: power-of-two scaling */
    double r = rint(n);         /* default rounding mode: nearest, ties to even */
    double val = r * quantum;   /* exactly a bf16 value */
    float f = (float)val;       /* exact */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------- */
/* element and scale formats, decoded bit by bit                             */
/* ------------------------------------------------------------------------- */

/* E2M1 [MXFP4-page, Fundamentos]: bit 3 sign, bits 2-1 exponent with bias 1,
 * bit 0 mantissa.  Exponent field 0 is subnormal: 0 or 0.5. */
double orc_e2m1_decode(uint8_t code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 (OCP "fn" variant named by the MXFP8 definition): bias 7, no infinities,
 * S.1111.111 is NaN, largest finite 448 = 1.75 * 2^8 [MXFP4-page table, FP8 (E4M3)
 * range [-448, 448]]. */
double orc_e4m3_decode(uint8_t code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* E5M2: bias 15, IEEE-style infinities and NaNs, largest finite 57344. */
double orc_e5m2_decode(uint8_t code) {
    int s = (code >> 7) & 1, e = (code >> 2) & 31, m = code & 3;
    double mag;
    if (e == 31) {
        if (m != 0) return NAN;
        mag = INFINITY;
    } else if (e == 0) {
        mag = ldexp((double)m, -16);
    } else {
        mag = ldexp(1.0 + m / 4.0, e - 15);
    }
    return s ? -mag : mag;
}

/* E3M2 [MXFP4-page format table, MXFP6 (E3M2); reading R18]: bit 5 sign,
 * bits 4-2 exponent with bias 3, bits 1-0 mantissa; exponent field 0 is
 * subnormal (m/4 * 2^-2); every code is finite, the largest 1.75 * 2^4 = 28. */
double orc_e3m2_decode(uint8_t code) {
    int s = (code >> 5) & 1, e = (code >> 2) & 7, m = code & 3;
    double mag = (e == 0) ? ldexp((double)m, -4) : ldexp(1.0 + m / 4.0, e - 3);
    return s ? -mag : mag;
}

/* E8M0 [MXFP4-page, Fundamentos]: Escala = 2^(E - 127); 0xFF is NaN. */
double orc_e8m0_decode(uint8_t code) {
    if (code == 0xFF) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* Sorted tables of the non-negative finite values of each element format,
 * indexed by code.  Built from the decoders above. */
static double g_e2m1_pos[8];
static double g_e4m3_pos[127];   /* codes 0x00 .. 0x7E */
static double g_e5m2_pos[124];   /* codes 0x00 .. 0x7B */
static double g_e3m2_pos[32];    /* codes 0x00 .. 0x1F */
static int g_tables_ready = 0;

static void build_tables(void) {
    if (g_tables_ready) return;
    for (int c = 0; c < 8; ++c) g_e2m1_pos[c] = orc_e2m1_decode((uint8_t)c);
    for (int c = 0; c < 127; ++c) g_e4m3_pos[c] = orc_e4m3_decode((uint8_t)c);
    for (int c = 0; c < 124; ++c) g_e5m2_pos[c] = orc_e5m2_decode((uint8_t)c);
    for (int c = 0; c < 32; ++c) g_e3m2_pos[c] = orc_e3m2_decode((uint8_t)c);
    g_tables_ready = 1;
}

/* Round |v| onto a sorted table with round-to-nearest, ties to the even code
 * (consecutive codes differ in their mantissa LSB, so "even code" is "even
 * mantissa"), saturating at the last entry [reading R1]. */
static int rne_index(const double *tab, int n, double a) {
    if (a >= tab[n - 1]) return n - 1;
    int lo = 0, hi = n - 1;           /* invariant: tab[lo] <= a < tab[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (tab[mid] <= a) lo = mid; else hi = mid;
    }
    double midpoint = 0.5 * (tab[lo] + tab[hi]);   /* exact in fp64 */
    if (a < midpoint) return lo;
    if (a > midpoint) return hi;
    return (lo % 2 == 0) ? lo : hi;
}

/* Encoders: sign kept even when the magnitude rounds to zero [reading R2]. */
uint8_t orc_e2m1_encode(double v) {
    build_tables();
    int c = rne_index(g_e2m1_pos, 8, fabs(v));
    return (uint8_t)(c | (signbit(v) ? 0x8 : 0));
}

uint8_t orc_e4m3_encode(double v) {
    build_tables();
    if (isnan(v)) return 0x7F;
    int c = rne_index(g_e4m3_pos, 127, fabs(v));
    return (uint8_t)(c | (signbit(v) ? 0x80 : 0));
}

uint8_t orc_e5m2_encode(double v) {
    build_tables();
    if (isnan(v)) return 0x7F;
    int c = rne_index(g_e5m2_pos, 124, fabs(v));
    return (uint8_t)(c | (signbit(v) ? 0x80 : 0));
}

uint8_t orc_e3m2_encode(double v) {
    build_tables();
    int c = rne_index(g_e3m2_pos, 32, fabs(v));
    return (uint8_t)(c | (signbit(v) ? 0x20 : 0));
}

/* ------------------------------------------------------------------------- */
/* format parameters                                                         */
/* ------------------------------------------------------------------------- */
static int fmt_block(int fmt) { return (fmt == ORC_NVFP4 || fmt == ORC_MXFP4_MBS) ? 16 : 32; }
static int fmt_ok(int fmt) { return fmt >= 0 && fmt <= 5; }
static int fmt_bits(int fmt) {
    return (fmt == ORC_MXFP4 || fmt == ORC_NVFP4 || fmt == ORC_MXFP4_MBS) ? 4 : (fmt == ORC_MXFP6_E3M2 ? 6 : 8);
}
static double fmt_maxelem(int fmt) {
    switch (fmt) {
    case ORC_MXFP8_E4M3: return 448.0;
    case ORC_MXFP8_E5M2: return 57344.0;
    case ORC_MXFP6_E3M2: return 28.0;
    default: return 6.0;
    }
}
static double fmt_decode(int fmt, uint8_t code) {
    switch (fmt) {
    case ORC_MXFP8_E4M3: return orc_e4m3_decode(code);
    case ORC_MXFP8_E5M2: return orc_e5m2_decode(code);
    case ORC_MXFP6_E3M2: return orc_e3m2_decode(code & 0x3F);
    default: return orc_e2m1_decode(code & 0xF);
    }
}
static uint8_t fmt_encode(int fmt, double v) {
    switch (fmt) {
    case ORC_MXFP8_E4M3: return orc_e4m3_encode(v);
    case ORC_MXFP8_E5M2: return orc_e5m2_encode(v);
    case ORC_MXFP6_E3M2: return orc_e3m2_encode(v);
    default: return orc_e2m1_encode(v);
    }
}

int orc_block_size(int fmt) { return fmt_block(fmt); }
double orc_max_element(int fmt) { return fmt_maxelem(fmt); }

/* ------------------------------------------------------------------------- */
/* storage: packed codes and the 128x4-tiled block-scale layout              */
/* ------------------------------------------------------------------------- */
static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t orc_codes_bytes(int fmt, int64_t rows, int64_t cols) {
    return (size_t)(rows * cols * fmt_bits(fmt) / 8);
}

/* Bytes of the 128x4 scale tiles; MXFP4-MBS appends its macro bytes. */
static size_t tile_bytes(int fmt, int64_t rows, int64_t cols) {
    int64_t sc = cols / fmt_block(fmt);
    return (size_t)(ceil_div(rows, 128) * 128 * ceil_div(sc, 4) * 4);
}

size_t orc_scales_bytes(int fmt, int64_t rows, int64_t cols) {
    size_t t = tile_bytes(fmt, rows, cols);
    if (fmt == ORC_MXFP4_MBS) t += (size_t)(ceil_div(rows * (cols / 128), 16) * 16);
    return t;
}

/* [reading R20] offset of macro byte (r, mb) in an MXFP4-MBS scale buffer */
size_t orc_mbs_macro_offset(int64_t rows, int64_t cols, int64_t r, int64_t mb) {
    return tile_bytes(ORC_MXFP4_MBS, rows, cols) + (size_t)(r * (cols / 128) + mb);
}

/* [reading R7] position of scale (r, c) in a scale matrix with sf_cols columns */
size_t orc_sf_offset(int64_t r, int64_t c, int64_t sf_cols) {
    int64_t tiles_per_row = ceil_div(sf_cols, 4);
    int64_t tile = (r / 128) * tiles_per_row + c / 4;
    return (size_t)(tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4));
}

/* ------------------------------------------------------------------------- */
/* scale rules                                                               */
/* ------------------------------------------------------------------------- */

/* MX block exponent [MXFP4-page, FAQ on E8M0]:
 *   E = ceil(log2(max_val / max_elem)) + 127,
 * i.e. the smallest integer e with max_val <= max_elem * 2^e, found exactly by
 * comparing against ldexp (never a floating log2).  Clamped to [0, 254]
 * [reading R3]; max_val == 0 gives 0. */
int orc_mx_scale_byte(double amax, double maxelem) {
    if (!(amax > 0.0)) return 0;
    int e = ilogb(amax) - ilogb(maxelem);
    while (amax > ldexp(maxelem, e)) ++e;
    while (amax <= ldexp(maxelem, e - 1)) --e;
    int E = e + 127;
    if (E < 0) E = 0;
    if (E > 254) E = 254;
    return E;
}

/* [reading R4] g = RU_fp32(amax_t / 2688); the real quotient is bracketed by
 * exact fp64 products f * 2688 (f has 24 significant bits, 2688 = 21 * 2^7). */
float orc_nvfp4_global_scale(double amax_t) {
    if (!(amax_t > 0.0)) return 1.0f;
    float f = (float)(amax_t / 2688.0);
    while ((double)f * 2688.0 < amax_t) f = nextafterf(f, INFINITY);
    for (;;) {
        float p = nextafterf(f, 0.0f);
        if (p > 0.0f && (double)p * 2688.0 >= amax_t) f = p; else break;
    }
    return f;
}

/* [reading R20] MBS-static macro mantissa of a macro block with max alpha:
 * e with 6 * 2^e <= alpha < 6 * 2^(e+1), then the smallest m in [0, 255]
 * with alpha <= 6 (256 + m) 2^(e - 8); 0 if alpha == 0 or no m suffices.
 * Every product is an integer of at most 12 bits times a power of two: exact. */
int orc_mbs_static_mantissa(double alpha) {
    if (!(alpha > 0.0)) return 0;
    int e = ilogb(alpha) - 2;
    while (ldexp(6.0, e) > alpha) --e;
    while (ldexp(6.0, e + 1) <= alpha) ++e;
    for (int m = 0; m < 256; ++m)
        if (alpha <= ldexp(6.0 * (256 + m), e - 8)) return m;
    return 0;
}

/* [reading R20] base-block exponent under macro mantissa m: the smallest E in
 * [0, 254] with amax_b <= 6 (256 + m) 2^(E - 135), i.e. amax_b / (1 + m/256)
 * <= 6 * 2^(E - 127); 254 if none. */
int orc_mbs_block_exponent(double amax_b, int m) {
    for (int E = 0; E <= 254; ++E)
        if (amax_b <= ldexp(6.0 * (256 + m), E - 135)) return E;
    return 254;
}

/* [reading R5] smallest positive finite E4M3 s with amax_b <= 6 * g * s.
 * 6 * g * s has at most 24 + 4 + 2 significant bits: exact in fp64. */
uint8_t orc_nvfp4_block_scale(double amax_b, float g) {
    build_tables();
    if (!(amax_b > 0.0)) return 0x00;
    for (int c = 1; c <= 126; ++c)
        if (amax_b <= 6.0 * (double)g * g_e4m3_pos[c]) return (uint8_t)c;
    return 0x7E;
}

/* ------------------------------------------------------------------------- */
/* quantize / dequantize                                                     */
/* ------------------------------------------------------------------------- */

static void put_code(int fmt, uint8_t *codes, int64_t K, int64_t r, int64_t k, uint8_t q) {
    if (fmt_bits(fmt) == 8) {
        codes[r * K + k] = q;
    } else if (fmt_bits(fmt) == 6) {
        uint8_t *row = &codes[r * (K / 4) * 3];        /* [reading R18] bit 6k + i of the row */
        for (int i = 0; i < 6; ++i) {
            int64_t bit = 6 * k + i;
            uint8_t mask = (uint8_t)(1u << (bit % 8));
            if ((q >> i) & 1) row[bit / 8] |= mask; else row[bit / 8] &= (uint8_t)~mask;
        }
    } else {
        uint8_t *byte = &codes[r * (K / 2) + k / 2];
        if (k % 2 == 0) *byte = (uint8_t)((*byte & 0xF0) | (q & 0xF));      /* [reading R6] */
        else            *byte = (uint8_t)((*byte & 0x0F) | ((q & 0xF) << 4));
    }
}

static uint8_t get_code(int fmt, const uint8_t *codes, int64_t K, int64_t r, int64_t k) {
    if (fmt_bits(fmt) == 8) return codes[r * K + k];
    if (fmt_bits(fmt) == 6) {
        const uint8_t *row = &codes[r * (K / 4) * 3];
        uint8_t q = 0;
        for (int i = 0; i < 6; ++i) {
            int64_t bit = 6 * k + i;
            q |= (uint8_t)(((row[bit / 8] >> (bit % 8)) & 1) << i);
        }
        return q;
    }
    uint8_t byte = codes[r * (K / 2) + k / 2];
    return (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
}

/* Largest |x| over a bf16 tensor (fp64). */
double orc_amax_bf16(const uint16_t *src, int64_t M, int64_t K, int64_t ld) {
    double amax = 0.0;
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            double a = fabs(orc_bf16_to_double(src[r * ld + k]));
            if (a > amax) amax = a;
        }
    return amax;
}

/* NVFP4 element: RNE of the real quotient |x| / denom onto E2M1 (ties to the
 * even code), saturating at 6, decided by comparing |x| with each midpoint m
 * times denom.  m has at most 3 significant bits and denom = g * s at most
 * 28, so m * denom is exact in fp64 and every comparison is exact, whatever
 * the precision of x (bf16 or fp32). */
static uint8_t e2m1_encode_quotient(double x, double denom) {
    static const double mids[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
    double a = fabs(x);
    int c = 0;
    for (int k = 0; k < 7; ++k) {
        double t = mids[k] * denom;
        if (a > t) c = k + 1;
        else {
            if (a == t) c = (k % 2 == 0) ? k : k + 1;   /* tie: the even code */
            break;
        }
    }
    return (uint8_t)(c | (signbit(x) ? 0x8 : 0));
}

int orc_mbs_dynamic_mantissa(const double *mac);

/* Quantize a dense row-major [M x K] matrix of exactly-held values xv (fp64).
 * codes: orc_codes_bytes bytes; scales: orc_scales_bytes bytes (fully written,
 * padding 0).  NVFP4: if gscale_given, *gscale is used as g, else g is computed
 * from max |xv| and stored to *gscale.  mx_threshold: the value a block's max
 * |x| is mapped at or below by the MX scale (the format's largest element for
 * the OCP rule). */
static int quantize_core(int fmt, double mx_threshold, const double *xv, int64_t M, int64_t K, uint8_t *codes,
                         uint8_t *scales, float *gscale, int gscale_given, int mbs_dynamic) {
    build_tables();
    int bs = fmt_block(fmt);
    int64_t sf_cols = K / bs;
    memset(scales, 0, orc_scales_bytes(fmt, M, K));
    memset(codes, 0, orc_codes_bytes(fmt, M, K));
    double maxelem = mx_threshold;
    float g = 1.0f;
    if (fmt == ORC_NVFP4) {
        if (gscale_given) g = *gscale;
        else {
            double amax_t = 0.0;
            for (int64_t i = 0; i < M * K; ++i)
                if (fabs(xv[i]) > amax_t) amax_t = fabs(xv[i]);
            g = orc_nvfp4_global_scale(amax_t);
            *gscale = g;
        }
    }
    if (fmt == ORC_MXFP4_MBS) {
        /* [reading R20]: macro mantissa per 128 elements (R21: by error
         * search), then 16-element blocks on x / (1 + m/256), elements decided
         * by exact comparisons with the quotient's E2M1 midpoints (denominator
         * (256+m) 2^(E-135)). */
        #pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < M; ++r) {
            for (int64_t mb = 0; mb < K / 128; ++mb) {
                const double *mac = xv + r * K + mb * 128;
                int m;
                if (mbs_dynamic) {
                    m = orc_mbs_dynamic_mantissa(mac);
                } else {
                    double alpha = 0.0;
                    for (int i = 0; i < 128; ++i)
                        if (fabs(mac[i]) > alpha) alpha = fabs(mac[i]);
                    m = orc_mbs_static_mantissa(alpha);
                }
                scales[orc_mbs_macro_offset(M, K, r, mb)] = (uint8_t)m;
                for (int jb = 0; jb < 8; ++jb) {
                    const double *blk = mac + jb * 16;
                    double amax = 0.0;
                    for (int i = 0; i < 16; ++i)
                        if (fabs(blk[i]) > amax) amax = fabs(blk[i]);
                    int E = orc_mbs_block_exponent(amax, m);
                    int64_t j = mb * 8 + jb;
                    scales[orc_sf_offset(r, j, sf_cols)] = (uint8_t)E;
                    double denom = ldexp((double)(256 + m), E - 135);
                    for (int i = 0; i < 16; ++i)
                        put_code(fmt, codes, K, r, j * 16 + i, e2m1_encode_quotient(blk[i], denom));
                }
            }
        }
        return ORC_OK;
    }
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t j = 0; j < sf_cols; ++j) {
            const double *blk = xv + r * K + j * bs;
            double amax = 0.0;
            for (int i = 0; i < bs; ++i)
                if (fabs(blk[i]) > amax) amax = fabs(blk[i]);
            uint8_t sbyte;
            double denom;            /* the real number each element is divided by */
            if (fmt == ORC_NVFP4) {
                sbyte = orc_nvfp4_block_scale(amax, g);
                denom = (double)g * orc_e4m3_decode(sbyte);   /* exact product */
            } else {
                sbyte = (uint8_t)orc_mx_scale_byte(amax, maxelem);
                denom = orc_e8m0_decode(sbyte);
            }
            scales[orc_sf_offset(r, j, sf_cols)] = sbyte;
            for (int i = 0; i < bs; ++i) {
                double x = blk[i];
                uint8_t q;
                if (denom == 0.0)
                    q = fmt_encode(fmt, signbit(x) ? -0.0 : 0.0);  /* all-zero NVFP4 block */
                else if (fmt == ORC_NVFP4)
                    q = e2m1_encode_quotient(x, denom);
                else
                    q = fmt_encode(fmt, x / denom);                /* exact: a power of two */
                put_code(fmt, codes, K, r, j * bs + i, q);
            }
        }
    }
    return ORC_OK;
}

/* [reading R21] the squared error of one macro block (128 values) quantized
 * with macro mantissa m: per 16-element base block the exponent of R20, each
 * element's E2M1 value times (256 + m) 2^(E - 135) as xhat; every term
 * (x - xhat)^2 is exact in fp64 (xhat is 0 or within a factor of 3 of |x|, so
 * x - xhat has at most 22 significant bits), added in element order. */
double orc_mbs_macro_sse(const double *mac, int m) {
    double sse = 0.0;
    for (int jb = 0; jb < 8; ++jb) {
        const double *blk = mac + jb * 16;
        double amax = 0.0;
        for (int i = 0; i < 16; ++i)
            if (fabs(blk[i]) > amax) amax = fabs(blk[i]);
        int E = orc_mbs_block_exponent(amax, m);
        double denom = ldexp((double)(256 + m), E - 135);
        for (int i = 0; i < 16; ++i) {
            uint8_t q = e2m1_encode_quotient(blk[i], denom);
            double xhat = orc_e2m1_decode(q) * denom;
            double d = blk[i] - xhat;
            sse = sse + d * d;
        }
    }
    return sse;
}

/* [reading R21] the macro mantissa of the smallest squared error (ties: the
 * smallest m). */
int orc_mbs_dynamic_mantissa(const double *mac) {
    int best = 0;
    double best_sse = orc_mbs_macro_sse(mac, 0);
    for (int m = 1; m < 256; ++m) {
        double e = orc_mbs_macro_sse(mac, m);
        if (e < best_sse) {
            best_sse = e;
            best = m;
        }
    }
    return best;
}

/* bf16 source with row pitch ld: checks, widening to fp64 (exact), quantize. */
static int quantize_impl(int fmt, double mx_threshold, const uint16_t *src, int64_t M, int64_t K, int64_t ld,
                         uint8_t *codes, uint8_t *scales, float *gscale, int gscale_given, int mbs_dynamic) {
    int bs = fmt_block(fmt);
    if (!fmt_ok(fmt) || M < 0 || K < 0 || K % bs != 0 || ld < K) return ORC_EINVAL;
    if (fmt == ORC_MXFP4_MBS && K % 128 != 0) return ORC_EINVAL;
    double *xv = (double *)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    if (!xv) return ORC_EINVAL;
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            double x = orc_bf16_to_double(src[r * ld + k]);
            if (!isfinite(x)) {
                free(xv);
                return ORC_ENONFINITE;
            }
            xv[r * K + k] = x;
        }
    int rc = quantize_core(fmt, mx_threshold, xv, M, K, codes, scales, gscale, gscale_given, mbs_dynamic);
    free(xv);
    return rc;
}

/* Quantize an fp32 source [M x K] (row pitch ld), e.g. a rotated tensor. */
int orc_quantize_f32(int fmt, const float *src, int64_t M, int64_t K, int64_t ld, uint8_t *codes, uint8_t *scales,
                     float *gscale, int gscale_given) {
    int bs = fmt_block(fmt);
    if (!fmt_ok(fmt) || M < 0 || K < 0 || K % bs != 0 || ld < K) return ORC_EINVAL;
    if (fmt == ORC_MXFP4_MBS && K % 128 != 0) return ORC_EINVAL;
    double *xv = (double *)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    if (!xv) return ORC_EINVAL;
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            double x = (double)src[r * ld + k];
            if (!isfinite(x)) {
                free(xv);
                return ORC_ENONFINITE;
            }
            xv[r * K + k] = x;
        }
    int rc = quantize_core(fmt, fmt_maxelem(fmt), xv, M, K, codes, scales, gscale, gscale_given, 0);
    free(xv);
    return rc;
}

/* Walsh-Hadamard rotation of every 32-element block along K [MX page, section
 * "Técnicas de preservação de acurácia": Hadamard / Walsh-Hadamard rotations
 * spread a block's outlier energy over its 32 elements]:
 *   y_b = c * (H32 x_b),  H32 the Sylvester-ordered Hadamard matrix
 *   (H1 = [1], H2n = [[Hn, Hn], [Hn, -Hn]]),  c = RN_fp32(1 / sqrt(32)),
 * evaluated in fp32 exactly this way: butterflies with half-widths 1, 2, 4, 8,
 * 16 in that order, each (a, b) -> (a + b, a - b) rounded to fp32, then one
 * fp32 multiplication by c.  (The rounding of the intermediate sums is part of
 * the definition, so that a device computing the same steps matches bit for
 * bit.)  K % 32 == 0. */
int orc_rht32_f32(const uint16_t *src, int64_t M, int64_t K, int64_t ld, float *dst) {
    if (M < 0 || K < 0 || K % 32 != 0 || ld < K) return ORC_EINVAL;
    const float c = (float)(1.0 / sqrt(32.0));
    for (int64_t r = 0; r < M; ++r)
        for (int64_t j = 0; j < K / 32; ++j) {
            float v[32];
            for (int i = 0; i < 32; ++i) v[i] = (float)orc_bf16_to_double(src[r * ld + j * 32 + i]);
            for (int h = 1; h < 32; h <<= 1)
                for (int i0 = 0; i0 < 32; i0 += 2 * h)
                    for (int i = i0; i < i0 + h; ++i) {
                        float a = v[i], b = v[i + h];
                        v[i] = a + b;
                        v[i + h] = a - b;
                    }
            for (int i = 0; i < 32; ++i) dst[r * K + j * 32 + i] = v[i] * c;
        }
    return ORC_OK;
}

int orc_quantize(int fmt, const uint16_t *src, int64_t M, int64_t K, int64_t ld,
                 uint8_t *codes, uint8_t *scales, float *gscale, int gscale_given) {
    return quantize_impl(fmt, fmt_maxelem(fmt), src, M, K, ld, codes, scales, gscale, gscale_given, 0);
}

/* MXFP4 with dynamic macro-block scaling [reading R21]: MXFP4-MBS storage,
 * the macro mantissa of each 128 elements chosen by the squared-error search. */
int orc_quantize_mbs_dynamic(const uint16_t *src, int64_t M, int64_t K, int64_t ld, uint8_t *codes,
                             uint8_t *scales) {
    return quantize_impl(ORC_MXFP4_MBS, 6.0, src, M, K, ld, codes, scales, NULL, 0, 1);
}

/* MXFP4 with overflow-aware scaling [OAS page, section 2.A]: the block scale
 * maps the block's max |x| into (3.5, 7] instead of (3, 6], i.e.
 * E = ceil(log2(max_val / 7)) + 127; elements above 6 after scaling saturate
 * to 6 as any E2M1 value does.  Same storage as MXFP4. */
int orc_quantize_oas(const uint16_t *src, int64_t M, int64_t K, int64_t ld, uint8_t *codes, uint8_t *scales) {
    return quantize_impl(ORC_MXFP4, 7.0, src, M, K, ld, codes, scales, NULL, 0, 0);
}

/* Quantization SNR in dB [OAS page, section 3: "QSNR"]: 10 log10(sum x^2 /
 * sum (x - xhat)^2) over the tensor, in fp64 (xhat from orc_dequantize_f64).
 * sums[0] = sum x^2, sums[1] = sum (x - xhat)^2.  Returns +inf for zero error. */
double orc_qsnr_db(const uint16_t *src, int64_t M, int64_t K, int64_t ld, const double *xhat, double *sums) {
    double sx = 0.0, se = 0.0;
    for (int64_t r = 0; r < M; ++r)
        for (int64_t k = 0; k < K; ++k) {
            double x = orc_bf16_to_double(src[r * ld + k]);
            double e = x - xhat[r * K + k];
            sx += x * x;
            se += e * e;
        }
    if (sums) {
        sums[0] = sx;
        sums[1] = se;
    }
    if (se == 0.0) return INFINITY;
    return 10.0 * log10(sx / se);
}

/* The real factor of element (r, k): g * s (NVFP4), 2^(E-127) (MX), or
 * (1 + m/256) * 2^(E-127) (MXFP4-MBS, reading R20); exact in fp64. */
static double block_scale(int fmt, const uint8_t *scales, int64_t M, int64_t K, int64_t r, int64_t k, float gscale) {
    int bs = fmt_block(fmt);
    uint8_t sb = scales[orc_sf_offset(r, k / bs, K / bs)];
    if (fmt == ORC_NVFP4) return (double)gscale * orc_e4m3_decode(sb);
    if (fmt == ORC_MXFP4_MBS) {
        int m = scales[orc_mbs_macro_offset(M, K, r, k / 128)];
        return ldexp((double)(256 + m), (int)sb - 135);
    }
    return orc_e8m0_decode(sb);
}

/* Dequantize to fp64: x = g * s * q (g = 1 for MX) [MXFP4-page, Fundamentos:
 * x_real = S_E8M0 * x_E2M1].  The products are exact in fp64. */
int orc_dequantize_f64(int fmt, const uint8_t *codes, const uint8_t *scales, float gscale,
                       int64_t M, int64_t K, double *dst) {
    int bs = fmt_block(fmt);
    if (!fmt_ok(fmt) || K % bs != 0 || (fmt == ORC_MXFP4_MBS && K % 128 != 0)) return ORC_EINVAL;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            dst[r * K + k] = block_scale(fmt, scales, M, K, r, k, gscale) * fmt_decode(fmt, get_code(fmt, codes, K, r, k));
        }
    }
    return ORC_OK;
}

/* Dequantize to bf16 with one RNE rounding of the exact value. */
int orc_dequantize_bf16(int fmt, const uint8_t *codes, const uint8_t *scales, float gscale,
                        int64_t M, int64_t K, uint16_t *dst, int64_t ld) {
    int bs = fmt_block(fmt);
    if (!fmt_ok(fmt) || K % bs != 0 || ld < K || (fmt == ORC_MXFP4_MBS && K % 128 != 0)) return ORC_EINVAL;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            dst[r * ld + k] =
                orc_double_to_bf16_rne(block_scale(fmt, scales, M, K, r, k, gscale) * fmt_decode(fmt, get_code(fmt, codes, K, r, k)));
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* GEMM on dequantized operands                                              */
/* ------------------------------------------------------------------------- */

/* C[i][j] = sum_k A[i][k] * B[j][k] in fp64, and Cabs = sum_k |A||B| (for the
 * tolerance), for the listed rows of A only (rows == NULL: all M rows).
 * Output row t corresponds to A row rows[t]. */
int orc_gemm_f64(const double *A, const double *B, const int64_t *rows, int64_t nrows,
                 int64_t N, int64_t K, double *C, double *Cabs) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < nrows; ++t) {
        int64_t i = rows ? rows[t] : t;
        const double *a = A + i * K;
        for (int64_t j = 0; j < N; ++j) {
            const double *b = B + j * K;
            double acc = 0.0, accabs = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = a[k] * b[k];
                acc += p;
                accabs += fabs(p);
            }
            C[t * N + j] = acc;
            if (Cabs) Cabs[t * N + j] = accabs;
        }
    }
    return ORC_OK;
}

/* GELU with the exact erf form (the pages give no GELU; PyTorch's default form
 * is taken): 0.5 * x * (1 + erf(x / sqrt(2))), evaluated as
 * 0.5 * x * erfc(-x / sqrt(2)), the same function (1 + erf(y) = erfc(-y)) without
 * the cancellation that leaves nothing of the negative tail (x <= -8.5 would
 * come out as -0 where GELU is about -1e-18 at -9, a normal bf16 value). */
double orc_gelu(double x) { return 0.5 * x * erfc(-x / sqrt(2.0)); }

void orc_gelu_array(const double *x, double *y, int64_t n) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) y[i] = orc_gelu(x[i]);
}
