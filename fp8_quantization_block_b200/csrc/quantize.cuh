// quantize.cuh -- HBM-bound microscaling quantize / dequantize kernels (sm_100a).
//
// What is computed (page "Microscaling MXFP4/NVFP4 on Blackwell for reasoning
// LLMs", section "Fundamentos matemáticos do formato MXFP4 e E8M0", its format
// table (MXFP6 = E3M2 elements, E8M0 scale per 32) and the FAQ entry on how
// E8M0 picks the block exponent; NVFP4/MXFP8 block sizes from "NVIDIA's FP4
// format delivers 1.68x speedup"):
//   MX:    E = ceil(log2(max|x| / max_elem)) + 127, clamped to [0, 254];
//          q = RNE_sat(x / 2^(E-127)).
//   NVFP4: s = smallest positive finite E4M3 with max|x| <= 6 g s;
//          q = RNE_sat(x / (g s)) of the exact quotient.
//
// Kernel shape: one CTA quantizes a 128-row x 128-column tile of the bf16 input
// (32 KB).  Each thread owns 16 consecutive elements of a row (32 bytes, two
// 16-byte loads) per pass, 8 threads per row, 4 passes; all eight loads of a
// thread are issued up front.  A 16-element NVFP4 block is one thread's, a
// 32-element MX block two neighbouring lanes' (one shuffle).  Block maxima use
// packed bf16x2 max on the magnitude bits.  The scale bytes of the tile (one or
// two 512-byte tensor-core tiles of 128 rows x 4 scale columns) are assembled in
// shared memory and written out with 16-byte stores.
#pragma once

#include "mx_common.cuh"

namespace mx {

enum { FMT_E4M3 = 0, FMT_E5M2 = 1, FMT_MXFP4 = 2, FMT_NVFP4 = 3, FMT_MXFP6 = 4, FMT_MXFP4_MBS = 5 };

template <int FMT>
struct FmtTraits;
template <>
struct FmtTraits<FMT_E4M3> {
    static constexpr int kBlock = 32, kBits = 8;
    // 448 = 1.75 * 2^8: E = expfield(amax) - 8 + (mantissa7(amax) > 0x60)
    static constexpr int kExpOff = 8, kMantThr = 0x60;
};
template <>
struct FmtTraits<FMT_E5M2> {
    static constexpr int kBlock = 32, kBits = 8;
    static constexpr int kExpOff = 15, kMantThr = 0x60;  // 57344 = 1.75 * 2^15
};
template <>
struct FmtTraits<FMT_MXFP4> {
    static constexpr int kBlock = 32, kBits = 4;
    static constexpr int kExpOff = 2, kMantThr = 0x40;  // 6 = 1.5 * 2^2
};
template <>
struct FmtTraits<FMT_NVFP4> {
    static constexpr int kBlock = 16, kBits = 4;
    static constexpr int kExpOff = 0, kMantThr = 0;
};
template <>
struct FmtTraits<FMT_MXFP4_MBS> {  // E2M1 elements, E8M0 per 16, macro mantissa per 128
    static constexpr int kBlock = 16, kBits = 4;
    static constexpr int kExpOff = 0, kMantThr = 0;
};
template <>
struct FmtTraits<FMT_MXFP6> {  // E3M2 elements
    static constexpr int kBlock = 32, kBits = 6;
    static constexpr int kExpOff = 4, kMantThr = 0x60;  // 28 = 1.75 * 2^4
};

// ------------------------------------------------------------------ scale rules
// MX exponent from the bf16 bit pattern of a block's max |x| (non-negative,
// finite).  amax = 1.m * 2^(f-127) with max_elem = M * 2^k: the smallest e with
// amax <= max_elem * 2^e is f - 127 - k, plus one when 1.m > M.  Zero and bf16
// subnormals land below 0 and clamp to 0; finite inputs never exceed 253.
//
// RULE_OAS (MXFP4 only; page "Unveiling the Potential of Quantization with
// MXFP4", section 2.A, overflow-aware scaling): the block max is mapped into
// (3.5, 7] instead of (3, 6], i.e. the threshold is 7 = 1.75 * 2^2; elements
// above 6 then saturate to 6 as usual.
enum { RULE_OCP = 0, RULE_OAS = 1 };

template <int FMT, int RULE = RULE_OCP>
MX_DEVICE_INLINE int mx_scale_byte(uint32_t amax_bits) {
    using T = FmtTraits<FMT>;
    static_assert(RULE == RULE_OCP || FMT == FMT_MXFP4, "overflow-aware scaling is defined for MXFP4");
    constexpr uint32_t thr = RULE == RULE_OAS ? 0x60u : (uint32_t)T::kMantThr;
    int e = (int)(amax_bits >> 7) - T::kExpOff + (((amax_bits & 0x7Fu) > thr) ? 1 : 0);
    return e < 0 ? 0 : e;
}

// 2^(127 - E) as fp32, E in [0, 253].
MX_DEVICE_INLINE float mx_inv_scale(int E) { return __uint_as_float((uint32_t)(254 - E) << 23); }

// Positive E4M3 code (1..126) -> its value.
MX_DEVICE_INLINE float e4m3_pos_value(uint32_t c) {
    uint32_t e = c >> 3, m = c & 7u;
    return e == 0 ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Does 6 * g * s >= amax hold exactly?  fma rounds once, so the sign of
// fma(6s, g, -amax) is the sign of the exact difference (6s is exact in fp32).
MX_DEVICE_INLINE bool nv_scale_ok(float s, float g, float amax) { return __fmaf_rn(6.0f * s, g, -amax) >= 0.0f; }

// NVFP4 block scale: smallest positive finite E4M3 s with amax <= 6 g s,
// 0 for an all-zero block, 0x7E (448) if none suffices.  t = amax * inv6g is
// within a few ulps of the exact quotient q = amax / (6 g), far less than the
// E4M3 spacing (2^-3 relative, or 2^-9 below 2^-6), so its nearest E4M3 code
// is either the answer c* (the smallest value >= q) or the code just below:
// one exact test of 6 g s >= amax decides.  (For g below ~2^-102, where
// 1/(6g) is no longer that accurate or overflows, the estimate only seeds an
// exact walk up and down the codes.)  The common path has no branch: the
// clamp, the correction and the all-zero case are selects (3-4% of the NVFP4
// quantize's time against early returns and compare-and-set).
MX_DEVICE_INLINE uint32_t nv_block_scale(float amax, float g, float inv6g, const float *val) {
    const float approx = amax * inv6g;
    uint32_t c;
    asm("{\n\t.reg .b16 h;\n\tcvt.rn.satfinite.e4m3x2.f32 h, %1, %1;\n\tcvt.u32.u16 %0, h;\n\t}"
        : "=r"(c)
        : "f"(approx));
    c = min(max(c & 0x7Fu, 1u), 0x7Eu);   // NaN (g not positive) saturates; 0 -> the smallest
    if (inv6g <= 0x1p100f) {
        c += (c < 0x7Eu && !nv_scale_ok(val[c], g, amax)) ? 1u : 0u;
        return amax > 0.0f ? c : 0u;
    } else {
        if (!(amax > 0.0f)) return 0u;
        // bounded by the code range
        while (c < 0x7Eu && !nv_scale_ok(val[c], g, amax)) ++c;
        while (c > 1u && nv_scale_ok(val[c - 1u], g, amax)) --c;
    }
    return c;
}

// ------------------------------------------------------------------ element casts
// Four fp32 -> four fp8 codes (byte i = element i), RNE, saturating.
template <int FMT>
MX_DEVICE_INLINE uint32_t cvt4_fp8(float a0, float a1, float a2, float a3) {
    uint32_t out;
    if (FMT == FMT_E4M3) {
        asm("{\n\t.reg .b16 lo, hi;\n\t"
            "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
            "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
            "mov.b32 %0, {lo, hi};\n\t}"
            : "=r"(out)
            : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
    } else {
        asm("{\n\t.reg .b16 lo, hi;\n\t"
            "cvt.rn.satfinite.e5m2x2.f32 lo, %2, %1;\n\t"
            "cvt.rn.satfinite.e5m2x2.f32 hi, %4, %3;\n\t"
            "mov.b32 %0, {lo, hi};\n\t}"
            : "=r"(out)
            : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
    }
    return out;
}

// Eight fp32 -> eight E2M1 codes packed (element i in nibble i), RNE, saturating.
MX_DEVICE_INLINE uint32_t cvt8_e2m1(const float (&a)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
    return out;
}

// Four fp32 -> four E3M2 codes, one per byte in bits 0-5, RNE, saturating.
MX_DEVICE_INLINE uint32_t cvt4_e3m2(float a0, float a1, float a2, float a3) {
    uint32_t out;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e3m2x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e3m2x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(out)
        : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
    return out & 0x3F3F3F3Fu;
}

// The four 6-bit codes of w's bytes as 24 contiguous bits (byte i at bit 6i).
MX_DEVICE_INLINE uint32_t pack4x6(uint32_t w) {
    const uint32_t x = (w & 0x003F003Fu) | ((w & 0x3F003F00u) >> 2);   // 12-bit pairs in each half
    return (x & 0xFFFu) | ((x >> 4) & 0xFFF000u);
}

// Store the codes of 16 MX elements already divided by their block scale
// (row `row`, columns col .. col+15, col % 16 == 0).  FP8: one byte each; FP6:
// code k of a row at bits 6k .. 6k+5 of the row's little-endian bit string
// (16 codes in 12 bytes, the packed form the tensor map's 16 x U6 type reads);
// FP4: two per byte, the even element in the low nibble.
template <int FMT>
MX_DEVICE_INLINE void store_mx_codes16(uint8_t *__restrict__ codes, int64_t row, int64_t K, int64_t col,
                                       const float (&f)[16]) {
    using T = FmtTraits<FMT>;
    if (T::kBits == 8) {
        uint4 q;
        q.x = cvt4_fp8<FMT>(f[0], f[1], f[2], f[3]);
        q.y = cvt4_fp8<FMT>(f[4], f[5], f[6], f[7]);
        q.z = cvt4_fp8<FMT>(f[8], f[9], f[10], f[11]);
        q.w = cvt4_fp8<FMT>(f[12], f[13], f[14], f[15]);
        *reinterpret_cast<uint4 *>(codes + row * K + col) = q;
    } else if (T::kBits == 6) {
        const uint32_t t0 = pack4x6(cvt4_e3m2(f[0], f[1], f[2], f[3]));
        const uint32_t t1 = pack4x6(cvt4_e3m2(f[4], f[5], f[6], f[7]));
        const uint32_t t2 = pack4x6(cvt4_e3m2(f[8], f[9], f[10], f[11]));
        const uint32_t t3 = pack4x6(cvt4_e3m2(f[12], f[13], f[14], f[15]));
        // 12 bytes at a 4-byte aligned offset (K % 32 == 0, col % 16 == 0)
        uint32_t *p = reinterpret_cast<uint32_t *>(codes + row * (K / 4 * 3) + col / 4 * 3);
        p[0] = t0 | (t1 << 24);
        p[1] = (t1 >> 8) | (t2 << 16);
        p[2] = (t2 >> 16) | (t3 << 8);
    } else {
        const float(&f0)[8] = *reinterpret_cast<const float(*)[8]>(&f[0]);
        const float(&f1)[8] = *reinterpret_cast<const float(*)[8]>(&f[8]);
        *reinterpret_cast<uint2 *>(codes + row * (K / 2) + col / 2) = make_uint2(cvt8_e2m1(f0), cvt8_e2m1(f1));
    }
}

MX_DEVICE_INLINE float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
MX_DEVICE_INLINE float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E2M1 magnitude of code c (0..7).
MX_DEVICE_INLINE float e2m1_mag(uint32_t c) {
    return c < 2u ? 0.5f * (float)c : __uint_as_float(((c >> 1) + 126u) << 23) * (1.0f + 0.5f * (float)(c & 1u));
}

// NVFP4 elements: codes of x / (g s) for 16 values, the exact RNE of the real
// quotient q.  r_lo <= 1/(g s) <= r_hi.  lo = x * r_lo rounded toward zero
// bounds |q| from below; hi = x * r_hi (1 + 2^-21) (the factor rounded up),
// also rounded toward zero, bounds it from above: the product exceeds |q| by
// a relative 2^-21, more than the 2^-23 that rounding toward zero can take
// off.  Both are sign-symmetric, so each pair of elements takes one packed
// f32x2 multiply per bound.  RNE is monotone, so the code lies between lo's
// and hi's; the bracket is a few ulps wide, so they differ by at most one
// step, and only when a midpoint m between the two codes lies inside it.
// Such an element (typically a tie: bf16 inputs divided by a short scale often
// land exactly on a midpoint) is settled by the sign of |x| - g*s*m, which one
// fma computes exactly (s*m is exact in fp32); a tie goes to the even code.

// Midpoint between E2M1 magnitudes c and c + 1 (c = 0..6).
MX_DEVICE_INLINE float e2m1_mid(uint32_t c) {
    return c < 4u ? 0.25f + 0.5f * (float)c : (c < 6u ? (float)c - 1.5f : 5.0f);
}

// Settle the elements of one packed word (8 codes) whose bracket straddles a
// midpoint.  diff has a nonzero nibble where lo's and hi's magnitudes differ;
// w0..w3 hold the word's 8 bf16 inputs (element 2j in the low half of wj).
MX_DEVICE_INLINE uint32_t nv_settle(uint32_t code, uint32_t diff, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                    float g, float s, float sc) {
    while (diff != 0u) {
        const int nib = (__ffs(diff) - 1) >> 2;
        diff &= ~(0xFu << (4 * nib));
        const int j = nib >> 1;
        const uint32_t wj = j == 0 ? w0 : (j == 1 ? w1 : (j == 2 ? w2 : w3));
        const float ax = fabsf((nib & 1) ? __uint_as_float(wj & 0xFFFF0000u) : __uint_as_float(wj << 16)) * sc;
        const uint32_t c = (code >> (4 * nib)) & 7u;                  // lo's magnitude, < hi's <= 7
        const float d = __fmaf_rn(-g, s * e2m1_mid(c), ax);           // sign(|x| - g*s*mid)
        if (d > 0.0f || (d == 0.0f && (c & 1u))) code += 1u << (4 * nib);
    }
    return code;
}

// lo / hi brackets of 16 values held as 8 packed pairs (see above).
MX_DEVICE_INLINE void bracket16(const uint64_t (&P)[8], float r_lo, float r_hi, float (&lo)[16], float (&hi)[16]) {
    const float r_up = __fmul_ru(r_hi, 1.0f + 0x1p-21f);
    const uint64_t RL = pk2(r_lo, r_lo), RU = pk2(r_up, r_up);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        upk2(mul2_rz(P[i], RL), lo[2 * i], lo[2 * i + 1]);
        upk2(mul2_rz(P[i], RU), hi[2 * i], hi[2 * i + 1]);
    }
}

// sc: a power of two the values are multiplied by (exactly) before the
// division, 1 unless g is so small that 1/g would overflow (see the kernel).
MX_DEVICE_INLINE void nv_codes16(const uint4 &v0, const uint4 &v1, float g, float s, float r_lo, float r_hi,
                                 uint32_t &out0, uint32_t &out1, float sc) {
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint64_t P[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) P[i] = pk2(bf16lo(w[i]), bf16hi(w[i]));
    if (sc != 1.0f) {
        const uint64_t SC = pk2(sc, sc);
#pragma unroll
        for (int i = 0; i < 8; ++i) P[i] = mul2(P[i], SC);
    }
    float lo[16], hi[16];
    bracket16(P, r_lo, r_hi, lo, hi);
    const float(&lo0)[8] = *reinterpret_cast<const float(*)[8]>(&lo[0]);
    const float(&lo1)[8] = *reinterpret_cast<const float(*)[8]>(&lo[8]);
    const float(&hi0)[8] = *reinterpret_cast<const float(*)[8]>(&hi[0]);
    const float(&hi1)[8] = *reinterpret_cast<const float(*)[8]>(&hi[8]);
    uint32_t c0 = cvt8_e2m1(lo0), c1 = cvt8_e2m1(lo1);
    const uint32_t d0 = (c0 ^ cvt8_e2m1(hi0)) & 0x77777777u, d1 = (c1 ^ cvt8_e2m1(hi1)) & 0x77777777u;
    if ((d0 | d1) != 0u) {
        c0 = nv_settle(c0, d0, w[0], w[1], w[2], w[3], g, s, sc);
        c1 = nv_settle(c1, d1, w[4], w[5], w[6], w[7], g, s, sc);
    }
    out0 = c0;
    out1 = c1;
}

MX_DEVICE_INLINE void unpack16(const uint4 &v0, const uint4 &v1, float (&x)[16]) {
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = bf16lo(w[i]);
        x[2 * i + 1] = bf16hi(w[i]);
    }
}

// E2M1 codes of 16 fp32 values x / (g s): the bracket of nv_codes16 on fp32
// inputs (r_lo <= 1/(g s) <= r_hi; g * s * mid must be exact for the settle).
MX_DEVICE_INLINE uint32_t nv_settle_f32(uint32_t code, uint32_t diff, const float *x8, float g, float s) {
    while (diff != 0u) {
        const int nib = (__ffs(diff) - 1) >> 2;
        diff &= ~(0xFu << (4 * nib));
        float ax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i == nib) ax = fabsf(x8[i]);
        const uint32_t c = (code >> (4 * nib)) & 7u;
        const float d = __fmaf_rn(-g, s * e2m1_mid(c), ax);
        if (d > 0.0f || (d == 0.0f && (c & 1u))) code += 1u << (4 * nib);
    }
    return code;
}

MX_DEVICE_INLINE void nv_codes16_f32(const float (&x)[16], float g, float s, float r_lo, float r_hi,
                                     uint32_t &out0, uint32_t &out1) {
    uint64_t P[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) P[i] = pk2(x[2 * i], x[2 * i + 1]);
    float lo[16], hi[16];
    bracket16(P, r_lo, r_hi, lo, hi);
    const float(&lo0)[8] = *reinterpret_cast<const float(*)[8]>(&lo[0]);
    const float(&lo1)[8] = *reinterpret_cast<const float(*)[8]>(&lo[8]);
    const float(&hi0)[8] = *reinterpret_cast<const float(*)[8]>(&hi[0]);
    const float(&hi1)[8] = *reinterpret_cast<const float(*)[8]>(&hi[8]);
    uint32_t c0 = cvt8_e2m1(lo0), c1 = cvt8_e2m1(lo1);
    const uint32_t d0 = (c0 ^ cvt8_e2m1(hi0)) & 0x77777777u, d1 = (c1 ^ cvt8_e2m1(hi1)) & 0x77777777u;
    if ((d0 | d1) != 0u) {
        c0 = nv_settle_f32(c0, d0, &x[0], g, s);
        c1 = nv_settle_f32(c1, d1, &x[8], g, s);
    }
    out0 = c0;
    out1 = c1;
}

// Per-CTA tables for NVFP4, indexed by positive E4M3 code c (1..126):
// the value s, and 1/s rounded down and up.
struct NvTables {
    float val[128];
    float inv_lo[128];
    float inv_hi[128];
};

// ------------------------------------------------------------------ loads / stores
MX_DEVICE_INLINE uint4 ldg_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// ------------------------------------------------------------------ kernels
constexpr int kQTileRows = 128;
constexpr int kQTileCols = 128;
constexpr int kQThreads = 256;

// Largest bf16 magnitude (as its bit pattern) among the 16 values of v0, v1.
// Per half: a value whose magnitude is max(|a|, |b|) (its sign is the XOR of
// the inputs' signs, which the caller masks off once at the end).
MX_DEVICE_INLINE uint32_t bf16x2_maxabs(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

MX_DEVICE_INLINE uint32_t absmax16(const uint4 &v0, const uint4 &v1) {
    const uint32_t r = bf16x2_maxabs(bf16x2_maxabs(bf16x2_maxabs(v0.x, v0.y), bf16x2_maxabs(v0.z, v0.w)),
                                     bf16x2_maxabs(bf16x2_maxabs(v1.x, v1.y), bf16x2_maxabs(v1.z, v1.w)));
    const uint32_t rb = r & 0x7FFF7FFFu;
    return max(rb & 0xFFFFu, rb >> 16);
}

// NVFP4 per-tensor constants of the quantize, formed once per CTA from g: the
// bracket reciprocals of 1/g rounded down and up and 1/(6g).  Below 2^-100,
// 1/g loses accuracy or overflows: the values are then divided as x * 2^64 by
// g * 2^64 instead (both exact; every quotient is unchanged), sc = 2^64.
struct NvScale {
    float g, rg_lo, rg_hi, inv6g, sc;
};
MX_DEVICE_INLINE NvScale nv_scale_setup(float g) {
    NvScale n;
    n.sc = 1.0f;
    if (g < 0x1p-100f) {
        n.sc = 0x1p64f;
        g *= n.sc;
    }
    n.g = g;
    n.rg_lo = __frcp_rd(g);
    n.rg_hi = __frcp_ru(g);
    n.inv6g = 1.0f / (6.0f * g);
    return n;
}
// g of an NVFP4 tensor from *src: g itself, or (from_amax) amax(|x|) with
// g = RU(amax / (6 * 448)), 1 for an all-zero tensor.
MX_DEVICE_INLINE float nv_g_from(const float *src, int from_amax) {
    float g = *src;
    if (from_amax) g = g > 0.0f ? __fdiv_ru(g, 2688.0f) : 1.0f;
    return g;
}
// Entry c (0..127) of the per-CTA NVFP4 tables.
MX_DEVICE_INLINE void nv_tables_fill(NvTables *nvt, uint32_t c) {
    const float v = (c == 0u || c == 127u) ? 0.0f : e4m3_pos_value(c);
    nvt->val[c] = v;
    nvt->inv_lo[c] = v > 0.0f ? __frcp_rd(v) : 0.0f;
    nvt->inv_hi[c] = v > 0.0f ? __frcp_ru(v) : 0.0f;
}

// One 16-element segment of a 128 x 128 quantize tile: values (v0, v1) of
// global row `row` (tile row rl), columns col .. col + 15 (tile columns cl ..
// cl + 15).  Stores the segment's codes when row and columns exist, and the
// block's scale byte into the tile's 512-byte tensor-core chunks in sf_tile
// (0 for padding).  A 32-element MX block spans lanes lane and lane ^ 1, which
// must call together (one shuffle).
template <int FMT, int RULE>
MX_DEVICE_INLINE void quantize_seg16(const uint4 &v0, const uint4 &v1, int64_t row, int64_t M, int64_t col, int64_t K,
                                     int64_t col0, int rl, int cl, int lane, const NvScale &ns,
                                     const NvTables *__restrict__ nvt, uint8_t *__restrict__ codes,
                                     uint8_t *__restrict__ sf_tile) {
    using T = FmtTraits<FMT>;
    const bool col_ok = col < K;   // K % 16 == 0: all 16 or none
    const bool ok = row < M && col_ok;
    const int jb = cl / T::kBlock;  // block index inside the tile row
    uint32_t m = absmax16(v0, v1);
    if (T::kBlock == 32) m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    uint32_t sbyte;
    if (FMT == FMT_NVFP4) {
        sbyte = nv_block_scale(__uint_as_float(m << 16) * ns.sc, ns.g, ns.inv6g, nvt->val);
        if (ok) {
            uint32_t q0, q1;
            // r_lo <= 1/(g s) <= r_hi: products of one-sided bounds, rounded outward.
            // An all-zero block has s = 0 and both bounds 0, so its products are
            // the zeros themselves and its codes their signs (0x0 / 0x8).
            const float r_lo = __fmul_rd(ns.rg_lo, nvt->inv_lo[sbyte]);
            const float r_hi = __fmul_ru(ns.rg_hi, nvt->inv_hi[sbyte]);
            nv_codes16(v0, v1, ns.g, nvt->val[sbyte], r_lo, r_hi, q0, q1, ns.sc);
            *reinterpret_cast<uint2 *>(codes + row * (K / 2) + col / 2) = make_uint2(q0, q1);
        }
    } else {
        const int E = mx_scale_byte<FMT, RULE>(m);
        sbyte = (uint32_t)E;
        if (ok) {
            const float inv = mx_inv_scale(E);
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            float f[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                f[2 * e] = bf16lo(w[e]) * inv;
                f[2 * e + 1] = bf16hi(w[e]) * inv;
            }
            store_mx_codes16<FMT>(codes, row, K, col, f);
        }
    }
    // Scale byte of (rl, jb) inside the tile's 512-byte tensor-core tiles.
    const bool owner = T::kBlock == 16 || (lane & 1) == 0;
    if (owner) {
        const int64_t jglob = col0 / T::kBlock + jb;
        if (!(row < M) || jglob >= K / T::kBlock) sbyte = 0u;   // padding bytes are 0
        sf_tile[(jb >> 2) * 512 + (rl & 31) * 16 + (rl >> 5) * 4 + (jb & 3)] = (uint8_t)sbyte;
    }
}

// Bytes of a 128 x 128 tile's scale chunks (one or two 512-byte tensor-core tiles).
template <int FMT>
__host__ __device__ constexpr int quantize_sf_bytes() {
    return kQTileRows * (kQTileCols / FmtTraits<FMT>::kBlock);
}

// Write a tile's scale chunks from shared memory (16 bytes per thread t <
// bytes / 16): tile (band, tile_x) owns the consecutive chunks from
// band * sf_tiles_k + tile_x * chunks, cut at the band's last chunk.
template <int FMT>
MX_DEVICE_INLINE void store_sf_chunks(const uint8_t *sf_tile, uint8_t *__restrict__ scales, int64_t band,
                                      int64_t tile_x, int64_t sf_tiles_k, int t) {
    constexpr int kChunks = quantize_sf_bytes<FMT>() / 512;
    const int64_t chunk0 = band * sf_tiles_k + tile_x * kChunks;
    const int64_t max_chunk = band * sf_tiles_k + sf_tiles_k;   // past this band's last tile
    if (t < quantize_sf_bytes<FMT>() / 16) {
        const int c = t / 32;
        if (chunk0 + c < max_chunk) {
            const uint4 val = *reinterpret_cast<const uint4 *>(sf_tile + t * 16);
            *reinterpret_cast<uint4 *>(scales + chunk0 * 512 + t * 16) = val;
        }
    }
}

// ROWS rows x 128 columns of src quantized by NT threads (t = 0 .. NT - 1,
// whole warps): 8 threads per row, 16 elements per thread per pass, ROWS /
// (NT / 8) passes.  tile_load issues every load of the rows (two 16-byte loads
// per pass) into registers; tile_quantize then stores the codes and writes each
// block's scale byte into the 128-row tile's scale chunks in sf_tile (shared
// memory, quantize_sf_bytes<FMT>() bytes; rows are placed by their row index
// inside the 128-row band, rl0 being that of the first).
template <int NT, int ROWS = kQTileRows>
struct TileRegs {
    static_assert(NT % 32 == 0 && NT >= 32 && ROWS % (NT / 8) == 0 && ROWS <= kQTileRows, "whole warps and passes");
    static constexpr int kRowsPerPass = NT / 8;
    static constexpr int kPasses = ROWS / kRowsPerPass;
    uint4 v[kPasses][2];
};

template <int NT, int ROWS>
MX_DEVICE_INLINE void tile_load(TileRegs<NT, ROWS> &r, const uint16_t *__restrict__ src, int64_t M, int64_t K,
                                int64_t ld, int64_t row0, int64_t col0, int t) {
    using R = TileRegs<NT, ROWS>;
    const int lane = t & 31, warp = t >> 5;
    const int64_t col = col0 + (lane & 7) * 16;
#pragma unroll
    for (int i = 0; i < R::kPasses; ++i) {
        const int64_t row = row0 + i * R::kRowsPerPass + warp * 4 + (lane >> 3);
        if (row < M && col < K) {
            const uint16_t *p = src + row * ld + col;
            r.v[i][0] = ldg_stream(p);
            r.v[i][1] = ldg_stream(p + 8);
        } else {
            r.v[i][0] = r.v[i][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

template <int FMT, int NT, int ROWS>
MX_DEVICE_INLINE void tile_quantize(const TileRegs<NT, ROWS> &r, int64_t M, int64_t K, int64_t band_row0, int rl0,
                                    int64_t col0, const NvScale &ns, const NvTables *nvt,
                                    uint8_t *__restrict__ codes, uint8_t *sf_tile, int t) {
    using R = TileRegs<NT, ROWS>;
    const int lane = t & 31, warp = t >> 5;
    const int cl = (lane & 7) * 16;
#pragma unroll
    for (int i = 0; i < R::kPasses; ++i) {
        const int rl = rl0 + i * R::kRowsPerPass + warp * 4 + (lane >> 3);
        quantize_seg16<FMT, RULE_OCP>(r.v[i][0], r.v[i][1], band_row0 + rl, M, col0 + cl, K, col0, rl, cl, lane, ns,
                                      nvt, codes, sf_tile);
    }
}

// amax(|x|) of a whole bf16 tensor of at most kTinyAmaxElements elements,
// computed by every thread of one CTA (which all receive it): each thread
// issues the loads of its four 16-element segments (row-aligned, as the
// quantize tiles and amax_kernel cut them) at once, and the segment maxima
// reduce exactly as in amax_kernel, so the value is the one its pre-pass
// would store.  For an NVFP4 quantize of a tensor this small, every CTA
// computing the maximum itself costs one read of at most 32 KB from L2, less
// than the two kernels of the pre-pass (the slot reset and amax_kernel).
constexpr int64_t kTinyAmaxElements = 16 * 4 * kQThreads;   // 16384
MX_DEVICE_INLINE float tiny_tensor_amax(const uint16_t *__restrict__ src, int64_t M, int64_t K, int64_t ld) {
    __shared__ uint32_t red[kQThreads / 32];
    const int64_t segs_row = K / 16, n = M * segs_row;   // K % 16 == 0
    uint4 v[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t sg = threadIdx.x + (int64_t)i * kQThreads;
        if (sg < n) {
            const uint16_t *p = src + (sg / segs_row) * ld + (sg % segs_row) * 16;
            v[i][0] = ldg_stream(p);
            v[i][1] = ldg_stream(p + 8);
        } else {
            v[i][0] = v[i][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) m = max(m, absmax16(v[i][0], v[i][1]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = m;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kQThreads / 32; ++w) m = max(m, red[w]);
    return __uint_as_float(m << 16);   // bf16 magnitude -> fp32 (0 for an all-zero tensor)
}

// src bf16 [M x K] (row pitch ld).  codes / scales as in mx.h.  sf_tiles_k =
// ceil((K / block) / 4) 512-byte tiles per 128-row band.  NVFP4: *gscale_in
// is g, or amax(|src|) when g_from_amax (then g = RU(amax / 2688), 1 for 0);
// SELF_AMAX (tensors of at most kTinyAmaxElements elements): every CTA
// computes amax(|src|) itself, gscale_in unused (a separate instantiation, so
// that the common kernel's code is unchanged).  If gscale_out != nullptr, CTA
// 0 also stores g there.  band_ready (nullable):
// each CTA adds one to its 128-row band's counter once its codes and scales
// are written (release, gpu scope).  clear (nullable): n_clear words that CTA
// 0 zeroes once the previous kernel in the stream has completed (the partial-
// sum counters of the fused call's GEMM, which runs after this grid).
// CTAs per SM that the register allocation of quantize_kernel<FMT> targets,
// chosen by timing 2^28-element inputs: the FP8 and FP4 MX casts run fastest
// with the registers left free (1), NVFP4 with four resident CTAs (the
// bracket's working set), MXFP6 with five.
template <int FMT>
constexpr int quantize_min_blocks() {
    return FMT == FMT_NVFP4 ? 4 : (FMT == FMT_MXFP6 ? 5 : 1);
}

template <int FMT, int RULE = RULE_OCP, bool SELF_AMAX = false>
__global__ void __launch_bounds__(kQThreads, quantize_min_blocks<FMT>()) quantize_kernel(const uint16_t *__restrict__ src, int64_t M, int64_t K,
                                                             int64_t ld, uint8_t *__restrict__ codes,
                                                             uint8_t *__restrict__ scales, int64_t sf_tiles_k,
                                                             const float *__restrict__ gscale_in,
                                                             float *__restrict__ gscale_out, int g_from_amax,
                                                             uint32_t *__restrict__ band_ready,
                                                             uint32_t *__restrict__ clear, int n_clear) {
    constexpr int kPasses = kQTileRows / 32;               // 32 rows per pass (8 warps x 4 rows)
    __shared__ __align__(16) uint8_t sf_tile[quantize_sf_bytes<FMT>()];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row0 = (int64_t)blockIdx.y * kQTileRows;
    const int64_t col0 = (int64_t)blockIdx.x * kQTileCols;
    const int cl = (lane & 7) * 16;                 // first of this lane's 16 columns inside the tile
    const int64_t col = col0 + cl;

    NvScale ns{1.0f, 1.0f, 1.0f, 1.0f, 1.0f};
    __shared__ NvTables nvt;
    // src and g may come from the previous kernel in the stream
    griddep_wait();
    // Every CTA of this grid has started once all have passed here, so the next
    // kernel in the stream may take SMs as this grid's CTAs leave them (it still
    // waits for this grid's completion before reading anything).
    griddep_launch_dependents();
    if (clear != nullptr && blockIdx.x == 0 && blockIdx.y == 0)
        for (int i = threadIdx.x; i < n_clear; i += blockDim.x) clear[i] = 0u;
    if (FMT == FMT_NVFP4) {
        float g;
        if (SELF_AMAX) {
            const float amax = tiny_tensor_amax(src, M, K, ld);
            g = nv_g_from(&amax, 1);
        } else {
            g = nv_g_from(gscale_in, g_from_amax);
        }
        if (gscale_out != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *gscale_out = g;
        ns = nv_scale_setup(g);
        if (threadIdx.x < 128) nv_tables_fill(&nvt, threadIdx.x);
        __syncthreads();
    }

    uint4 v[kPasses][2];
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
        const int rl = i * 32 + warp * 4 + (lane >> 3);
        const int64_t row = row0 + rl;
        if (row < M && col < K) {
            const uint16_t *p = src + row * ld + col;
            v[i][0] = ldg_stream(p);
            v[i][1] = ldg_stream(p + 8);
        } else {
            v[i][0] = v[i][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }

#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
        const int rl = i * 32 + warp * 4 + (lane >> 3);
        quantize_seg16<FMT, RULE>(v[i][0], v[i][1], row0 + rl, M, col, K, col0, rl, cl, lane, ns, &nvt, codes,
                                  sf_tile);
    }
    __syncthreads();
    store_sf_chunks<FMT>(sf_tile, scales, blockIdx.y, blockIdx.x, sf_tiles_k, threadIdx.x);
    if (band_ready != nullptr) {
        // a GEMM of the same fused call reads this tile with TMA as soon as its
        // band's count is complete (one count per CTA of the band)
        fence_proxy_async_global();
        __syncthreads();
        if (threadIdx.x == 0) red_release_gpu_add(band_ready + blockIdx.y, 1u);
    }
}

// ------------------------------------------------------------------ MXFP4 with macro-block scaling
// Page "Unveiling the Potential of Quantization with MXFP4", section B (Macro
// Block Scaling), static variant: per 1x128 macro block a factor 1 + m/256
// with m chosen from the block max alpha (e = floor(log2(alpha / 6)); m the
// smallest byte with alpha <= 6 (256 + m) 2^(e-8), 0 if none), then E2M1
// elements in 1x16 blocks with E8M0 scales applied to x / (1 + m/256).
//
// With alpha = M_a 2^(ea-7), M_a in [128, 255] (bf16 mantissa with its
// leading one; subnormals normalised), alpha / 2^(e-8) is the integer
// A = 16 M_a (M_a < 192) or 8 M_a, and m = ceil(A / 6) - 256.
MX_DEVICE_INLINE void bf16_normalise(uint32_t bits, uint32_t &mant, int &ex) {
    const uint32_t ef = (bits >> 7) & 0xFFu, fr = bits & 0x7Fu;
    if (ef != 0u) {
        mant = 128u + fr;
        ex = (int)ef - 127;
    } else {
        // subnormal: fr != 0 (the caller handles zero); 8 - bit length of fr shifts
        const int sh = __clz(fr) - 24;
        mant = fr << sh;
        ex = -126 - sh;
    }
}

MX_DEVICE_INLINE uint32_t mbs_static_mantissa(uint32_t alpha_bits) {
    if (alpha_bits == 0u) return 0u;
    uint32_t ma;
    int ea;
    bf16_normalise(alpha_bits, ma, ea);
    const uint32_t A = ma < 192u ? 16u * ma : 8u * ma;   // in [1536, 3072)
    const uint32_t m = (A + 5u) / 6u - 256u;
    return m > 255u ? 0u : m;
}

// Smallest E in [0, 254] with amax_b <= 6 (256 + m) 2^(E - 135): with
// amax_b = M_b 2^(eb-7), M_b in [128, 255], the condition reads
// M_b 2^(eb + 128 - E) <= 6 (256 + m), whose largest shift is 2, 3 or 4.
MX_DEVICE_INLINE uint32_t mbs_block_exponent(uint32_t amax_bits, uint32_t m) {
    if (amax_bits == 0u) return 0u;
    uint32_t mb;
    int eb;
    bf16_normalise(amax_bits, mb, eb);
    const uint32_t km = 6u * (256u + m);
    const int d = (mb << 4) <= km ? 4 : ((mb << 3) <= km ? 3 : 2);
    const int E = eb + 128 - d;
    return (uint32_t)(E < 0 ? 0 : (E > 254 ? 254 : E));
}

// Per-CTA reciprocals of k = 256 + m (m = 0..255), rounded down and up.
struct MbsTables {
    float rcp_lo[256];
    float rcp_hi[256];
};

// Same tile structure as quantize_kernel: a 128-column tile row is exactly one
// macro block, spread over 8 lanes (16 elements each, one base block per lane).
// Elements: v = x 2^(135-E) (two exact power-of-two products), code = RNE of
// v / (256 + m) on E2M1 by the directed-rounding bracket, ties settled exactly.
// macro_out: the [M][K/128] macro mantissa bytes (K % 128 == 0).
__global__ void __launch_bounds__(kQThreads) quantize_mbs_kernel(const uint16_t *__restrict__ src, int64_t M,
                                                                 int64_t K, int64_t ld, uint8_t *__restrict__ codes,
                                                                 uint8_t *__restrict__ scales, int64_t sf_tiles_k,
                                                                 uint8_t *__restrict__ macro_out) {
    constexpr int kBlocksPerRow = kQTileCols / 16;
    constexpr int kSfBytes = kQTileRows * kBlocksPerRow;   // 1024
    constexpr int kPasses = kQTileRows / 32;
    __shared__ __align__(16) uint8_t sf_tile[kSfBytes];
    __shared__ MbsTables tab;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row0 = (int64_t)blockIdx.y * kQTileRows;
    const int64_t col0 = (int64_t)blockIdx.x * kQTileCols;
    const int cl = (lane & 7) * 16;
    const int64_t col = col0 + cl;
    const int jb = cl / 16;
    {
        const float k = (float)(256 + threadIdx.x);   // kQThreads == 256
        tab.rcp_lo[threadIdx.x] = __frcp_rd(k);
        tab.rcp_hi[threadIdx.x] = __frcp_ru(k);
    }
    griddep_wait();
    __syncthreads();

    uint4 v[kPasses][2];
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
        const int rl = i * 32 + warp * 4 + (lane >> 3);
        const int64_t row = row0 + rl;
        if (row < M) {
            const uint16_t *p = src + row * ld + col;
            v[i][0] = ldg_stream(p);
            v[i][1] = ldg_stream(p + 8);
        } else {
            v[i][0] = v[i][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }

#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
        const int rl = i * 32 + warp * 4 + (lane >> 3);
        const int64_t row = row0 + rl;
        const bool ok = row < M;
        const uint32_t amax = absmax16(v[i][0], v[i][1]);
        uint32_t alpha = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        alpha = max(alpha, __shfl_xor_sync(0xffffffffu, alpha, 2));
        alpha = max(alpha, __shfl_xor_sync(0xffffffffu, alpha, 4));
        const uint32_t m = mbs_static_mantissa(alpha);
        const uint32_t E = mbs_block_exponent(amax, m);
        if (ok) {
            // The quotient is x / D, D = (256 + m) 2^(E - 135).  Its bracket
            // reciprocals are 1/(256 + m) from the tables times 2^(135 - E),
            // formed with outward rounding (two power-of-two factors, since
            // 135 - E spans [-119, 135]); the settle compares |x| with
            // 2^(E - 135) * ((256 + m) mid) inside one exact fma.
            const int t = 135 - (int)E, t1 = t / 2, t2 = t - t / 2;
            const float p1 = __uint_as_float((uint32_t)(127 + t1) << 23), p2 = __uint_as_float((uint32_t)(127 + t2) << 23);
            const float r_lo = __fmul_rd(__fmul_rd(tab.rcp_lo[m], p1), p2);
            const float r_hi = __fmul_ru(__fmul_ru(tab.rcp_hi[m], p1), p2);
            // 2^(E - 135) as an fp32 (subnormal below E = 9, exact down to 2^-149)
            const float d2 = E >= 9u ? __uint_as_float((uint32_t)(E - 8u) << 23)
                                     : __uint_as_float(1u << (E + 14u));
            float x[16];
            unpack16(v[i][0], v[i][1], x);
            uint32_t q0, q1;
            nv_codes16_f32(x, d2, (float)(256u + m), r_lo, r_hi, q0, q1);
            *reinterpret_cast<uint2 *>(codes + row * (K / 2) + col / 2) = make_uint2(q0, q1);
            if ((lane & 7) == 0) macro_out[row * (K / 128) + blockIdx.x] = (uint8_t)m;
        }
        sf_tile[(jb >> 2) * 512 + (rl & 31) * 16 + (rl >> 5) * 4 + (jb & 3)] = ok ? (uint8_t)E : (uint8_t)0;
    }
    // the macro section's padding to 16 bytes is zero, as every padding byte
    if (blockIdx.x == 0 && blockIdx.y == 0) {
        const int64_t n = M * (K / 128), pad = ((n + 15) & ~(int64_t)15) - n;
        if (threadIdx.x < pad) macro_out[n + threadIdx.x] = 0;
    }
    __syncthreads();
    const int64_t chunk0 = (int64_t)blockIdx.y * sf_tiles_k + (int64_t)blockIdx.x * 2;
    if (threadIdx.x < kSfBytes / 16) {
        const uint4 val = *reinterpret_cast<const uint4 *>(sf_tile + threadIdx.x * 16);
        *reinterpret_cast<uint4 *>(scales + chunk0 * 512 + threadIdx.x * 16) = val;
    }
    griddep_launch_dependents();
}

// ------------------------------------------------------------------ MXFP4 with dynamic macro-block scaling
// Same storage and per-m quantization as quantize_mbs_kernel; the macro
// mantissa of each 1x128 macro block is the byte m in [0, 255] whose
// quantization of the block has the smallest sum of squared errors
// sum_i (x_i - xhat_i)^2, the terms (exact in fp64) added in element order with
// round-to-nearest fp64 additions; ties go to the smallest m (page "Unveiling
// the Potential of Quantization with MXFP4", section 2.B: the dynamic variant's
// factor minimises the error).
//
// One CTA of 256 threads per macro block: thread t scores m = t, sequentially
// over the 128 elements (so its sum is rounded exactly as the definition says),
// then a (error, m) minimum over the CTA picks m, and threads 0..63 write the
// block's codes, 0..7 its base-block exponents, thread 0 its macro byte.  The
// element decision is exact: |x| against each E2M1 midpoint times the divisor
// (256 + m) 2^(E - 135), products of at most 12 significant bits.  The scale
// buffer (tiles and macro section) is cleared by the host first, so padding
// stays zero.
MX_DEVICE_INLINE uint32_t mbs_dyn_code(double a, double denom) {
    const double mids[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
    uint32_t c = 0;
#pragma unroll
    for (int k = 0; k < 7; ++k) {
        const double t = __dmul_rn(mids[k], denom);
        if (a > t) c = (uint32_t)k + 1u;
        else {
            if (a == t) c = (k & 1) ? (uint32_t)k + 1u : (uint32_t)k;   // tie: the even code
            break;
        }
    }
    return c;
}

__global__ void __launch_bounds__(256) quantize_mbs_dynamic_kernel(const uint16_t *__restrict__ src, int64_t M,
                                                                  int64_t K, int64_t ld,
                                                                  uint8_t *__restrict__ codes,
                                                                  uint8_t *__restrict__ scales, int64_t sf_tiles_k,
                                                                  uint8_t *__restrict__ macro_out) {
    __shared__ double xs[128];
    __shared__ uint32_t amax_bits[8];
    __shared__ double red_e[8];
    __shared__ uint32_t red_m[8];
    __shared__ uint32_t chosen;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t row = blockIdx.y, mb = blockIdx.x;
    const uint16_t *x = src + row * ld + mb * 128;
    griddep_wait();
    if (t < 128) {
        xs[t] = (double)__uint_as_float((uint32_t)x[t] << 16);
        // base-block maxima of the magnitude bits (16 lanes per block)
        uint32_t mbits = (uint32_t)x[t] & 0x7FFFu;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mbits = max(mbits, __shfl_xor_sync(0xffffffffu, mbits, o));
        if ((t & 15) == 0) amax_bits[t >> 4] = mbits;
    }
    __syncthreads();
    // score m = t
    const uint32_t m = (uint32_t)t;
    double sse = 0.0;
    for (int jb = 0; jb < 8; ++jb) {
        const uint32_t E = mbs_block_exponent(amax_bits[jb], m);
        const double denom = ldexp((double)(256u + m), (int)E - 135);
        for (int i = 0; i < 16; ++i) {
            const double v = xs[jb * 16 + i];
            const double a = fabs(v);
            const uint32_t c = mbs_dyn_code(a, denom);
            const double mag = __dmul_rn((double)e2m1_mag(c), denom);
            const double d = __dsub_rn(a, mag);    // |x - xhat| (same sign on both)
            sse = __dadd_rn(sse, __dmul_rn(d, d));
        }
    }
    // (error, m) minimum: within the warp, then over the 8 warps
    uint32_t bm = m;
    double be = sse;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double oe = __shfl_xor_sync(0xffffffffu, be, o);
        const uint32_t om = __shfl_xor_sync(0xffffffffu, bm, o);
        if (oe < be || (oe == be && om < bm)) {
            be = oe;
            bm = om;
        }
    }
    if (lane == 0) {
        red_e[warp] = be;
        red_m[warp] = bm;
    }
    __syncthreads();
    if (t == 0) {
        double e = red_e[0];
        uint32_t mm = red_m[0];
        for (int w = 1; w < 8; ++w)
            if (red_e[w] < e || (red_e[w] == e && red_m[w] < mm)) {
                e = red_e[w];
                mm = red_m[w];
            }
        chosen = mm;
        macro_out[row * (K / 128) + mb] = (uint8_t)mm;
    }
    __syncthreads();
    const uint32_t mc = chosen;
    if (t < 64) {
        // elements 2t and 2t + 1 (one byte of codes)
        const int jb = (2 * t) >> 4;
        const uint32_t E = mbs_block_exponent(amax_bits[jb], mc);
        const double denom = ldexp((double)(256u + mc), (int)E - 135);
        uint32_t byte = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const double v = xs[2 * t + h];
            const uint32_t c = mbs_dyn_code(fabs(v), denom) | (signbit(v) ? 8u : 0u);
            byte |= c << (4 * h);
        }
        codes[row * (K / 2) + mb * 64 + t] = (uint8_t)byte;
    } else if (t < 72) {
        const int jb = t - 64;
        const int64_t j = mb * 8 + jb;   // base-block column
        const uint32_t E = mbs_block_exponent(amax_bits[jb], mc);
        scales[((row >> 7) * sf_tiles_k + (j >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + (j & 3)] =
            (uint8_t)E;
    }
}

// max |x| over a bf16 tensor -> atomicMax on the float bits of *amax (init 0).
// Persistent: CTA b walks the 128 x 128 tiles n-1-b, n-1-b-G, ... (G CTAs), a
// thread issuing its 8 16-byte loads of a tile (4 rows x 16 columns, as in
// quantize_kernel) before reducing them.  Walking the tiles from the end of the
// tensor towards its start leaves the first rows in L2 when the pass ends, and
// the quantize kernel that follows reads those rows first.
__global__ void __launch_bounds__(kQThreads) amax_kernel(const uint16_t *__restrict__ src, int64_t M, int64_t K,
                                                         int64_t ld, unsigned int *__restrict__ amax_bits) {
    // src and the zeroed slot may come from the previous kernel in the stream
    // (launched with programmatic serialization, this kernel starts early);
    // the quantize kernel that follows may launch now and waits for this
    // grid's completion itself
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t tiles_x = (K + kQTileCols - 1) / kQTileCols;
    const int64_t n_tiles = tiles_x * ((M + kQTileRows - 1) / kQTileRows);
    const int cl = (lane & 7) * 16;
    uint32_t m = 0;
    for (int64_t t = n_tiles - 1 - (int64_t)blockIdx.x; t >= 0; t -= gridDim.x) {
        const int64_t row0 = (t / tiles_x) * kQTileRows, col = (t % tiles_x) * kQTileCols + cl;
        uint4 v[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t row = row0 + i * 32 + warp * 4 + (lane >> 3);
            if (row < M && col < K) {
                const uint16_t *p = src + row * ld + col;
                v[i][0] = ldg_stream(p);
                v[i][1] = ldg_stream(p + 8);
            } else {
                v[i][0] = v[i][1] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, absmax16(v[i][0], v[i][1]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ uint32_t red[kQThreads / 32];
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kQThreads / 32; ++w) m = max(m, red[w]);
        if (m != 0u) atomicMax(amax_bits, m << 16);   // bf16 magnitude -> fp32 bits (order-preserving)
    }
}

// CTAs for amax_kernel: enough resident per SM to keep HBM busy, never more
// than there are tiles.
inline int64_t amax_grid(int64_t M, int64_t K, int num_sms) {
    const int64_t tiles = ((K + kQTileCols - 1) / kQTileCols) * ((M + kQTileRows - 1) / kQTileRows);
    const int64_t cap = (int64_t)num_sms * 4;
    return tiles < 1 ? 1 : (tiles < cap ? tiles : cap);
}

// g = RU_fp32(amax / 2688), 1 for an all-zero tensor; in place (amax bits -> g).
// Launched with programmatic serialization, it waits for the amax pass before
// reading the slot, and lets the quantize kernel launch at once.
__global__ void gscale_from_amax_kernel(float *__restrict__ slot) {
    griddep_wait();
    griddep_launch_dependents();
    const float amax = *slot;
    *slot = amax > 0.0f ? __fdiv_ru(amax, 2688.0f) : 1.0f;
}

// Decode 8 consecutive elements (row r, columns c..c+7) of a quantized matrix:
// the block's scale s (g*s for NVFP4, exact in fp64) and the 8 element values.
// macro: MXFP4-MBS only, the [rows][K/128] macro mantissas after the scale tiles.
template <int FMT>
MX_DEVICE_INLINE void load_dequant8(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                                    const float *__restrict__ gscale, const uint8_t *__restrict__ macro, int64_t K,
                                    int64_t r, int64_t c, double &s, float (&q)[8]) {
    using T = FmtTraits<FMT>;
    const int64_t sf_cols = K / T::kBlock, tiles_k = (sf_cols + 3) / 4, j = c / T::kBlock;
    const uint8_t sb = scales[((r >> 7) * tiles_k + (j >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3)];
    if (FMT == FMT_NVFP4) s = (double)(*gscale) * (double)(sb == 0 ? 0.0f : e4m3_pos_value(sb));
    else if (FMT == FMT_MXFP4_MBS) s = ldexp((double)(256 + macro[r * (K / 128) + c / 128]), (int)sb - 135);
    else s = sb == 0xFF ? (double)NAN : ldexp(1.0, (int)sb - 127);
    if (T::kBits == 8) {
        const uint2 w = *reinterpret_cast<const uint2 *>(codes + r * K + c);
        const uint32_t ww[2] = {w.x, w.y};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint16_t pair = (uint16_t)(ww[h] >> (16 * p));
                uint32_t f16x2;
                if (FMT == FMT_E4M3)
                    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(f16x2) : "h"(pair));
                else
                    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(f16x2) : "h"(pair));
                const __half2 hh = *reinterpret_cast<const __half2 *>(&f16x2);
                q[4 * h + 2 * p] = __low2float(hh);
                q[4 * h + 2 * p + 1] = __high2float(hh);
            }
        }
    } else if (T::kBits == 6) {
        // 8 codes = 6 bytes at a 2-byte aligned offset
        const uint16_t *p = reinterpret_cast<const uint16_t *>(codes + r * (K / 4 * 3) + c / 4 * 3);
        const uint64_t w = (uint64_t)p[0] | ((uint64_t)p[1] << 16) | ((uint64_t)p[2] << 32);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t code = (uint32_t)(w >> (6 * e)) & 0x3Fu;
            const uint32_t ex = (code >> 2) & 7u, m = code & 3u;
            // E3M2: subnormal m * 2^-4, else (1 + m/4) * 2^(ex - 3)
            const float mag = ex == 0u ? 0.0625f * (float)m : __uint_as_float(((ex + 124u) << 23) | (m << 21));
            q[e] = (code & 0x20u) ? -mag : mag;
        }
    } else {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(codes + r * (K / 2) + c / 2);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t code = (w >> (4 * e)) & 0xFu;
            const float mag = e2m1_mag(code & 7u);
            q[e] = (code & 8u) ? -mag : mag;
        }
    }
}

// Dequantize: 8 elements of one row per thread.  The exact value g*s*q is
// formed in fp64 (at most 30 significant bits) and rounded once to bf16.
template <int FMT>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t *__restrict__ codes,
                                                         const uint8_t *__restrict__ scales,
                                                         const float *__restrict__ gscale,
                                                         const uint8_t *__restrict__ macro, int64_t M, int64_t K,
                                                         uint16_t *__restrict__ dst, int64_t ld) {
    const int64_t vec_per_row = K / 8;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= M * vec_per_row) return;
    const int64_t r = i / vec_per_row, c = (i % vec_per_row) * 8;
    double s;
    float q[8];
    load_dequant8<FMT>(codes, scales, gscale, macro, K, r, c, s, q);
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat16 lo = __double2bfloat16(s * (double)q[2 * e]);
        const __nv_bfloat16 hi = __double2bfloat16(s * (double)q[2 * e + 1]);
        out[e] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
    }
    *reinterpret_cast<uint4 *>(dst + r * ld + c) = make_uint4(out[0], out[1], out[2], out[3]);
}

// QSNR sums (page "Unveiling the Potential of Quantization with MXFP4",
// sections 3-4: fidelity as quantization SNR): sums[0] += sum x^2 and
// sums[1] += sum (x - xhat)^2 over a bf16 source [M x K] (pitch ld) and its
// quantized form, in fp64 (x and xhat are exact there, the squares nearly so).
// Grid-stride over 8-element vectors; one atomic add per block and sum.
template <int FMT>
__global__ void __launch_bounds__(256) qsnr_kernel(const uint16_t *__restrict__ src, int64_t ld,
                                                   const uint8_t *__restrict__ codes,
                                                   const uint8_t *__restrict__ scales,
                                                   const float *__restrict__ gscale,
                                                   const uint8_t *__restrict__ macro, int64_t M, int64_t K,
                                                   double *__restrict__ sums) {
    const int64_t vec_per_row = K / 8, nvec = M * vec_per_row;
    double sx = 0.0, se = 0.0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / vec_per_row, c = (i % vec_per_row) * 8;
        double s;
        float q[8];
        load_dequant8<FMT>(codes, scales, gscale, macro, K, r, c, s, q);
        const uint4 v = *reinterpret_cast<const uint4 *>(src + r * ld + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double x = (double)((e & 1) ? bf16hi(w[e >> 1]) : bf16lo(w[e >> 1]));
            const double d = x - s * (double)q[e];
            sx += x * x;
            se += d * d;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sx += __shfl_xor_sync(0xffffffffu, sx, o);
        se += __shfl_xor_sync(0xffffffffu, se, o);
    }
    __shared__ double red[2][8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[0][warp] = sx;
        red[1][warp] = se;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0, b = 0.0;
        for (int k = 0; k < (int)(blockDim.x >> 5); ++k) {
            a += red[0][k];
            b += red[1][k];
        }
        atomicAdd(&sums[0], a);
        atomicAdd(&sums[1], b);
    }
}

}  // namespace mx
