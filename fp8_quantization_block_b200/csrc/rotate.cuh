// rotate.cuh -- 32-point Walsh-Hadamard block rotation fused with quantization.
//
// Page "Microscaling MXFP4/NVFP4 on Blackwell for reasoning LLMs", section
// "Técnicas de preservação de acurácia: QuaRot, SpinQuant e ReSET": Hadamard /
// Walsh-Hadamard rotations spread a block's outlier energy over its 32
// elements before 4-bit quantization.  Each 32-element block b of a row is
// replaced by y_b = c * (H32 x_b), H32 the Sylvester-ordered Hadamard matrix
// and c = RN_fp32(1/sqrt(32)) (0x3E3504F3), evaluated in fp32 as butterflies of
// half-width 1, 2, 4, 8, 16 in that order, each (a, b) -> (a + b, a - b) with
// one rounding, then one product with c; the fp32 y is quantized by the usual
// rules (MX: E = ceil(log2(max|y| / max_elem)) + 127; NVFP4: s and RNE of
// y / (g s)).  Applying the same rotation to both GEMM operands leaves
// A * B^T unchanged up to rounding, since H32 H32^T = 32 I.
//
// Thread layout as in quantize_kernel: a 128 x 128 tile per CTA, 16
// consecutive elements per thread, so a 32-element block spans lanes 2m and
// 2m + 1; the last butterfly stage exchanges halves with __shfl_xor(., 1).
#pragma once

#include "quantize.cuh"

namespace mx {

constexpr uint32_t kRhtScaleBits = 0x3E3504F3u;  // RN_fp32(1 / sqrt(32))

// The unnormalised butterflies H32 x of the 32-element block whose half (16
// values) this thread holds: lower = even lane (block elements 0..15), upper =
// odd lane.  Stages of half-width 1, 2, 4 run on the pairs (x[j], x[j + 8]),
// two sums per instruction; half-width 8 pairs x[j] with x[j + 8] inside this
// thread; half-width 16 pairs this lane with lane ^ 1: lower keeps a + b,
// upper b' - a' = fma(-1, own, other), one rounding as in the scalar form.
// On return z[j] = (H32 x)[j] (this half), every sum rounded to fp32 in the
// stage order of the definition; the caller applies c = RN_fp32(1/sqrt(32)).
// All 32 lanes of the warp must call this together.
MX_DEVICE_INLINE void rht32_butterflies(float (&z)[16], int lane) {
    uint64_t P[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) P[j] = pk2(z[j], z[j + 8]);
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int j0 = 0; j0 < 8; j0 += 2 * h) {
#pragma unroll
            for (int j = j0; j < j0 + h; ++j) {
                const uint64_t a = P[j], b = P[j + h];
                P[j] = add2(a, b);
                P[j + h] = sub2(a, b);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a, b;
        upk2(P[j], a, b);
        z[j] = __fadd_rn(a, b);
        z[j + 8] = __fsub_rn(a, b);
    }
    const float sg = (lane & 1) ? -1.0f : 1.0f;
    const uint64_t S = pk2(sg, sg);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float o0 = __shfl_xor_sync(0xffffffffu, z[2 * j], 1);
        const float o1 = __shfl_xor_sync(0xffffffffu, z[2 * j + 1], 1);
        float r0, r1;
        upk2(fma2(S, pk2(z[2 * j], z[2 * j + 1]), pk2(o0, o1)), r0, r1);
        z[2 * j] = r0;
        z[2 * j + 1] = r1;
    }
}

// y = RN(c * z) for the 16 values (the normalised rotation).
MX_DEVICE_INLINE void rht32_scale(float (&z)[16]) {
    const float c = __uint_as_float(kRhtScaleBits);
    const uint64_t C = pk2(c, c);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a, b;
        upk2(mul2(C, pk2(z[2 * j], z[2 * j + 1])), a, b);
        z[2 * j] = a;
        z[2 * j + 1] = b;
    }
}

// The rotated half-block: y = c * (H32 x) as defined above.
MX_DEVICE_INLINE void rht32_halves(float (&x)[16], int lane) {
    rht32_butterflies(x, lane);
    rht32_scale(x);
}

// MX exponent from the fp32 bits of a block's max |y| (non-negative, finite):
// amax = 1.m * 2^(f-127), max_elem = M * 2^k: E = f - k + (m > (M - 1) 2^23),
// clamped below at 0 (zero and tiny maxima).
template <int FMT>
MX_DEVICE_INLINE int mx_scale_byte_f32(float amax) {
    using T = FmtTraits<FMT>;
    const uint32_t bits = __float_as_uint(amax);
    const uint32_t thr = (uint32_t)T::kMantThr << 16;   // the bf16 threshold, widened to 23 mantissa bits
    int e = (int)(bits >> 23) - T::kExpOff + (((bits & 0x7FFFFFu) > thr) ? 1 : 0);
    return e < 0 ? 0 : e;
}

// Rotate and quantize a bf16 [M x K] matrix (K % 32 == 0) into codes / scales
// laid out as quantize_kernel's.  NVFP4: *gscale_in is g, or max|y| when
// g_from_amax (then g = RU(max|y| / 2688), 1 for 0); gscale_out as there.
template <int FMT>
// (four resident CTAs per SM for the register allocation: measured fastest)
__global__ void __launch_bounds__(kQThreads, 4) quantize_rht_kernel(const uint16_t *__restrict__ src, int64_t M,
                                                                 int64_t K, int64_t ld, uint8_t *__restrict__ codes,
                                                                 uint8_t *__restrict__ scales, int64_t sf_tiles_k,
                                                                 const float *__restrict__ gscale_in,
                                                                 float *__restrict__ gscale_out, int g_from_amax) {
    using T = FmtTraits<FMT>;
    constexpr int kBlocksPerRow = kQTileCols / T::kBlock;
    constexpr int kSfBytes = kQTileRows * kBlocksPerRow;
    constexpr int kPasses = kQTileRows / 32;
    __shared__ __align__(16) uint8_t sf_tile[kSfBytes];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row0 = (int64_t)blockIdx.y * kQTileRows;
    const int64_t col0 = (int64_t)blockIdx.x * kQTileCols;
    const int cl = (lane & 7) * 16;
    const int64_t col = col0 + cl;
    const bool col_ok = col < K;   // K % 32 == 0: both halves of a block exist or neither
    const int jb = cl / T::kBlock;

    float g = 1.0f, rg_lo = 1.0f, rg_hi = 1.0f, inv6g = 1.0f, sc = 1.0f;
    __shared__ NvTables nvt;
    // the NVFP4 tables are constants: filled while the previous kernel in the
    // stream finishes
    if (FMT == FMT_NVFP4 && threadIdx.x < 128) {
        const uint32_t c = threadIdx.x;
        const float v = (c == 0u || c == 127u) ? 0.0f : e4m3_pos_value(c);
        nvt.val[c] = v;
        nvt.inv_lo[c] = v > 0.0f ? __frcp_rd(v) : 0.0f;
        nvt.inv_hi[c] = v > 0.0f ? __frcp_ru(v) : 0.0f;
    }
    griddep_wait();

    // the tile's loads first, so that they are in flight while g is read
    uint4 v[kPasses][2];
#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
        const int rl = i * 32 + warp * 4 + (lane >> 3);
        const int64_t row = row0 + rl;
        if (row < M && col_ok) {
            const uint16_t *p = src + row * ld + col;
            v[i][0] = ldg_stream(p);
            v[i][1] = ldg_stream(p + 8);
        } else {
            v[i][0] = v[i][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    if (FMT == FMT_NVFP4) {
        g = *gscale_in;
        if (g_from_amax) g = g > 0.0f ? __fdiv_ru(g, 2688.0f) : 1.0f;
        if (gscale_out != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *gscale_out = g;
        // as in quantize_kernel: a tiny g is handled as (y 2^64) / (g 2^64)
        if (g < 0x1p-100f) {
            sc = 0x1p64f;
            g *= sc;
        }
        rg_lo = __frcp_rd(g);
        rg_hi = __frcp_ru(g);
        inv6g = 1.0f / (6.0f * g);
        __syncthreads();  // the tables
    }

#pragma unroll
    for (int i = 0; i < kPasses; ++i) {
        const int rl = i * 32 + warp * 4 + (lane >> 3);
        const int64_t row = row0 + rl;
        const bool ok = row < M && col_ok;
        // z = H32 x (unnormalised); y = RN(c z).  max |y| = RN(c max |z|), since
        // rounding is monotone and c > 0.
        float y[16];
        unpack16(v[i][0], v[i][1], y);
        rht32_butterflies(y, lane);
        float mz = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) mz = fmaxf(mz, fabsf(y[e]));
        if (T::kBlock == 32) mz = fmaxf(mz, __shfl_xor_sync(0xffffffffu, mz, 1));
        const float m = __fmul_rn(__uint_as_float(kRhtScaleBits), mz);
        uint32_t sbyte;
        if (FMT == FMT_NVFP4) {
            rht32_scale(y);
            if (sc != 1.0f) {
#pragma unroll
                for (int e = 0; e < 16; ++e) y[e] *= sc;   // exact: a power of two, scaling up
            }
            sbyte = nv_block_scale(m * sc, g, inv6g, nvt.val);
            if (ok) {
                uint32_t q0 = 0, q1 = 0;
                if (sbyte == 0u) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint32_t sgn = (__float_as_uint(y[e]) >> 31) & 1u;
                        if (e < 8) q0 |= sgn << (4 * e + 3);
                        else q1 |= sgn << (4 * (e - 8) + 3);
                    }
                } else {
                    const float r_lo = __fmul_rd(rg_lo, nvt.inv_lo[sbyte]);
                    const float r_hi = __fmul_ru(rg_hi, nvt.inv_hi[sbyte]);
                    nv_codes16_f32(y, g, nvt.val[sbyte], r_lo, r_hi, q0, q1);
                }
                *reinterpret_cast<uint2 *>(codes + row * (K / 2) + col / 2) = make_uint2(q0, q1);
            }
        } else {
            const int E = mx_scale_byte_f32<FMT>(m);
            sbyte = (uint32_t)E;
            if (ok) {
                // RN(c z) * 2^(127-E) = RN(z * (c 2^(127-E))) whenever RN(c z) is a
                // normal fp32 and c 2^(127-E) is too (E <= 250): scaling by a power
                // of two commutes with rounding there.  With max |y| >= 2^-90, an
                // element whose RN(c z) is subnormal scales to below 2^-17 of the
                // element grid's top (448 x 2^-126 / 2^-90 at most): both forms
                // give it a zero code of the same sign.  Other blocks take the
                // two-step form.
                const float inv = mx_inv_scale(E);
                float f[16];
                if (E <= 250 && m >= 0x1p-90f) {
                    const float cs = __uint_as_float(kRhtScaleBits) * inv;   // exact
                    const uint64_t CS = pk2(cs, cs);
#pragma unroll
                    for (int j = 0; j < 8; ++j) upk2(mul2(CS, pk2(y[2 * j], y[2 * j + 1])), f[2 * j], f[2 * j + 1]);
                } else {
                    rht32_scale(y);
#pragma unroll
                    for (int e = 0; e < 16; ++e) f[e] = y[e] * inv;
                }
                store_mx_codes16<FMT>(codes, row, K, col, f);
            }
        }
        const bool owner = T::kBlock == 16 || (lane & 1) == 0;
        if (owner) {
            const int64_t jglob = col0 / T::kBlock + jb;
            if (!(row < M) || jglob >= K / T::kBlock) sbyte = 0u;
            sf_tile[(jb >> 2) * 512 + (rl & 31) * 16 + (rl >> 5) * 4 + (jb & 3)] = (uint8_t)sbyte;
        }
    }
    __syncthreads();
    constexpr int kChunks = kSfBytes / 512;
    const int64_t chunk0 = (int64_t)blockIdx.y * sf_tiles_k + (int64_t)blockIdx.x * kChunks;
    const int64_t max_chunk = (int64_t)blockIdx.y * sf_tiles_k + sf_tiles_k;
    if (threadIdx.x < kSfBytes / 16) {
        const int c = threadIdx.x / 32;
        if (chunk0 + c < max_chunk) {
            uint4 val = *reinterpret_cast<const uint4 *>(sf_tile + threadIdx.x * 16);
            *reinterpret_cast<uint4 *>(scales + chunk0 * 512 + threadIdx.x * 16) = val;
        }
    }
    // the next kernel in the stream may start its setup now
    griddep_launch_dependents();
}

// max |y| over the rotated tensor (for the NVFP4 global scale): one 32-element
// block per thread pair, grid-stride over pairs; atomicMax on float bits.
__global__ void __launch_bounds__(256) amax_rht_kernel(const uint16_t *__restrict__ src, int64_t M, int64_t K,
                                                       int64_t ld, unsigned int *__restrict__ amax_bits) {
    const int lane = threadIdx.x & 31;
    const int64_t halves_per_row = K / 16;   // even: a block's two halves are 2b, 2b + 1
    const int64_t nhalves = M * halves_per_row;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    float m = 0.0f;
    // every lane of a warp runs the same iterations, so each shuffle has both halves
    for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w * 32 < nhalves; w += nwarps) {
        const int64_t i = w * 32 + lane;
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (i < nhalves) {
            const int64_t r = i / halves_per_row, c = (i % halves_per_row) * 16;
            const uint16_t *p = src + r * ld + c;
            v0 = ldg_stream(p);
            v1 = ldg_stream(p + 8);
        }
        float z[16];
        unpack16(v0, v1, z);
        rht32_butterflies(z, lane);
#pragma unroll
        for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(z[e]));
    }
    m = __fmul_rn(__uint_as_float(kRhtScaleBits), m);   // max |RN(c z)| = RN(c max |z|)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0 && m > 0.0f) atomicMax(amax_bits, __float_as_uint(m));
}

}  // namespace mx
