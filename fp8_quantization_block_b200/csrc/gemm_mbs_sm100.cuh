// gemm_mbs_sm100.cuh -- GEMM of two MXFP4 operands with macro-block scaling
// (MXFP4-MBS) on the sm_100a tensor cores.
//
// Page "Unveiling the Potential of Quantization with MXFP4: Strategies for
// Quantization Error Reduction", section 2.B (Macro Block Scaling): E2M1
// elements in 1x16 base blocks with E8M0 scales, and per 1x128 macro block one
// factor 1 + m/256; the macro-block math runs beside the tensor cores, which
// only apply the base blocks' scales.  Here
//
//   C[i][j] = sum over macro blocks b of fA[i][b] fB[j][b] P_b[i][j],
//   P_b[i][j] = sum_{k in b} (2^(EA-127) qA[i][k]) (2^(EB-127) qB[j][k]),
//   fA = (256 + mA) / 256, fB = (256 + mB) / 256,
//
// P_b on the tensor core (FP32 in TMEM), the factors on the CUDA cores.
//
// The tensor core takes E8M0 scales on 32-element groups (kind::mxf4,
// block32); a group holds two 16-element base blocks with their own scales.
// Each macro block therefore runs as two passes of MMAs: pass 0 on A with the
// second half of every 32-element group cleared (in 128-byte-swizzled shared
// memory a 16-byte unit is one group: bytes 0-7 hold elements 0-15, bytes 8-15
// elements 16-31, whatever the swizzle), with each group's first base-block
// scales of A and B; pass 1 on a copy of A with the first halves cleared, with
// the second base-block scales.  The cleared half contributes exact zeros, so
// both passes are exact block-scaled products and P_b is their sum.
//
// One CTA per 128 x 128 output tile (14 warps):
//   warp 0      TMA producer: A and B code tiles (128 bytes of K = two macro
//               blocks per stage) and the stage's 512-byte scale chunks of A
//               and B (four per operand) into a STAGES-deep ring;
//   warps 2-5   prep: per stage, build A's two pass operands (clear half of
//               every group in place, the other half in a copy) and write the
//               pass scales into the stage's TMEM scale slot (tcgen05.st);
//   warp 1      MMA issuer: per macro block, 2 + 2 MMAs (K = 64 elements
//               each) into one of two partial accumulators, then a commit;
//   warps 6-13  drain: per macro block, each warp reads 64 columns of its TMEM
//               lane quadrant's partial, adds fA fB P to a running sum in
//               registers and releases the partial; at the end the sums are
//               rounded to bf16 and stored.
// Every mbarrier wait is bounded (mx_common.cuh).
#pragma once

#include "gemm_sm100.cuh"

namespace mx {

constexpr int kMbsThreads = 14 * 32;
constexpr int kMbsStages = 4;
constexpr int kMbsBN = 128;

struct MbsLayout {
    static constexpr int kTileBytes = 128 * kStageKBytes;            // 16 KB: A, A's pass-1 copy, B
    static constexpr int kSfBytes = 4 * 512;                         // a stage's scale chunks of one operand
    static constexpr int kOffA = 0;
    static constexpr int kOffA2 = kOffA + kMbsStages * kTileBytes;
    static constexpr int kOffB = kOffA2 + kMbsStages * kTileBytes;
    static constexpr int kOffSfa = kOffB + kMbsStages * kTileBytes;
    static constexpr int kOffSfb = kOffSfa + kMbsStages * kSfBytes;
    static constexpr int kOffBar = kOffSfb + kMbsStages * kSfBytes;
    // full[S], ready[S], empty[S], pfull[2], pempty[2], mma_done
    static constexpr int kNumBars = 3 * kMbsStages + 5;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(kAlloc <= kSmemLimit, "shared memory budget");
    // TMEM: partial accumulators at columns 0 and 128, then one 32-column
    // scale slot per stage: [pass][A chunk 0, 1 | B chunk 0, 1] x 4 columns
    static constexpr int kTmemSf = 2 * kMbsBN;
    static constexpr int kSlotCols = 32;
    static constexpr int kTmemCols = 512;
    static_assert(kTmemSf + kMbsStages * kSlotCols <= kTmemCols, "TMEM budget");
};

struct MbsParams {
    uint16_t *C;
    int64_t ldc;
    int M, N, K;
    int num_kt;          // stages along K (128 bytes = 256 elements each)
    int n_macro;         // macro blocks along K = K / 128
    int m_blocks;
    const uint8_t *macro_a;   // [M][K/128] macro mantissas of A
    const uint8_t *macro_b;   // [N][K/128] of B
    int vec_store;            // C 16-byte aligned and ldc % 8 == 0
    int skip_producer;
    uint64_t wait_limit_ns;
};

// Pass scales of one stage for this lane's rows.  sf points at the stage's four
// 512-byte chunks of 16-element scales (chunk c: scale columns 4c .. 4c + 3);
// lane r of a chunk holds word w = the four columns of row 32w + r.  The pass-h
// operand of 32-element group g (g = 0..7 in the stage) takes base block 2g + h,
// laid out as two MXFP4 chunks (chunk c': groups 4c' .. 4c' + 3).
MX_DEVICE_INLINE void mbs_pass_words(const uint8_t *sf, int lane, uint32_t (&p0)[8], uint32_t (&p1)[8]) {
    uint4 ch[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) ch[c] = *reinterpret_cast<const uint4 *>(sf + c * 512 + lane * 16);
#pragma unroll
    for (int cp = 0; cp < 2; ++cp) {
        const uint32_t lo[4] = {ch[2 * cp].x, ch[2 * cp].y, ch[2 * cp].z, ch[2 * cp].w};
        const uint32_t hi[4] = {ch[2 * cp + 1].x, ch[2 * cp + 1].y, ch[2 * cp + 1].z, ch[2 * cp + 1].w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            // group columns 0, 1 come from chunk 2c' (base blocks 0..3), 2, 3 from
            // chunk 2c' + 1 (base blocks 4..7): bytes {h, 2 + h} of each word
            p0[4 * cp + w] = __byte_perm(lo[w], hi[w], 0x6420);
            p1[4 * cp + w] = __byte_perm(lo[w], hi[w], 0x7531);
        }
    }
}

__global__ void __launch_bounds__(kMbsThreads, 1)
    gemm_mbs_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSfa, const __grid_constant__ CUtensorMap tmSfb,
                    MbsParams p) {
    using L = MbsLayout;
    constexpr int S = kMbsStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *ready = full + S;
    uint64_t *empty = ready + S;
    uint64_t *pfull = empty + S;     // [2]
    uint64_t *pempty = pfull + 2;    // [2]
    uint64_t *mma_done = pempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = (int)(blockIdx.x % (unsigned)p.m_blocks) * 128;
    const int n0 = (int)(blockIdx.x / (unsigned)p.m_blocks) * kMbsBN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ready[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pfull[i], 1);
            mbar_init(&pempty[i], 8);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSfa);
        tma_prefetch_desc(&tmSfb);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (!p.skip_producer) {
            int used = 0;
            for (int kt = 0; kt < p.num_kt; ++kt) {
                const int s = kt % S;
                const uint32_t ph = (uint32_t)((kt / S) & 1);
                if (!mbar_wait_bounded(&empty[s], ph ^ 1u, p.wait_limit_ns, SITE_GEMM_PRODUCER_EMPTY, abort_flag))
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(2 * L::kTileBytes + 2 * L::kSfBytes));
                    tma_load_2d(smem + L::kOffA + s * L::kTileBytes, &tmA, kt * kStageKBytes, m0, &full[s]);
                    tma_load_2d(smem + L::kOffB + s * L::kTileBytes, &tmB, kt * kStageKBytes, n0, &full[s]);
                    tma_load_3d(smem + L::kOffSfa + s * L::kSfBytes, &tmSfa, 0, kt * 4, m0 / 128, &full[s]);
                    tma_load_3d(smem + L::kOffSfb + s * L::kSfBytes, &tmSfb, 0, kt * 4, n0 / 128, &full[s]);
                }
                __syncwarp();
                ++used;
            }
            for (int u = max(0, used - S); u < used; ++u)
                mbar_wait_bounded(&full[u % S], (uint32_t)((u / S) & 1), p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
        }
    } else if (warp >= 2 && warp < 6) {
        // ------------------------------------------------------------ prep
        const int q = warp & 3;     // the TMEM lane quadrant this warp may write
        const int t = threadIdx.x - 64;
        for (int kt = 0; kt < p.num_kt; ++kt) {
            const int s = kt % S;
            if (!mbar_wait_bounded(&full[s], (uint32_t)((kt / S) & 1), p.wait_limit_ns, SITE_GEMM_SF_LOAD,
                                   abort_flag))
                break;
            // the two pass operands of A: 1024 16-byte units, 8 per thread
            uint4 *a = reinterpret_cast<uint4 *>(smem + L::kOffA + s * L::kTileBytes);
            uint4 *a2 = reinterpret_cast<uint4 *>(smem + L::kOffA2 + s * L::kTileBytes);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int u = t + 128 * i;
                const uint4 v = a[u];
                a2[u] = make_uint4(0u, 0u, v.z, v.w);
                a[u] = make_uint4(v.x, v.y, 0u, 0u);
            }
            fence_proxy_async_smem();
            // the pass scales into this stage's TMEM slot
            uint32_t a0[8], a1[8], b0[8], b1[8];
            mbs_pass_words(smem + L::kOffSfa + s * L::kSfBytes, lane, a0, a1);
            mbs_pass_words(smem + L::kOffSfb + s * L::kSfBytes, lane, b0, b1);
            const uint32_t slot = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(L::kTmemSf + s * L::kSlotCols);
            tmem_st8(slot + 0, a0);
            tmem_st8(slot + 8, b0);
            tmem_st8(slot + 16, a1);
            tmem_st8(slot + 24, b1);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[s]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint64_t desc_ab = smem_desc(0, 16, 1024, 2);
        const uint32_t leader = lane == 0 ? 1u : 0u;
        int mb = 0;   // macro blocks issued
        bool stop = false;
        for (int kt = 0; kt < p.num_kt && !stop; ++kt) {
            const int s = kt % S;
            if (!mbar_wait_bounded(&ready[s], (uint32_t)((kt / S) & 1), p.wait_limit_ns, SITE_GEMM_MMA_FULL,
                                   abort_flag))
                break;
            tc_fence_after();
            const uint64_t ad = desc_ab | (uint64_t)((smem_u32(smem + L::kOffA + s * L::kTileBytes) >> 4) & 0x3FFFu);
            const uint64_t ad2 = desc_ab | (uint64_t)((smem_u32(smem + L::kOffA2 + s * L::kTileBytes) >> 4) & 0x3FFFu);
            const uint64_t bd = desc_ab | (uint64_t)((smem_u32(smem + L::kOffB + s * L::kTileBytes) >> 4) & 0x3FFFu);
            const uint32_t slot = tmem + (uint32_t)(L::kTmemSf + s * L::kSlotCols);
            for (int h = 0; h < 2 && kt * 2 + h < p.n_macro; ++h, ++mb) {
                const int pi = mb & 1;
                if (!mbar_wait_bounded(&pempty[pi], (uint32_t)(((mb >> 1) & 1) ^ 1), p.wait_limit_ns,
                                       SITE_GEMM_MMA_ACC_EMPTY, abort_flag)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(pi * kMbsBN);
                // macro block h: K steps 2h and 2h + 1 (32 bytes = 64 elements
                // each), group-scale chunk c' = h, scale ids 0 and 2
#pragma unroll
                for (int pass = 0; pass < 2; ++pass) {
                    const uint64_t a_desc = pass == 0 ? ad : ad2;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = 2 * h + e;
                        const uint32_t sf_id = (uint32_t)(e * 2);
                        tc_mma_mxf4_if(d, a_desc + 2u * j, bd + 2u * j, gemm_idesc<2, kMbsBN>(sf_id),
                                       slot + (uint32_t)(16 * pass + 4 * h), slot + (uint32_t)(16 * pass + 8 + 4 * h),
                                       (pass | e) ? 1u : 0u, leader);
                    }
                }
                tc_commit_if(&pfull[pi], leader);
            }
            tc_commit_if(&empty[s], leader);
        }
        tc_commit_if(mma_done, leader);
        __syncwarp();
    } else if (warp >= 6) {
        // ------------------------------------------------------------ drain
        const int q = warp & 3;                 // TMEM lane quadrant
        const int half = (warp - 6) >> 2;       // columns 64 * half .. 64 * half + 63
        const int row = m0 + 32 * q + lane;
        const int col0 = n0 + 64 * half;
        float acc[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] = 0.0f;
        const int kmac = p.K / 128;
        for (int mb = 0; mb < p.n_macro; ++mb) {
            const int pi = mb & 1;
            // the factors of this macro block (rows / columns past the matrix: 1)
            const float fa = row < p.M ? (float)(256 + p.macro_a[(int64_t)row * kmac + mb]) : 256.0f;
            const int cb0 = col0 + lane, cb1 = col0 + 32 + lane;
            const float fb0 = (cb0 < p.N ? (float)(256 + p.macro_b[(int64_t)cb0 * kmac + mb]) : 256.0f) * 0x1p-16f;
            const float fb1 = (cb1 < p.N ? (float)(256 + p.macro_b[(int64_t)cb1 * kmac + mb]) : 256.0f) * 0x1p-16f;
            if (!mbar_wait_bounded(&pfull[pi], (uint32_t)((mb >> 1) & 1), p.wait_limit_ns, SITE_GEMM_EPI_ACC,
                                   abort_flag))
                break;
            tc_fence_after();
            const uint32_t t_p = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(pi * kMbsBN + 64 * half);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t r[32];
                tmem_ld32(t_p + (uint32_t)(32 * ch), r);
                tmem_wait_ld();
                const float fbv = ch == 0 ? fb0 : fb1;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    // (256 + mA)(256 + mB) / 2^16 is exact in fp32
                    const float f = fa * __shfl_sync(0xffffffffu, fbv, c);
                    acc[32 * ch + c] = __fmaf_rn(f, __uint_as_float(r[c]), acc[32 * ch + c]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[pi]);
        }
        if (!*abort_flag && row < p.M) {
            uint16_t *dst = p.C + (int64_t)row * p.ldc + col0;
            if (p.vec_store && col0 + 64 <= p.N) {
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h = __floats2bfloat162_rn(acc[8 * v + 2 * e], acc[8 * v + 2 * e + 1]);
                        w[e] = *reinterpret_cast<const uint32_t *>(&h);
                    }
                    *reinterpret_cast<uint4 *>(dst + 8 * v) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (col0 + c < p.N) dst[c] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[c]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        // every MMA has completed once mma_done has fired
        mbar_wait_bounded(mma_done, 0, p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
        tmem_dealloc(tmem, L::kTmemCols);
    }
    griddep_launch_dependents();
}

}  // namespace mx
