// gemm_sm100.cuh -- block-scaled GEMM on the sm_100a tensor cores (tcgen05).
//
// C[M x N] (bf16) = A_dq [M x K] * B_dq [N x K]^T, where A and B are stored as
// microscaling codes plus per-block scales ([MX] page "Microscaling MXFP4/NVFP4
// on Blackwell", section "Arquitetura Blackwell SM100 e aceleração nativa de
// NVFP4": the 5th-generation tensor core consumes the block codes directly and
// applies the block scale during FP32 accumulation).
//
// One CTA computes one 128 x BN output tile with four warp roles:
//   warp 0     TMA producer: code tiles of A and B (128-byte swizzled, K-major)
//              plus their 512-byte scale tiles into a STAGES-deep smem ring;
//   warp 1     TMEM owner and MMA issuer: tcgen05.cp moves each stage's scale
//              tiles into TMEM, then one thread issues the block-scaled
//              tcgen05.mma instructions (4 per stage, 32 bytes of K each) into
//              an FP32 accumulator in TMEM, and tcgen05.commit frees the stage;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (one row per thread),
//              x gA*gB for NVFP4, optional GELU and |C| max, bf16 RNE, stores.
// Every mbarrier wait is bounded (mx_common.cuh).
#pragma once

#include "mx_common.cuh"

namespace mx {

// Per-format MMA parameters.  A stage covers 128 bytes of K per row, i.e. 128
// FP8 or 256 FP4 elements; one MMA consumes 32 bytes of K.
template <int FMT>
struct GemmFmt;
template <>
struct GemmFmt<0> {  // MXFP8 E4M3: kind::mxf8f6f4, scale_vec 1X, UE8M0
    static constexpr int kElemPerByte = 1, kBlock = 32, kChunks = 1, kMmaPerChunk = 4, kSfPerMma = 1;
    static constexpr uint32_t kAFmt = 0, kScaleUE8M0 = 1;
};
template <>
struct GemmFmt<1> {  // MXFP8 E5M2
    static constexpr int kElemPerByte = 1, kBlock = 32, kChunks = 1, kMmaPerChunk = 4, kSfPerMma = 1;
    static constexpr uint32_t kAFmt = 1, kScaleUE8M0 = 1;
};
template <>
struct GemmFmt<2> {  // MXFP4: kind::mxf4, scale_vec 2X (32-element blocks), UE8M0
    static constexpr int kElemPerByte = 2, kBlock = 32, kChunks = 2, kMmaPerChunk = 2, kSfPerMma = 2;
    static constexpr uint32_t kAFmt = 1, kScaleUE8M0 = 1;
};
template <>
struct GemmFmt<3> {  // NVFP4: kind::mxf4nvf4, scale_vec 4X (16-element blocks), UE4M3
    static constexpr int kElemPerByte = 2, kBlock = 16, kChunks = 4, kMmaPerChunk = 1, kSfPerMma = 4;
    static constexpr uint32_t kAFmt = 1, kScaleUE8M0 = 0;
};

constexpr int kBM = 128;
constexpr int kStageKBytes = 128;
constexpr int kGemmThreads = 192;

struct GemmParams {
    const uint8_t *sfa;
    const uint8_t *sfb;
    int64_t sf_tiles_k;  // 512-byte scale tiles per 128-row band (= ceil(K / block / 4))
    uint16_t *C;
    int64_t ldc;
    int M, N, K;
    int num_kt;           // stages along K = ceil(K_bytes / 128)
    const float *ga;      // NVFP4 per-tensor scales (nullptr for MX)
    const float *gb;
    float *amax_out;      // nullable: max |C| (bf16) via atomicMax on float bits
    int epilogue;         // 0 none, 1 GELU
    int skip_producer;    // test hook: never issue loads
    uint64_t wait_limit_ns;
};

template <int FMT, int BN, int STAGES>
struct GemmSmem {
    using F = GemmFmt<FMT>;
    static constexpr int kBBands = BN / 128;
    static constexpr int kABytes = kBM * kStageKBytes;
    static constexpr int kBBytes = BN * kStageKBytes;
    static constexpr int kSfaBytes = F::kChunks * 512;
    static constexpr int kSfbBytes = F::kChunks * 512 * kBBands;
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + STAGES * kABytes;
    static constexpr int kOffSfa = kOffB + STAGES * kBBytes;
    static constexpr int kOffSfb = kOffSfa + STAGES * kSfaBytes;
    static constexpr int kOffBar = kOffSfb + STAGES * kSfbBytes;
    static constexpr int kNumBars = 2 * STAGES + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
    // TMEM columns: accumulator, then scale tiles of A and B for one stage.
    static constexpr int kTmemSfa = BN;
    static constexpr int kTmemSfb = BN + 4 * F::kChunks;
    static constexpr int kTmemUsed = kTmemSfb + 4 * F::kChunks * kBBands;
    static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256 : 512;
};

// Instruction descriptor of the block-scaled MMA (M = 128, K-major A and B).
template <int FMT, int BN>
MX_DEVICE_INLINE uint32_t gemm_idesc(uint32_t sf_id) {
    using F = GemmFmt<FMT>;
    return (sf_id << 4) | (F::kAFmt << 7) | (F::kAFmt << 10) | ((uint32_t)(BN >> 3) << 17) |
           (F::kScaleUE8M0 << 23) | ((uint32_t)(kBM >> 4) << 24) | (sf_id << 29);
}

template <int FMT>
MX_DEVICE_INLINE void gemm_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                               uint32_t acc) {
    if (FMT <= 1) tc_mma_mxf8f6f4(d, a, b, idesc, sfa, sfb, acc);
    else if (FMT == 2) tc_mma_mxf4(d, a, b, idesc, sfa, sfb, acc);
    else tc_mma_nvf4(d, a, b, idesc, sfa, sfb, acc);
}

MX_DEVICE_INLINE float gelu_erf(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752440f)); }

// Number of valid 32-byte MMA steps and 512-byte scale chunks in stage kt.
template <int FMT>
MX_DEVICE_INLINE void stage_extent(int kt, int K, int &n_mma, int &n_chunk) {
    using F = GemmFmt<FMT>;
    const int stage_elems = kStageKBytes * F::kElemPerByte;
    int kv = K - kt * stage_elems;
    if (kv > stage_elems) kv = stage_elems;
    n_mma = kv / (32 * F::kElemPerByte);
    n_chunk = (n_mma + F::kMmaPerChunk - 1) / F::kMmaPerChunk;
}

template <int FMT, int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
    using F = GemmFmt<FMT>;
    using L = GemmSmem<FMT, BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && !p.skip_producer) {
            const int n_bands_total = (p.N + 127) / 128;
            int last_round[STAGES];
            for (int s = 0; s < STAGES; ++s) last_round[s] = -1;
            for (int kt = 0; kt < p.num_kt; ++kt) {
                const int s = kt % STAGES, round = kt / STAGES;
                if (!mbar_wait_bounded(&empty[s], (round & 1) ^ 1, p.wait_limit_ns, SITE_GEMM_PRODUCER_EMPTY,
                                       abort_flag))
                    break;
                int n_mma, n_chunk;
                stage_extent<FMT>(kt, p.K, n_mma, n_chunk);
                const int bands = min(L::kBBands, n_bands_total - n0 / 128);
                const uint32_t bytes = L::kABytes + L::kBBytes + (uint32_t)n_chunk * 512u * (1u + (uint32_t)bands);
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(smem + L::kOffA + s * L::kABytes, &tmA, kt * kStageKBytes, m0, &full[s]);
                tma_load_2d(smem + L::kOffB + s * L::kBBytes, &tmB, kt * kStageKBytes, n0, &full[s]);
                const int64_t sf_k = (int64_t)kt * F::kChunks;
                bulk_load(smem + L::kOffSfa + s * L::kSfaBytes, p.sfa + ((int64_t)(m0 / 128) * p.sf_tiles_k + sf_k) * 512,
                          (uint32_t)n_chunk * 512u, &full[s]);
                for (int h = 0; h < bands; ++h)
                    bulk_load(smem + L::kOffSfb + s * L::kSfbBytes + h * F::kChunks * 512,
                              p.sfb + ((int64_t)(n0 / 128 + h) * p.sf_tiles_k + sf_k) * 512, (uint32_t)n_chunk * 512u,
                              &full[s]);
                last_round[s] = round;
            }
            // Do not leave while copies into this CTA's shared memory are in flight.
            for (int s = 0; s < STAGES; ++s)
                if (last_round[s] >= 0)
                    mbar_wait_bounded(&full[s], last_round[s] & 1, p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t t_acc = tmem, t_sfa = tmem + L::kTmemSfa, t_sfb = tmem + L::kTmemSfb;
            const uint32_t a_base = smem_u32(smem + L::kOffA), b_base = smem_u32(smem + L::kOffB);
            const uint32_t sfa_base = smem_u32(smem + L::kOffSfa), sfb_base = smem_u32(smem + L::kOffSfb);
            for (int kt = 0; kt < p.num_kt; ++kt) {
                const int s = kt % STAGES, round = kt / STAGES;
                if (!mbar_wait_bounded(&full[s], round & 1, p.wait_limit_ns, SITE_GEMM_MMA_FULL, abort_flag)) break;
                tc_fence_after();
                int n_mma, n_chunk;
                stage_extent<FMT>(kt, p.K, n_mma, n_chunk);
                for (int c = 0; c < n_chunk; ++c) {
                    tc_cp_sf(t_sfa + 4 * c, smem_desc(sfa_base + s * L::kSfaBytes + c * 512, 0, 128, 0));
#pragma unroll
                    for (int h = 0; h < L::kBBands; ++h)
                        tc_cp_sf(t_sfb + 4 * (c * L::kBBands + h),
                                 smem_desc(sfb_base + s * L::kSfbBytes + (h * F::kChunks + c) * 512, 0, 128, 0));
                }
                const uint32_t a_stage = a_base + s * L::kABytes, b_stage = b_base + s * L::kBBytes;
                for (int j = 0; j < n_mma; ++j) {
                    const int chunk = j / F::kMmaPerChunk;
                    const uint32_t sf_id = (uint32_t)((j % F::kMmaPerChunk) * F::kSfPerMma);
                    const uint64_t ad = smem_desc(a_stage + 32 * j, 16, 1024, 2);
                    const uint64_t bd = smem_desc(b_stage + 32 * j, 16, 1024, 2);
                    gemm_mma<FMT>(t_acc, ad, bd, gemm_idesc<FMT, BN>(sf_id), t_sfa + 4 * chunk,
                                  t_sfb + 4 * L::kBBands * chunk, (kt > 0 || j > 0) ? 1u : 0u);
                }
                tc_commit(&empty[s]);
            }
            tc_commit(acc_full);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const bool ok = mbar_wait_bounded(acc_full, 0, p.wait_limit_ns, SITE_GEMM_EPI_ACC, abort_flag);
        tc_fence_after();
        if (ok && !*abort_flag) {
            const int row = m0 + 32 * q + lane;
            float scale = 1.0f;
            if (FMT == 3) scale = (*p.ga) * (*p.gb);
            uint32_t amax = 0;
            const bool vec_ok = ((p.ldc & 7) == 0) && ((reinterpret_cast<uintptr_t>(p.C) & 15) == 0);
            for (int c0 = 0; c0 < BN; c0 += 32) {
                if (n0 + c0 >= p.N) break;  // warp-uniform
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, r);
                tmem_wait_ld();
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float x0 = __uint_as_float(r[2 * i]) * scale, x1 = __uint_as_float(r[2 * i + 1]) * scale;
                    if (p.epilogue == 1) {
                        x0 = gelu_erf(x0);
                        x1 = gelu_erf(x1);
                    }
                    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
                    packed[i] = *reinterpret_cast<const uint32_t *>(&h);
                }
                if (p.amax_out != nullptr && row < p.M) {
                    const int valid = min(32, p.N - (n0 + c0));
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < valid) amax = max(amax, (packed[i >> 1] >> (16 * (i & 1))) & 0x7FFFu);
                }
                if (row < p.M) {
                    uint16_t *dst = p.C + (int64_t)row * p.ldc + n0 + c0;
                    if (vec_ok && n0 + c0 + 32 <= p.N) {
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            reinterpret_cast<uint4 *>(dst)[v] =
                                make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                    } else {
                        for (int i = 0; i < 32 && n0 + c0 + i < p.N; ++i)
                            dst[i] = (uint16_t)(packed[i >> 1] >> (16 * (i & 1)));
                    }
                }
            }
            if (p.amax_out != nullptr) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (lane == 0 && amax != 0u) atomicMax(reinterpret_cast<unsigned int *>(p.amax_out), amax << 16);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        // All MMAs issued by this CTA have completed once acc_full has fired.
        mbar_wait_bounded(acc_full, 0, p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

}  // namespace mx
