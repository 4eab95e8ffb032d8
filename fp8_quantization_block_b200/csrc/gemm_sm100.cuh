// gemm_sm100.cuh -- block-scaled GEMM on the sm_100a tensor cores (tcgen05).
//
// C[M x N] (bf16) = A_dq [M x K] * B_dq [N x K]^T, where A and B are stored as
// microscaling codes plus per-block scales ([MX] page "Microscaling MXFP4/NVFP4
// on Blackwell", section "Arquitetura Blackwell SM100 e aceleração nativa de
// NVFP4": the 5th-generation tensor core consumes the block codes directly and
// applies the block scale during FP32 accumulation).
//
// Persistent kernel: one CTA per SM walks its work units (ksplit.cuh: output
// tiles of 128 x BN, t, t + gridDim.x, ..., and with a split plan pieces of
// the last wave's tiles along K) with six warp roles:
//   warp 0     TMA producer of the code tiles of A and B (128-byte swizzled,
//              K-major) into a STAGES-deep smem ring that runs continuously
//              across tiles;
//   warp 10    TMA producer of the 512-byte scale tiles: one 3D copy per
//              operand brings kSfGroup stages' tiles (all of B's bands) into
//              a ring of its own, ahead of the scale warps;
//   warps 6-9  scale warps (one per TMEM lane quadrant): copy each stage's
//              scale tiles from shared memory into one of the TMEM scale slots
//              with tcgen05.st, as soon as the MMAs that read the slot's
//              previous contents have completed.  (Staging the scales with
//              tcgen05.cp instead costs tensor-pipe cycles that do not overlap
//              the MMAs; register stores from other warps do.)
//   warp 11    gate: waits for each stage's code tiles and scale slot and
//              publishes the count of ready stages in shared memory, so that
//              the MMA issuer reads one word (rarely, as it runs behind)
//              instead of waiting on two mbarriers per stage, whose latency
//              would leave the tensor pipe idle between stages;
//   warp 1     TMEM owner and MMA issuer: one lane issues the block-scaled
//              tcgen05.mma instructions (4 per stage, 32 bytes of K each) into
//              an FP32 accumulator in TMEM once a stage's code tiles and scale
//              slot are ready; tcgen05.commit frees the smem stage and the slot;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (one row per thread),
//              x gA*gB for NVFP4, optional GELU and |C| max, bf16 RNE, staged
//              in shared memory and written with TMA bulk-tensor stores.
// The two accumulators alternate between tiles so that the epilogue of one
// tile overlaps the MMAs of the next.  TMEM has 512 columns: the accumulators
// sit at [0, BN) and [S, S + BN) and share BN - S columns, which the epilogue
// drains first and then releases; the scale slots take the columns from
// S + BN up.  Every mbarrier wait is bounded (mx_common.cuh).
#pragma once

#include "ksplit.cuh"
#include "mx_common.cuh"
#include "quantize.cuh"

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
// kind::mxf8f6f4 with each operand's element type chosen at run time
// (GemmParams::ab_types): MXFP6 E3M2 and mixed MX operands (E4M3 / E5M2 /
// E3M2 / E2M1 on either side).  FP6 and FP4 codes arrive in shared memory
// unpacked by the tensor-map copy to one 16-byte group per 16 elements, so a
// stage is 128 elements = 128 bytes per row for every type, as for FP8.
constexpr int kGemmRuntimeTypes = 4;
template <>
struct GemmFmt<kGemmRuntimeTypes> {
    static constexpr int kElemPerByte = 1, kBlock = 32, kChunks = 1, kMmaPerChunk = 4, kSfPerMma = 1;
    static constexpr uint32_t kAFmt = 0, kScaleUE8M0 = 1;
};
// Element-type fields of the kind::mxf8f6f4 instruction descriptor.
enum : uint32_t { kTypeE4M3 = 0, kTypeE5M2 = 1, kTypeE3M2 = 4, kTypeE2M1 = 5 };

constexpr int kBM = 128;
constexpr int kStageKBytes = 128;
constexpr int kGemmThreads = 384;  // 12 warps
constexpr int kSfWarp = 10;        // the scale-tile producer
constexpr int kGateWarp = 11;      // publishes how many stages the MMA issuer may consume
constexpr int kSfSlots = 4;        // TMEM scale slots (the layouts may use more, see kSlots)
constexpr int kSfGroup = 2;        // stages per scale-tile copy
constexpr int kEpiWarps = 4;
constexpr int kEpiChunkBytes = 32 * 32 * 2;  // 32 rows x 32 bf16 columns per epilogue warp
constexpr int kSmemLimit = 232448;           // dynamic shared memory per CTA (opt-in maximum)

struct GemmParams {
    int64_t sf_tiles_k;   // 512-byte scale tiles per 128-row band (= ceil(K / block / 4))
    uint16_t *C;          // used by the direct-store epilogue (when TMA stores are not possible)
    int64_t ldc;
    int M, N, K;
    int num_kt;           // stages along K = ceil(K_bytes / 128)
    int m_blocks, n_blocks;
    const float *ga;      // NVFP4 per-tensor scales (nullptr for MX)
    const float *gb;
    float *amax_out;      // nullable: max |C| (bf16) via atomicMax on float bits
    int epilogue;         // 0 none, 1 GELU
    int use_tma_store;    // 1: C via TMA bulk-tensor stores (ldc % 8 == 0, C 16-B aligned)
    int skip_producer;    // test hook: never issue loads
    uint32_t ab_types;    // kGemmRuntimeTypes: (A type << 7) | (B type << 10) of the descriptor
    uint32_t stage_tx;    // kGemmRuntimeTypes: bytes one stage's code copies report to this CTA's
                          // barrier (the packed global bytes of FP6 / FP4 boxes, not their
                          // unpacked shared-memory footprint)
    uint64_t wait_limit_ns;
    int ga_from_amax;     // NVFP4: *ga holds amax(|A|) and gA = RU(amax / 2688) (1 for 0)
    int band_major;       // tile order: 1 = N fastest (consecutive tiles share A's band), 0 = M fastest
    // Fused activation quantize.  A is the bf16 matrix x [M x K] (row pitch
    // ldx) quantized to format x_fmt into xq_codes / xq_scales, which the TMA
    // producers read once band_ready[b] of A's 128-row band b has reached
    // x_band_target:
    //   fused == 1: by the epilogue warps of every CTA before their first tile
    //     (fused_quantize_role); work unit 32 rows x 128 columns of x (one
    //     warp's), handed out by next_item in band-major order;
    //   fused == 2: by the quantize kernel just before this one in the stream,
    //     one count per 128 x 128 CTA of it; this kernel then starts without
    //     waiting for that grid to complete (griddepcontrol.wait), so its CTAs
    //     work on the bands already written while the quantize still runs.
    int fused;
    uint32_t x_band_target;
    int x_fmt;
    int x_items_k;        // 128-column tiles per band = ceil(K / 128)
    int x_bands;          // ceil(M / 128)
    int64_t ldx;
    int64_t x_sf_tiles_k; // 512-byte scale chunks per band of x's format
    const uint16_t *x;
    uint8_t *xq_codes;
    uint8_t *xq_scales;
    uint32_t *band_ready;
    uint32_t *next_item;
    // Work schedule (ksplit.cuh): whole tiles, and with ks.on the tiles of
    // the last wave split along K.  Partial sums go to ks_partials, slot
    // worker (x 2 + rank on CTA pairs), in 4 KB blocks (ks_block);
    // ks_flags[slot] reaches kSplitSlotDone once the slot is written.
    KSplitPlan ks;
    float *ks_partials;
    uint32_t *ks_flags;
    int ks_slot_quads;    // 32-row quadrants of a slot (of the rows that exist)
};

// gA of an NVFP4 A operand (the epilogue multiplies by gA * gB).
MX_DEVICE_INLINE float gemm_ga(const GemmParams &p) { return nv_g_from(p.ga, p.ga_from_amax); }

// Fused quantize: wait until every 128 x 128 tile of A's 128-row band `band`
// is written (lane 0 polls, the warp learns the outcome); bands past x's end
// (the second half of a ragged CTA pair's rows) have nothing to wait for.
MX_DEVICE_INLINE bool wait_band_ready(const GemmParams &p, int band, int lane, volatile int *abort_flag) {
    bool ok = true;
    if (band < p.x_bands && lane == 0)
        ok = wait_global_at_least(p.band_ready + band, p.x_band_target, p.wait_limit_ns, SITE_FUSED_BAND_READY,
                                  abort_flag);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}


// Shared-memory and TMEM plan of a CTA whose MMAs read a 128-row A tile and
// B_BANDS 128-row bands of B per stage (B_ROWS rows of B in this CTA's smem).
// A_ROWS < 128 (matrices with at most A_ROWS rows, e.g. decode-time
// activations): only A_ROWS rows of A are loaded per stage, and the smem they
// leave free holds more stages of B.  The M = 128 MMA still reads 128 rows
// from the stage's base; the rows past A_ROWS are whatever the following
// shared memory holds and only produce accumulator rows >= M, which the
// epilogue neither stores nor counts.
template <int FMT, int B_BANDS, int B_ROWS, int STAGES, int A_ROWS = kBM>
struct GemmLayout {
    using F = GemmFmt<FMT>;
    static_assert(A_ROWS % 8 == 0 && A_ROWS <= kBM, "A rows: whole 8-row swizzle atoms");
    static constexpr int kBBands = B_BANDS;
    static constexpr int kARows = A_ROWS;
    static constexpr int kABytes = A_ROWS * kStageKBytes;
    static constexpr int kBBytes = B_ROWS * kStageKBytes;
    // scale tiles of one group: kSfGroup stages x kChunks 512-byte tiles of A's
    // band, and the same for each of B's bands (band-major)
    static constexpr int kSfaGroupBytes = kSfGroup * F::kChunks * 512;
    static constexpr int kSfbGroupBytes = kSfaGroupBytes * B_BANDS;
    static constexpr int kSfBandStride = kSfaGroupBytes;
    // TMEM scale slots in the ring: a slot is rewritten once the MMAs of the
    // stage kSlots earlier have completed, so more slots hide more of that
    // round trip (commit -> scale warps -> gate -> MMA issuer).  FP8-type
    // stages (one scale chunk) with 6 or more smem stages take 6 slots; the
    // FP4 kinds, whose slots are 2-4x wider, keep 4 so that TMEM still holds
    // the two accumulators.
    static constexpr int kSlots = (F::kChunks == 1 && STAGES >= 6)
                                      ? 6
                                      // FP4 kinds: 6 slots where they fit beside two whole accumulators
                                      : ((STAGES >= 6 && 2 * 128 * B_BANDS + 6 * 4 * F::kChunks * (1 + B_BANDS) <= 512)
                                             ? 6
                                             : kSfSlots);
    // full[S], empty[S], sfload[G], sfree[G], acc_full[2], acc_empty, mma_done, sf_full[slots]
    static constexpr int bytes_for(int groups, int bufs) {
        return STAGES * (kABytes + kBBytes) + groups * (kSfaGroupBytes + kSfbGroupBytes) +
               kEpiWarps * bufs * kEpiChunkBytes + (2 * STAGES + 2 * groups + 4 + kSlots) * 8 + 16 + 1024;
    }
    // as many scale groups in flight, then epilogue staging buffers, as fit
    static constexpr int kSfGroups = bytes_for(4, 2) <= kSmemLimit ? 4 : (bytes_for(3, 1) <= kSmemLimit ? 3 : 2);
    static constexpr int kEpiBufs = bytes_for(kSfGroups, 2) <= kSmemLimit ? 2 : 1;
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + STAGES * kABytes;
    static constexpr int kOffEpi = kOffB + STAGES * kBBytes;
    static constexpr int kOffSfa = kOffEpi + kEpiWarps * kEpiBufs * kEpiChunkBytes;
    static constexpr int kOffSfb = kOffSfa + kSfGroups * kSfaGroupBytes;
    static constexpr int kOffBar = kOffSfb + kSfGroups * kSfbGroupBytes;
    static constexpr int kNumBars = 2 * STAGES + 2 * kSfGroups + 4 + kSlots;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
    static_assert(kAlloc <= kSmemLimit, "shared memory budget");
    // the last stage's 128-row A read stays inside the allocation
    static_assert(kOffA + (STAGES - 1) * kABytes + kBM * kStageKBytes <= kBytes, "A tile read past the smem plan");
    // TMEM: two accumulators at columns 0 and kAccStride (sharing BN - kAccStride
    // columns), then kSlots scale slots of kSfSlotCols columns each.
    static constexpr int kAccCols = 128 * B_BANDS;  // accumulator columns = N of the MMA
    static constexpr int kTmemCols = 512;
    static constexpr int kSfSlotCols = 4 * F::kChunks * (1 + B_BANDS);
    static constexpr int kAccRoom = kTmemCols - kAccCols - kSlots * kSfSlotCols;
    static constexpr int kAccStride = (kAccRoom >= kAccCols ? kAccCols : kAccRoom) / 32 * 32;
    static constexpr int kTmemSf = kAccStride + kAccCols;
    static_assert(kAccStride >= 32, "accumulator double buffering needs TMEM room");
    static_assert(kTmemSf + kSlots * kSfSlotCols <= kTmemCols, "TMEM budget");
    static_assert(STAGES >= kSlots, "scale slots are recycled through the stage barriers");
    static constexpr int kEpiAreaBytes = kEpiWarps * kEpiBufs * kEpiChunkBytes;
};

template <int FMT, int BN, int STAGES, int A_ROWS = kBM>
using GemmSmem = GemmLayout<FMT, BN / 128, BN, STAGES, A_ROWS>;

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
    if (FMT <= 1 || FMT == kGemmRuntimeTypes) tc_mma_mxf8f6f4(d, a, b, idesc, sfa, sfb, acc);
    else if (FMT == 2) tc_mma_mxf4(d, a, b, idesc, sfa, sfb, acc);
    else tc_mma_nvf4(d, a, b, idesc, sfa, sfb, acc);
}

template <int FMT>
MX_DEVICE_INLINE void gemm_mma_if(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                  uint32_t acc, uint32_t issue) {
    if (FMT <= 1 || FMT == kGemmRuntimeTypes) tc_mma_mxf8f6f4_if(d, a, b, idesc, sfa, sfb, acc, issue);
    else if (FMT == 2) tc_mma_mxf4_if(d, a, b, idesc, sfa, sfb, acc, issue);
    else tc_mma_nvf4_if(d, a, b, idesc, sfa, sfb, acc, issue);
}

// Instruction descriptor of the CTA-pair MMA (M = 256 over two CTAs, N = BN).
template <int FMT, int BN = 256>
MX_DEVICE_INLINE uint32_t pair_idesc(uint32_t sf_id) {
    using F = GemmFmt<FMT>;
    return (sf_id << 4) | (F::kAFmt << 7) | (F::kAFmt << 10) | ((uint32_t)(BN >> 3) << 17) |
           (F::kScaleUE8M0 << 23) | ((uint32_t)(256 >> 4) << 24) | (sf_id << 29);
}

template <int FMT>
MX_DEVICE_INLINE void pair_mma_if(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                  uint32_t acc, uint32_t issue) {
    if (FMT <= 1 || FMT == kGemmRuntimeTypes) tc_mma_pair_mxf8f6f4_if(d, a, b, idesc, sfa, sfb, acc, issue);
    else if (FMT == 2) tc_mma_pair_mxf4_if(d, a, b, idesc, sfa, sfb, acc, issue);
    else tc_mma_pair_nvf4_if(d, a, b, idesc, sfa, sfb, acc, issue);
}

// Issue the MMAs of one stage (n_mma 32-byte K steps: 4, fewer only in a
// ragged last stage).  ad / bd: descriptors of the stage's A / B tiles;
// consecutive K steps are 32 bytes (2 descriptor units) apart inside the
// 128-byte swizzle atom.  SFB_STEP: TMEM columns per scale chunk of B (4 per
// 128-row band).  With n_mma == 4 the loop unrolls and every operand but the
// stage's bases folds to a constant, keeping the issuing thread's per-stage
// instruction chain short.  ab: run-time element-type bits of the descriptor
// (0 for the formats whose types are fixed at compile time).
template <int FMT, bool PAIR, int BN, int SFB_STEP>
MX_DEVICE_INLINE void issue_one(int j, uint32_t t_acc, uint64_t ad, uint64_t bd, uint32_t t_sfa, uint32_t t_sfb,
                                uint32_t acc, uint32_t issue, uint32_t ab) {
    using F = GemmFmt<FMT>;
    const int chunk = j / F::kMmaPerChunk;
    const uint32_t sf_id = (uint32_t)((j % F::kMmaPerChunk) * F::kSfPerMma);
    const uint32_t a = acc | (j > 0 ? 1u : 0u);
    if (PAIR)
        pair_mma_if<FMT>(t_acc, ad + 2u * j, bd + 2u * j, pair_idesc<FMT, BN>(sf_id) | ab, t_sfa + 4 * chunk,
                         t_sfb + SFB_STEP * chunk, a, issue);
    else
        gemm_mma_if<FMT>(t_acc, ad + 2u * j, bd + 2u * j, gemm_idesc<FMT, BN>(sf_id) | ab, t_sfa + 4 * chunk,
                         t_sfb + SFB_STEP * chunk, a, issue);
}

template <int FMT, bool PAIR, int BN, int SFB_STEP>
MX_DEVICE_INLINE void issue_stage(int n_mma, uint32_t t_acc, uint64_t ad, uint64_t bd, uint32_t t_sfa, uint32_t t_sfb,
                                  uint32_t acc, uint32_t issue, uint32_t ab) {
    if (n_mma == 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) issue_one<FMT, PAIR, BN, SFB_STEP>(j, t_acc, ad, bd, t_sfa, t_sfb, acc, issue, ab);
    } else {
        for (int j = 0; j < n_mma; ++j) issue_one<FMT, PAIR, BN, SFB_STEP>(j, t_acc, ad, bd, t_sfa, t_sfb, acc, issue, ab);
    }
}

// GELU of two values at once, the exact-erf form GELU(x) = x Phi(x), with
// Phi(x) = 1 - h for x > 0 and h for x <= 0, h = erfc(|x| / sqrt 2) / 2.
// erfc(z) = t exp(-z^2 + P(t)), t = 1 / (1 + z / 2), with P the degree-5
// polynomial a0 + a1 t + ... + a5 t^5 fitted to log(erfc(z) / t) + z^2 over
// z in [0, 10] (least squares reweighted towards the minimax fit):
//   a = -1.266541613, 1.018012027, 0.2544491856, 0.4744819897,
//       -0.7091808945, 0.22878691,  |P(t) - (log(erfc(z)/t) + z^2)| < 7.7e-6,
// so erfc's relative error is below 7.7e-6 plus the fp32 rounding.  The
// constants fold the steps: u = |x| sqrt(log2(e) / 2), so that u^2 = z^2
// log2(e); t / 2 = 1 / (2 + u / sqrt(log2 e)) from one reciprocal; the
// polynomial in t / 2 has the coefficients log2(e) 2^i a_i; then
// h = (t / 2) 2^(P' - u^2) with the hardware's base-2 exponential.  Emulated
// in fp32 against an fp64 GELU over [-16, 16]: relative error below 2e-5, and
// the bf16 result at most one ulp from the correctly rounded one (0.05% of
// the values differ).  Branch-free; the polynomial runs on packed f32x2 fmas
// for both values.
constexpr float kGeluU = 0.849321783f;   // sqrt(log2(e) / 2)
constexpr float kGeluT = 0.832554638f;   // 1 / sqrt(log2(e))
MX_DEVICE_INLINE void gelu_erf2(float &x0, float &x1) {
    const float u0 = fabsf(x0) * kGeluU, u1 = fabsf(x1) * kGeluU;
    float t0, t1;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t0) : "f"(fmaf(u0, kGeluT, 2.0f)));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t1) : "f"(fmaf(u1, kGeluT, 2.0f)));
    const uint64_t T = pk2(t0, t1);   // t / 2
    uint64_t P = fma2(pk2(10.562232f, 10.562232f), T, pk2(-16.3701077f, -16.3701077f));
    P = fma2(P, T, pk2(5.47626257f, 5.47626257f));
    P = fma2(P, T, pk2(1.46837032f, 1.46837032f));
    P = fma2(P, T, pk2(2.93736172f, 2.93736172f));
    P = fma2(P, T, pk2(-1.82723331f, -1.82723331f));
    P = fma2(pk2(-u0, -u1), pk2(u0, u1), P);
    float a0, a1;
    upk2(P, a0, a1);
    float e0, e1;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(a0));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(a1));
    // x h for both values, then x - x h where x > 0
    float g0, g1;
    upk2(mul2(pk2(x0, x1), mul2(T, pk2(e0, e1))), g0, g1);
    x0 = x0 > 0.0f ? x0 - g0 : g0;
    x1 = x1 > 0.0f ? x1 - g1 : g1;
}

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


// Scale warps: move one stage's scale tiles from shared memory into a TMEM
// slot of this warp's 32 lanes.  Lane r loads row r (16 bytes = 4 columns) of
// every 512-byte tile first, then writes them with wide tcgen05.st.  Slot
// layout: A tiles c at columns 4c; B tiles (c, band h) at 4*kChunks + 4*(c*bands + h).
// smem B tiles of band h start BAND_STRIDE bytes after those of band h - 1.
template <int CHUNKS, int BANDS, int BAND_STRIDE>
MX_DEVICE_INLINE void stage_scales_to_tmem(const uint8_t *sfa_stage, const uint8_t *sfb_stage, uint32_t t_slot,
                                           int lane) {
    uint32_t a[4 * CHUNKS];
    uint32_t b[4 * CHUNKS * BANDS];
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
        const uint4 v = *reinterpret_cast<const uint4 *>(sfa_stage + c * 512 + lane * 16);
        a[4 * c] = v.x, a[4 * c + 1] = v.y, a[4 * c + 2] = v.z, a[4 * c + 3] = v.w;
#pragma unroll
        for (int h = 0; h < BANDS; ++h) {
            const uint4 w = *reinterpret_cast<const uint4 *>(sfb_stage + h * BAND_STRIDE + c * 512 + lane * 16);
            const int o = 4 * (c * BANDS + h);
            b[o] = w.x, b[o + 1] = w.y, b[o + 2] = w.z, b[o + 3] = w.w;
        }
    }
    if (CHUNKS == 4) {
        tmem_st16(t_slot, *reinterpret_cast<const uint32_t(*)[16]>(&a[0]));
    } else if (CHUNKS == 2) {
        tmem_st8(t_slot, *reinterpret_cast<const uint32_t(*)[8]>(&a[0]));
    } else {
        tmem_st4(t_slot, a[0], a[1], a[2], a[3]);
    }
    constexpr int kB = 4 * CHUNKS * BANDS;  // 4, 8, 16 or 32 columns
    const uint32_t tb = t_slot + 4 * CHUNKS;
    if (kB == 32) {
        tmem_st16(tb, *reinterpret_cast<const uint32_t(*)[16]>(&b[0]));
        tmem_st16(tb + 16, *reinterpret_cast<const uint32_t(*)[16]>(&b[(kB == 32) ? 16 : 0]));
    } else if (kB == 16) {
        tmem_st16(tb, *reinterpret_cast<const uint32_t(*)[16]>(&b[0]));
    } else if (kB == 8) {
        tmem_st8(tb, *reinterpret_cast<const uint32_t(*)[8]>(&b[0]));
    } else {
        tmem_st4(tb, b[0], b[1], b[2], b[3]);
    }
    tmem_wait_st();
}

// ---------------------------------------------------------------- work units
// The work units of worker c (ksplit.cuh).  Kernels compiled without SPLIT
// run whole tiles c, c + workers, ... with K stages [0, num_kt): constant
// bounds, and none of the split's branches in their loops.
template <bool SPLIT>
MX_DEVICE_INLINE int unit_count(const GemmParams &p, int c) {
    if (SPLIT) return ks_units(p.ks, c);
    return c < p.ks.tiles ? (p.ks.tiles - c + p.ks.workers - 1) / p.ks.workers : 0;
}
template <bool SPLIT>
MX_DEVICE_INLINE KUnit unit_at(const GemmParams &p, int c, int u) {
    if (SPLIT) return ks_unit(p.ks, c, u);
    KUnit r;
    r.tile = c + u * p.ks.workers;
    r.kb = 0;
    r.ke = p.num_kt;
    r.kind = kUnitWhole;
    r.first = c;
    return r;
}
template <bool SPLIT>
MX_DEVICE_INLINE int unit_stages(const GemmParams &p, int c) {
    return SPLIT ? ks_stages(p.ks, c) : unit_count<false>(p, c) * p.num_kt;
}

// ---------------------------------------------------------------- scale-tile roles
// Producer of scale tiles (one warp; lane 0 issues): for each work unit of
// this worker (bands_of(tile, a_band, b_band)), one 3D TMA copy per operand
// and group of kSfGroup stages into ring slot g, once the scale warps have
// freed it.
// Coordinates past the scale buffer (a ragged K or N) read zeros.
template <typename L, bool SPLIT, typename BandsOf>
MX_DEVICE_INLINE void sf_producer_role(const GemmParams &p, const CUtensorMap *tmSfa, const CUtensorMap *tmSfb,
                                       uint8_t *smem, uint64_t *sfload, uint64_t *sfree, int worker,
                                       BandsOf bands_of, int lane, volatile int *abort_flag) {
    constexpr int NG = L::kSfGroups;
    constexpr int kChunks = L::F::kChunks;
    int used = 0, g = 0;
    uint32_t ph = 0;
    bool stop = false;
    int ready_band = -1;   // fused quantize: the last A band known to be written
    const int n_units = unit_count<SPLIT>(p, worker);
    for (int u = 0; u < n_units && !stop; ++u) {
        const KUnit U = unit_at<SPLIT>(p, worker, u);
        int a_band, b_band;
        bands_of(U.tile, a_band, b_band);
        if (p.fused && a_band != ready_band) {
            if (!wait_band_ready(p, a_band, lane, abort_flag)) {
                stop = true;
                break;
            }
            ready_band = a_band;
        }
        for (int kt0 = U.kb; kt0 < U.ke; kt0 += kSfGroup) {   // U.kb is even
            if (!mbar_wait_bounded(&sfree[g], ph ^ 1u, p.wait_limit_ns, SITE_GEMM_SF_FREE, abort_flag)) {
                stop = true;
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&sfload[g], (uint32_t)(L::kSfaGroupBytes + L::kSfbGroupBytes));
                tma_load_3d(smem + L::kOffSfa + g * L::kSfaGroupBytes, tmSfa, 0, kt0 * kChunks, a_band, &sfload[g]);
                tma_load_3d(smem + L::kOffSfb + g * L::kSfbGroupBytes, tmSfb, 0, kt0 * kChunks, b_band, &sfload[g]);
            }
            __syncwarp();
            ++used;
            if (++g == NG) {
                g = 0;
                ph ^= 1u;
            }
        }
    }
    // Do not leave while copies into shared memory are in flight.
    for (int u = max(0, used - NG); u < used; ++u)
        mbar_wait_bounded(&sfload[u % NG], (uint32_t)((u / NG) & 1), p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
}

// Scale warps (one per TMEM lane quadrant; lane r handles TMEM lane 32q + r):
// for every stage of this worker's units, wait for its scale group in smem and
// for the MMAs that last read the TMEM slot (stage kg - L::kSlots, whose
// commit completes empty[]), then write the slot and report it with
// arrive_full(slot).  After a group's last stage the warp frees the group.
// (Writing a group's two stages with one wait for the stores was measured
// slower: the second slot's wait for older MMAs costs more than the store
// latency it hides.)  before_wait(kg) runs just before the wait for stage
// kg - L::kSlots; the kernels use it to drain accumulator columns whose
// release that stage's MMAs may be waiting for.
template <typename L, int STAGES, bool SPLIT, typename ArriveFull, typename BeforeWait>
MX_DEVICE_INLINE void scale_role(const GemmParams &p, uint8_t *smem, uint64_t *sfload, uint64_t *sfree, uint64_t *empty,
                                 uint32_t t_sf0, int worker, int lane, volatile int *abort_flag,
                                 ArriveFull arrive_full, BeforeWait before_wait) {
    constexpr int NG = L::kSfGroups;
    constexpr int kChunks = L::F::kChunks;
    int g = 0, slot = 0, e = 0;
    uint32_t gph = 0, eph = 0;
    int kg = 0;
    bool stop = false;
    const int n_units = unit_count<SPLIT>(p, worker);
    for (int u = 0; u < n_units && !stop; ++u) {
        const KUnit U = unit_at<SPLIT>(p, worker, u);
        for (int kt = U.kb; kt < U.ke; ++kt, ++kg) {
            const int gi = kt % kSfGroup;
            if (gi == 0 && !mbar_wait_bounded(&sfload[g], gph, p.wait_limit_ns, SITE_GEMM_SF_LOAD, abort_flag)) {
                stop = true;
                break;
            }
            if (kg >= L::kSlots) {
                // stage kg reuses the slot of stage kg - kSlots: hand the wait's idle
                // time to before_wait first (false: give up, as on a timeout)
                if (!before_wait(kg) ||
                    !mbar_wait_bounded(&empty[e], eph, p.wait_limit_ns, SITE_GEMM_SF_EMPTY, abort_flag)) {
                    stop = true;
                    break;
                }
                if (++e == STAGES) {
                    e = 0;
                    eph ^= 1u;
                }
            }
            tc_fence_after();
            stage_scales_to_tmem<kChunks, L::kBBands, L::kSfBandStride>(
                smem + L::kOffSfa + g * L::kSfaGroupBytes + gi * kChunks * 512,
                smem + L::kOffSfb + g * L::kSfbGroupBytes + gi * kChunks * 512, t_sf0 + (uint32_t)(slot * L::kSfSlotCols),
                lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_full(slot);
            slot = (slot + 1 == L::kSlots) ? 0 : slot + 1;
            if (gi == kSfGroup - 1 || kt == U.ke - 1) {
                if (lane == 0) mbar_arrive(&sfree[g]);
                if (++g == NG) {
                    g = 0;
                    gph ^= 1u;
                }
            }
        }
    }
}

// Origin of output tile `tile` (bm x bn tiles): M-fastest order, or N-fastest
// (band-major) when the fused quantize produces A band by band.
MX_DEVICE_INLINE void tile_coords(const GemmParams &p, int tile, int &m0, int &n0, int bm, int bn) {
    int mb, nb;
    if (p.band_major) {
        mb = tile / p.n_blocks;
        nb = tile - mb * p.n_blocks;
    } else {
        mb = tile % p.m_blocks;
        nb = tile / p.m_blocks;
    }
    m0 = mb * bm;
    n0 = nb * bn;
}

// Shared memory of the fused quantize, inside the epilogue warps' staging
// buffers (idle until their first tile): each warp's scale chunks of the rows
// it is quantizing, and the NVFP4 tables.
struct FusedQuantSmem {
    uint8_t sf[kEpiWarps][1024];
    NvTables nvt;
};

// Work items of the fused quantize: 32 rows x 128 columns of x, one warp's
// (quadrant q of the 128 x 128 tile (band, tile_x)); item
// ((band * x_items_k) + tile_x) * 4 + q, handed out in that order, so bands
// complete in order.  A band is written once x_items_k * 4 items are counted.
constexpr int kFusedQuads = kQTileRows / 32;

// Each epilogue warp (w = 0..3) of a CTA: claim items from the global counter
// until none is left, quantize each (tile_load / tile_quantize: the arithmetic
// of quantize_kernel, so codes and scales are those of mx_quantize), write its
// rows' scale bytes and count it in its band.  The four warps run independent
// pipelines (no barrier between them until the end), and each issues its next
// item's loads as soon as this item's values are consumed, so they fly while
// this item is published.  Nothing here waits on another CTA, so the items get done as long
// as any CTA of the grid runs.
template <int XFMT>
MX_DEVICE_INLINE void fused_quantize_role_t(const GemmParams &p, FusedQuantSmem *fq, int t) {
    const int w = t >> 5, lane = t & 31;
    NvScale ns{1.0f, 1.0f, 1.0f, 1.0f, 1.0f};
    if (XFMT == FMT_NVFP4) {
        ns = nv_scale_setup(nv_g_from(p.ga, p.ga_from_amax));
        nv_tables_fill(&fq->nvt, (uint32_t)t);
        sync_epilogue_warps();
    }
    constexpr int kChunks = quantize_sf_bytes<XFMT>() / 512;
    uint8_t *sf = fq->sf[w];
    const uint32_t items_k = (uint32_t)p.x_items_k;
    const uint32_t n_items = (uint32_t)p.x_bands * items_k * kFusedQuads;
    uint32_t cur = 0;
    if (lane == 0) cur = atomicAdd(p.next_item, 1u);
    cur = __shfl_sync(0xffffffffu, cur, 0);
    TileRegs<32, 32> r;
    auto rows_of = [&](uint32_t item, int64_t &band, int64_t &tx, int &q) {
        q = (int)(item % kFusedQuads);
        const uint32_t tile = item / kFusedQuads;
        band = tile / items_k;
        tx = tile % items_k;
    };
    int64_t band, tx;
    int q;
    if (cur < n_items) {
        rows_of(cur, band, tx, q);
        tile_load<32, 32>(r, p.x, p.M, p.K, p.ldx, band * kQTileRows + q * 32, tx * kQTileCols, lane);
    }
    while (cur < n_items) {
        rows_of(cur, band, tx, q);
        uint32_t nxt = 0;
        if (lane == 0) nxt = atomicAdd(p.next_item, 1u);   // its latency hides behind this item's arithmetic
        tile_quantize<XFMT, 32, 32>(r, p.M, p.K, band * kQTileRows, q * 32, tx * kQTileCols, ns, &fq->nvt,
                                    p.xq_codes, sf, lane);
        __syncwarp();
        // this warp's rows of the tile's scale chunks: row lane's 4 bytes of each chunk
        const int64_t chunk0 = band * p.x_sf_tiles_k + tx * kChunks, chunk_end = (band + 1) * p.x_sf_tiles_k;
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
            if (chunk0 + c < chunk_end)
                *reinterpret_cast<uint32_t *>(p.xq_scales + (chunk0 + c) * 512 + lane * 16 + q * 4) =
                    *reinterpret_cast<const uint32_t *>(sf + c * 512 + lane * 16 + q * 4);
        nxt = __shfl_sync(0xffffffffu, nxt, 0);
        if (nxt < n_items) {
            int64_t nb, ntx;
            int nq;
            rows_of(nxt, nb, ntx, nq);
            tile_load<32, 32>(r, p.x, p.M, p.K, p.ldx, nb * kQTileRows + nq * 32, ntx * kQTileCols, lane);
        }
        fence_proxy_async_global();   // this lane's stores, before the band count (TMA reads them)
        __syncwarp();
        if (lane == 0) red_release_gpu_add(p.band_ready + band, 1u);
        cur = nxt;
    }
    // the epilogue reuses this shared memory as staging buffers: no warp starts
    // its epilogue while another still quantizes
    sync_epilogue_warps();
}

template <int FMT>
MX_DEVICE_INLINE void fused_quantize_role(const GemmParams &p, FusedQuantSmem *fq, int t) {
    if constexpr (FMT == kGemmRuntimeTypes) {
        switch (p.x_fmt) {
        case FMT_E4M3: fused_quantize_role_t<FMT_E4M3>(p, fq, t); break;
        case FMT_E5M2: fused_quantize_role_t<FMT_E5M2>(p, fq, t); break;
        case FMT_MXFP4: fused_quantize_role_t<FMT_MXFP4>(p, fq, t); break;
        default: fused_quantize_role_t<FMT_MXFP6>(p, fq, t); break;
        }
    } else {
        fused_quantize_role_t<FMT>(p, fq, t);
    }
}

// Gate warp: for every stage of this CTA's work units (my_stages in all), in
// order, wait for its code tiles (full) and its scale slot (sf_full), then
// publish the number of stages ready so far.
template <int STAGES, int SLOTS>
MX_DEVICE_INLINE void gate_role(const GemmParams &p, uint64_t *full, uint64_t *sf_full, uint32_t *ready,
                                int my_stages, int lane, volatile int *abort_flag) {
    int s = 0, slot = 0;
    uint32_t fph = 0, sph = 0, k = 0;
    for (int kt = 0; kt < my_stages; ++kt) {
        if (!mbar_wait_bounded(&full[s], fph, p.wait_limit_ns, SITE_GEMM_MMA_FULL, abort_flag) ||
            !mbar_wait_bounded(&sf_full[slot], sph, p.wait_limit_ns, SITE_GEMM_MMA_SF, abort_flag))
            return;
        ++k;
        __syncwarp();
        if (lane == 0) st_release_shared(ready, k);
        if (++s == STAGES) {
            s = 0;
            fph ^= 1u;
        }
        if (++slot == SLOTS) {
            slot = 0;
            sph ^= 1u;
        }
    }
}

// ---------------------------------------------------------------- epilogue
// One 32-column chunk of this warp's 32 accumulator rows: TMEM -> registers,
// x scale (NVFP4: gA * gB), optional GELU, bf16 round-to-nearest-even.  The
// options are template parameters so that the unused paths cost no issue
// slots (the epilogue warps share schedulers with the MMA and scale warps).
template <bool SCALED, bool GELU>
MX_DEVICE_INLINE void epi_load_convert(uint32_t t_addr, float scale, uint32_t (&packed)[16]) {
    uint32_t r[32];
    tmem_ld32(t_addr, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float x0 = __uint_as_float(r[2 * i]), x1 = __uint_as_float(r[2 * i + 1]);
        if (SCALED) upk2(mul2(pk2(x0, x1), pk2(scale, scale)), x0, x1);
        if (GELU) gelu_erf2(x0, x1);
        const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
        packed[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
}

// Write one converted chunk (rows m0q + lane, columns n0 + col ..) and fold
// it into the running |C| maximum.  TMA stores go through NBUF staging
// buffers of this warp, so a store only waits for the one issued NBUF
// chunks earlier to have finished reading shared memory.
template <int NBUF>
MX_DEVICE_INLINE void epi_emit(const GemmParams &p, const CUtensorMap *tmC, const uint32_t (&packed)[16], int m0q,
                               int n0, int col, int lane, uint8_t *bufs, uint32_t &nstore, uint32_t &amax,
                               bool via_tma) {
    const int row = m0q + lane;
    const int n_valid = p.N - n0;
    if (p.amax_out != nullptr && row < p.M) {
        const int valid = min(32, n_valid - col);
        if (valid == 32) {
            uint32_t m2 = packed[0];
#pragma unroll
            for (int i = 1; i < 16; ++i)
                asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(m2) : "r"(packed[i]));
            m2 &= 0x7FFF7FFFu;
            amax = max(amax, max(m2 & 0xFFFFu, m2 >> 16));
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (i < valid) amax = max(amax, (packed[i >> 1] >> (16 * (i & 1))) & 0x7FFFu);
        }
    }
    if (m0q >= p.M) return;  // warp-uniform: no rows of this quadrant exist
    if (via_tma) {
        uint8_t *buf = bufs + (nstore % NBUF) * kEpiChunkBytes;
        if (lane == 0) bulk_wait_group_read<NBUF - 1>();  // this buffer's previous store has read it
        __syncwarp();
        uint4 *dst = reinterpret_cast<uint4 *>(buf + lane * 64);
#pragma unroll
        for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmC, n0 + col, m0q, buf);
            bulk_commit_group();
        }
        ++nstore;
    } else if (row < p.M) {
        uint16_t *dst = p.C + (int64_t)row * p.ldc + n0 + col;
        if (p.use_tma_store && col + 32 <= n_valid) {
            // C 16-byte aligned and ldc % 8 == 0 (the TMA store's conditions):
            // this row's 64 bytes as four 16-byte stores
            uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
            for (int v = 0; v < 4; ++v)
                d4[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (col + i < n_valid) dst[i] = (uint16_t)(packed[i >> 1] >> (16 * (i & 1)));
        }
    }
}

// With GELU, the chunks of an accumulator whose columns the next tile shares
// are drained by two warps per TMEM lane quadrant: the epilogue warp and the
// scale warp, which would otherwise sit waiting for the MMAs that this release
// holds back.  The scale warp takes this many of them (the last ones in
// drain order), through direct global stores (shared memory has no room for
// its own staging buffers).
template <int BN, int ACC_STRIDE>
__host__ __device__ constexpr int gelu_help_chunks() {
    return ((BN - ACC_STRIDE) / 32) / 2;
}

// Drain one accumulator tile (BN columns) for this warp's TMEM quadrant.  The
// two accumulator buffers share BN - ACC_STRIDE columns (buffer 0's tail is
// buffer 1's head), and the next tile's MMAs wait for release().  Without
// GELU those chunks are pulled into registers first, so release() runs
// before any store is issued and the tensor pipe idles only for the TMEM
// reads.
template <int BN, int ACC_STRIDE, int NBUF, bool SCALED, bool GELU, typename Release>
MX_DEVICE_INLINE void epilogue_tile_t(const GemmParams &p, const CUtensorMap *tmC, uint32_t t_acc, int b, int m0q,
                                      int n0, int lane, uint8_t *bufs, uint32_t &nstore, uint32_t &amax, float scale,
                                      Release release) {
    constexpr int kChunks = BN / 32;
    constexpr int kOv = (BN - ACC_STRIDE) / 32;
    static_assert(kOv >= 0 && kOv <= kChunks, "accumulator overlap");
    const int n_valid = p.N - n0;
    if constexpr (GELU) {
        // GELU needs more live registers per chunk: drain in order, releasing
        // after the shared chunks have been written out.  The last
        // gelu_help_chunks() shared chunks are the scale warp's (help_drain_t).
        constexpr int kMine = kOv - gelu_help_chunks<BN, ACC_STRIDE>();
        auto drain = [&](int idx) {
            const int col = 32 * ((b == 0) ? (idx + (kChunks - kOv)) % kChunks : idx);
            if (col >= n_valid) return;  // warp-uniform
            uint32_t packed[16];
            epi_load_convert<SCALED, GELU>(t_acc + (uint32_t)col, scale, packed);
            epi_emit<NBUF>(p, tmC, packed, m0q, n0, col, lane, bufs, nstore, amax, p.use_tma_store);
        };
        for (int idx = 0; idx < kMine; ++idx) drain(idx);
        tc_fence_before();
        __syncwarp();
        release();
        for (int idx = kOv; idx < kChunks; ++idx) drain(idx);
    } else {
        uint32_t ov[kOv > 0 ? kOv : 1][16];
#pragma unroll
        for (int i = 0; i < kOv; ++i) {
            const int col = 32 * ((b == 0) ? (kChunks - kOv + i) : i);
            if (col < n_valid) epi_load_convert<SCALED, GELU>(t_acc + (uint32_t)col, scale, ov[i]);
        }
        tc_fence_before();
        __syncwarp();
        release();
#pragma unroll
        for (int i = 0; i < kOv; ++i) {
            const int col = 32 * ((b == 0) ? (kChunks - kOv + i) : i);
            if (col < n_valid) epi_emit<NBUF>(p, tmC, ov[i], m0q, n0, col, lane, bufs, nstore, amax, p.use_tma_store);
        }
        for (int i = 0; i < kChunks - kOv; ++i) {
            const int col = 32 * ((b == 0) ? i : (kOv + i));
            if (col >= n_valid) break;  // warp-uniform; columns ascend
            uint32_t packed[16];
            epi_load_convert<SCALED, GELU>(t_acc + (uint32_t)col, scale, packed);
            epi_emit<NBUF>(p, tmC, packed, m0q, n0, col, lane, bufs, nstore, amax, p.use_tma_store);
        }
    }
}

// Chunks [c_begin, c_end) of 32 columns of an accumulator in plain order (no
// shared columns to release first): the last tile of a CTA, whose columns are
// split between the epilogue warp and the scale warp of each TMEM lane
// quadrant (the scale warps are idle once the tile's scales are in TMEM).
template <int NBUF, bool SCALED, bool GELU>
MX_DEVICE_INLINE void epilogue_chunks_t(const GemmParams &p, const CUtensorMap *tmC, uint32_t t_acc, int m0q, int n0,
                                        int c_begin, int c_end, int lane, uint8_t *bufs, uint32_t &nstore,
                                        uint32_t &amax, float scale) {
    const int n_valid = p.N - n0;
    for (int c = c_begin; c < c_end; ++c) {
        const int col = 32 * c;
        if (col >= n_valid) break;  // warp-uniform; columns ascend
        uint32_t packed[16];
        epi_load_convert<SCALED, GELU>(t_acc + (uint32_t)col, scale, packed);
        epi_emit<NBUF>(p, tmC, packed, m0q, n0, col, lane, bufs, nstore, amax, p.use_tma_store);
    }
}
template <int NBUF, bool SCALED>
MX_DEVICE_INLINE void epilogue_chunks(const GemmParams &p, const CUtensorMap *tmC, uint32_t t_acc, int m0q, int n0,
                                      int c_begin, int c_end, int lane, uint8_t *bufs, uint32_t &nstore,
                                      uint32_t &amax, float scale) {
    if (p.epilogue == 1)
        epilogue_chunks_t<NBUF, SCALED, true>(p, tmC, t_acc, m0q, n0, c_begin, c_end, lane, bufs, nstore, amax, scale);
    else
        epilogue_chunks_t<NBUF, SCALED, false>(p, tmC, t_acc, m0q, n0, c_begin, c_end, lane, bufs, nstore, amax, scale);
}

template <int BN, int ACC_STRIDE, int NBUF, bool SCALED, typename Release>
MX_DEVICE_INLINE void epilogue_tile(const GemmParams &p, const CUtensorMap *tmC, uint32_t t_acc, int b, int m0q,
                                    int n0, int lane, uint8_t *bufs, uint32_t &nstore, uint32_t &amax, float scale,
                                    Release release) {
    if (p.epilogue == 1)
        epilogue_tile_t<BN, ACC_STRIDE, NBUF, SCALED, true>(p, tmC, t_acc, b, m0q, n0, lane, bufs, nstore, amax, scale,
                                                            release);
    else
        epilogue_tile_t<BN, ACC_STRIDE, NBUF, SCALED, false>(p, tmC, t_acc, b, m0q, n0, lane, bufs, nstore, amax, scale,
                                                             release);
}

// The scale warp's share of a GELU tile's shared chunks (the last
// gelu_help_chunks() of them in epilogue_tile_t's drain order), written to C
// with direct stores; the caller releases the columns afterwards.
template <int BN, int ACC_STRIDE, bool SCALED>
MX_DEVICE_INLINE void help_drain_t(const GemmParams &p, uint32_t t_acc, int b, int m0q, int n0, int lane,
                                   uint32_t &amax, float scale) {
    constexpr int kChunks = BN / 32;
    constexpr int kOv = (BN - ACC_STRIDE) / 32;
    const int n_valid = p.N - n0;
    uint32_t unused = 0;
    for (int idx = kOv - gelu_help_chunks<BN, ACC_STRIDE>(); idx < kOv; ++idx) {
        const int col = 32 * ((b == 0) ? (idx + (kChunks - kOv)) % kChunks : idx);
        if (col >= n_valid) continue;  // warp-uniform
        uint32_t packed[16];
        epi_load_convert<SCALED, true>(t_acc + (uint32_t)col, scale, packed);
        epi_emit<1>(p, nullptr, packed, m0q, n0, col, lane, nullptr, unused, amax, false);
    }
}

// Flush this warp's stores and publish its |C| maximum.
MX_DEVICE_INLINE void epilogue_finish(const GemmParams &p, int lane, uint32_t amax) {
    if (lane == 0) bulk_wait_group_all();
    if (p.amax_out != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0 && amax != 0u) atomicMax(reinterpret_cast<unsigned int *>(p.amax_out), amax << 16);
    }
}

// ---------------------------------------------------------------- K split
// The counter of a partial-sum slot reaches kSplitSlotDone once every warp
// that writes part of the slot has published: the four epilogue warps with 2
// each, or, on the worker's last unit (whose columns the scale warps share),
// the four epilogue and four scale warps with 1 each.
constexpr uint32_t kSplitSlotDone = 8;

// A partial-sum slot is 8 chunks x ks_slot_quads quadrants of 4 KB blocks;
// block (chunk c, quadrant q) holds rows 32q .. 32q + 31 and columns 32c ..
// 32c + 31 as [c4 = 0 .. 7][row 0 .. 31][4 fp32]: a warp's store of four
// columns is 512 contiguous bytes, and the finishing warp brings the block
// into shared memory with one bulk copy, each lane then reading its row's
// 16-byte groups without bank conflicts.
constexpr int kSplitBlockBytes = 4096;
MX_DEVICE_INLINE float4 *ks_block(const GemmParams &p, int slot, int chunk, int q) {
    return reinterpret_cast<float4 *>(p.ks_partials) + ((size_t)(slot * 8 + chunk) * p.ks_slot_quads + q) * 256;
}

// One 32-column chunk of this warp's accumulator quadrant into its block of
// a partial-sum slot (L2-only stores: another SM reads them).
MX_DEVICE_INLINE void ks_store_chunk(const GemmParams &p, uint32_t t_addr, int slot, int chunk, int q, int lane) {
    uint32_t r[32];
    tmem_ld32(t_addr, r);
    tmem_wait_ld();
    float4 *d = ks_block(p, slot, chunk, q) + lane;
#pragma unroll
    for (int v = 0; v < 8; ++v)
        __stcg(d + 32 * v, make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                       __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
}

// Publish this warp's share of a written slot: every lane's stores are made
// visible at gpu scope (and to the async proxy) before lane 0 adds to the
// slot's counter.
MX_DEVICE_INLINE void ks_publish(const GemmParams &p, int slot, uint32_t share, int lane) {
    __threadfence();
    fence_proxy_async_global();   // the finishing warp reads the slot with bulk copies
    __syncwarp();
    if (lane == 0) red_release_gpu_add(p.ks_flags + slot, share);
}

// Wait (lane 0 polls, bounded) until the n slots slot0, slot0 + step, ... are
// written; lane 0 then issues the bulk copies that read them (the wait ends
// with an async-proxy fence).
MX_DEVICE_INLINE bool ks_wait(const GemmParams &p, int slot0, int n, int step, int lane, volatile int *abort_flag) {
    bool ok = true;
    if (lane == 0)
        for (int j = 0; j < n && ok; ++j)
            ok = wait_global_at_least(p.ks_flags + slot0 + j * step, kSplitSlotDone, p.wait_limit_ns,
                                      SITE_KSPLIT_PARTIAL, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __threadfence();
    return ok;
}

// This warp's part of a partial piece of worker `worker` (its slot is worker
// * ranks + rank): TMEM quadrant q of the accumulator t_acc (rows m0q .. m0q +
// 31 of C, local rows 32q ..) into the slot, then `share` added to the slot's
// counter.  ordered: all chunks, those the next unit's accumulator shares
// (buffer b's) first, then release() and the rest; otherwise chunks
// [c_begin, c_end) and no release (the worker's last unit).
template <int BN, int ACC_STRIDE, typename Release>
MX_DEVICE_INLINE void ks_partial_drain(const GemmParams &p, int worker, int ranks, int rank, uint32_t t_acc, int b,
                                       int m0q, int n0, int q, int lane, bool ordered, int c_begin, int c_end,
                                       uint32_t share, Release release) {
    constexpr int kChunks = BN / 32;
    constexpr int kOv = (BN - ACC_STRIDE) / 32;
    const int n_valid = p.N - n0;
    const int slot = worker * ranks + rank;
    const bool any_rows = m0q < p.M;  // warp-uniform; a quadrant without rows has no block
    const int n_chunks = ordered ? kChunks : c_end - c_begin;
#pragma unroll 1
    for (int idx = 0; idx < n_chunks; ++idx) {
        int col;
        if (ordered) {
            if (idx == kOv) {
                tc_fence_before();
                __syncwarp();
                release();
            }
            col = 32 * ((b == 0) ? (idx + (kChunks - kOv)) % kChunks : idx);
        } else {
            col = 32 * (c_begin + idx);
        }
        if (any_rows && col < n_valid) ks_store_chunk(p, t_acc + (uint32_t)col, slot, col / 32, q, lane);
    }
    if (ordered && kOv == kChunks) {
        tc_fence_before();
        __syncwarp();
        release();
    }
    ks_publish(p, slot, share, lane);
}

// Shared memory of a finishing piece's fold (the worker's last unit, whose
// MMAs have completed, so the stage rings are idle): for each draining warp
// (two per TMEM lane quadrant: area 2q for the epilogue warp, 2q + 1 for the
// scale warp) a ring of 4 KB buffers and their mbarriers, carved from the B
// ring past the scale warps' staging buffers and from the A ring; the ring is
// as deep as the areas of the quadrants that hold rows allow (2 to 16
// buffers: 16 in the decode-shape kernel, where only one quadrant does).
template <typename L, int STAGES>
struct FoldPlan {
    static constexpr int kStaging = kEpiWarps * L::kEpiBufs * kEpiChunkBytes;
    static constexpr int kAPiece = STAGES * L::kABytes, kBPiece = STAGES * L::kBBytes - kStaging;
    __host__ __device__ static constexpr int area_bytes(int nb) { return nb * kSplitBlockBytes + 128; }
    __host__ __device__ static constexpr int fits(int nb) { return kBPiece / area_bytes(nb) + kAPiece / area_bytes(nb); }
    // the deepest ring (at most 16 buffers) that n_areas areas allow
    __host__ __device__ static constexpr int bufs_for(int n_areas) {
        int nb = 16;
        while (nb > 2 && fits(nb) < n_areas) --nb;
        return nb;
    }
    static_assert(fits(2) >= 2 * kEpiWarps, "fold areas in the stage rings");
};
// Area `area` of n_areas (2 per TMEM lane quadrant with rows): its buffers.
template <typename L, int STAGES>
MX_DEVICE_INLINE uint8_t *ks_fold_area(uint8_t *smem, int area, int nbufs) {
    using F = FoldPlan<L, STAGES>;
    const int a = F::area_bytes(nbufs), in_b = F::kBPiece / a;
    return area < in_b ? smem + L::kOffB + F::kStaging + area * a : smem + L::kOffA + (area - in_b) * a;
}

// This warp's part of a finishing piece, before its epilogue: wait for the
// partial sums of workers U.first .. worker - 1 (bounded), then add them,
// in that order, to chunks [c_begin, c_end) of quadrant q of the accumulator
// (read, added to and written back to TMEM for the ordinary epilogue).  The
// 4 KB blocks, partial sum by partial sum and chunk by chunk, stream through
// the warp's ring by bulk copies, so that the L2 round trips overlap.  Only a
// worker's last unit finishes a tile.
template <typename L, int STAGES>
MX_DEVICE_INLINE bool ks_finish_fold(const GemmParams &p, uint8_t *smem, int area, const KUnit &U, int worker,
                                     int ranks, int rank, uint32_t t_acc, int m0q, int n0, int q, int lane,
                                     int c_begin, int c_end, volatile int *abort_flag) {
    if (m0q >= p.M) return true;  // no rows in this quadrant (warp-uniform)
    const int n = worker - U.first;
    const int slot0 = U.first * ranks + rank;
    if (!ks_wait(p, slot0, n, ranks, lane, abort_flag)) return false;
    int nc = 0;
    while (c_begin + nc < c_end && 32 * (c_begin + nc) < p.N - n0) ++nc;
    const int nb = nc * n;
    if (nb == 0) return true;
    // with fewer quadrants holding rows, fewer warps fold, each with a deeper ring
    constexpr int kBufs2 = FoldPlan<L, STAGES>::bufs_for(2), kBufs4 = FoldPlan<L, STAGES>::bufs_for(4),
                  kBufs6 = FoldPlan<L, STAGES>::bufs_for(6), kBufs8 = FoldPlan<L, STAGES>::bufs_for(8);
    const int kBufs = p.ks_slot_quads == 1 ? kBufs2 : p.ks_slot_quads == 2 ? kBufs4
                                                     : p.ks_slot_quads == 3 ? kBufs6 : kBufs8;
    uint8_t *const buf = ks_fold_area<L, STAGES>(smem, area, kBufs);
    uint64_t *bar = reinterpret_cast<uint64_t *>(buf + kBufs * kSplitBlockBytes);
    // blocks in order: partial sum j (slot slot0 + j * ranks), then chunk
    // c_begin + c; lane 0 issues them ahead of the warp into ring buffer ik
    const float4 *blk0 = ks_block(p, slot0, c_begin, q);
    const size_t slot_step = (size_t)ranks * 8 * p.ks_slot_quads * 256, chunk_step = (size_t)p.ks_slot_quads * 256;
    int ij = 0, ic = 0, ik = 0, issued = 0;
    auto issue_next = [&]() {  // lane 0
        mbar_arrive_expect_tx(&bar[ik], kSplitBlockBytes);
        bulk_load(buf + ik * kSplitBlockBytes, blk0 + (size_t)ij * slot_step + (size_t)ic * chunk_step,
                  kSplitBlockBytes, &bar[ik]);
        if (++ic == nc) ic = 0, ++ij;
        if (++ik == kBufs) ik = 0;
        ++issued;
    };
    if (lane == 0) {
        for (int k = 0; k < kBufs; ++k) mbar_init(&bar[k], 1);
        fence_barrier_init();
        while (issued < kBufs && ij < n) issue_next();
    }
    __syncwarp();
    int k = 0, consumed = 0;
    uint32_t ph = 0;
    for (int j = 0; j < n; ++j) {
        for (int c = 0; c < nc; ++c) {
            if (!mbar_wait_bounded(&bar[k], ph, p.wait_limit_ns, SITE_KSPLIT_PARTIAL, abort_flag)) {
                // copies still in flight into this ring: let them land first
                if (lane == 0)
                    for (int x = consumed; x < issued; ++x)
                        mbar_wait_bounded(&bar[x % kBufs], (uint32_t)((x / kBufs) & 1), p.wait_limit_ns,
                                          SITE_GEMM_TAIL, nullptr);
                __syncwarp();
                return false;
            }
            const uint32_t ta = t_acc + (uint32_t)(32 * (c_begin + c));
            const float4 *src = reinterpret_cast<const float4 *>(buf + k * kSplitBlockBytes) + lane;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t r[16];
                tmem_ld16(ta + 16 * h, r);
                tmem_wait_ld();
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float4 a = src[32 * (4 * h + v)];
                    r[4 * v] = __float_as_uint(__uint_as_float(r[4 * v]) + a.x);
                    r[4 * v + 1] = __float_as_uint(__uint_as_float(r[4 * v + 1]) + a.y);
                    r[4 * v + 2] = __float_as_uint(__uint_as_float(r[4 * v + 2]) + a.z);
                    r[4 * v + 3] = __float_as_uint(__uint_as_float(r[4 * v + 3]) + a.w);
                }
                tmem_st16(ta + 16 * h, r);
            }
            tmem_wait_st();  // the next partial sum reads these columns again
            __syncwarp();    // every lane has read buffer k
            ++consumed;
            if (lane == 0 && ij < n) {
                fence_proxy_async_smem();
                issue_next();
            }
            if (++k == kBufs) k = 0, ph ^= 1u;
        }
    }
    return true;
}

template <int FMT, int BN, int STAGES, int A_ROWS = kBM, bool SPLIT = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmSfa,
                const __grid_constant__ CUtensorMap tmSfb, GemmParams p) {
    using F = GemmFmt<FMT>;
    using L = GemmSmem<FMT, BN, STAGES, A_ROWS>;
    static_assert(sizeof(FusedQuantSmem) <= L::kEpiAreaBytes, "fused quantize scratch in the staging buffers");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *empty = full + STAGES;
    uint64_t *sfload = empty + STAGES;           // [kSfGroups]
    uint64_t *sfree = sfload + L::kSfGroups;     // [kSfGroups]
    uint64_t *acc_full = sfree + L::kSfGroups;   // [2]
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 1;
    uint64_t *sf_full = mma_done + 1;            // [L::kSlots]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
    uint32_t *ready_count = reinterpret_cast<uint32_t *>(smem + L::kOffMisc + 8);  // gate -> MMA issuer

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int worker = (int)blockIdx.x;
    const int n_units = unit_count<SPLIT>(p, worker);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int g = 0; g < L::kSfGroups; ++g) {
            mbar_init(&sfload[g], 1);
            mbar_init(&sfree[g], 4);
        }
        mbar_init(&acc_full[0], 1);
        mbar_init(&acc_full[1], 1);
        // with GELU the scale warps also release shared accumulator columns
        mbar_init(acc_empty, (p.epilogue == 1 ? 2 : 1) * kEpiWarps);
        mbar_init(mma_done, 1);
        for (int i = 0; i < L::kSlots; ++i) mbar_init(&sf_full[i], 4);
        *abort_flag = 0;
        *ready_count = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSfa);
        tma_prefetch_desc(&tmSfb);
        if (p.use_tma_store) tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The setup above overlaps the previous kernel in the stream; its outputs
    // (our operands, NVFP4 scales, C's prior contents) are read only after this.
    // (fused == 2: that kernel is the quantize of A, whose CTAs started only
    // after everything before it had completed; A is read band by band as its
    // counters say.)
    if (p.fused != 2) griddep_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ code-tile producer
        // The whole warp walks the loop (all values warp-uniform); lane 0
        // issues the copies.
        if (!p.skip_producer) {
            int used = 0, s = 0;
            uint32_t ph = 0;
            bool stop = false;
            int ready_band = -1;   // fused quantize: the last A band known to be written
            for (int u = 0; u < n_units && !stop; ++u) {
                const KUnit U = unit_at<SPLIT>(p, worker, u);
                int m0, n0;
                tile_coords(p, U.tile, m0, n0, kBM, BN);
                if (p.fused && m0 / kBM != ready_band) {
                    if (!wait_band_ready(p, m0 / kBM, lane, abort_flag)) break;
                    ready_band = m0 / kBM;
                }
                for (int kt = U.kb; kt < U.ke; ++kt) {
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, p.wait_limit_ns, SITE_GEMM_PRODUCER_EMPTY, abort_flag)) {
                        stop = true;
                        break;
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[s], FMT == kGemmRuntimeTypes ? p.stage_tx
                                                                                 : (uint32_t)(L::kABytes + L::kBBytes));
                        tma_load_2d(smem + L::kOffA + s * L::kABytes, &tmA, kt * kStageKBytes, m0, &full[s]);
                        tma_load_2d(smem + L::kOffB + s * L::kBBytes, &tmB, kt * kStageKBytes, n0, &full[s]);
                    }
                    __syncwarp();
                    ++used;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // Do not leave while copies into this CTA's shared memory are in flight:
            // wait for the last fill of every stage that was used.
            for (int u = max(0, used - STAGES); u < used; ++u)
                mbar_wait_bounded(&full[u % STAGES], (uint32_t)((u / STAGES) & 1), p.wait_limit_ns, SITE_GEMM_TAIL,
                                  nullptr);
        }
    } else if (warp == kSfWarp) {
        // ------------------------------------------------------------ scale-tile producer
        if (!p.skip_producer)
            sf_producer_role<L, SPLIT>(p, &tmSfa, &tmSfb, smem, sfload, sfree, worker,
                                [&](int tile, int &a_band, int &b_band) {
                                    int m0, n0;
                                    tile_coords(p, tile, m0, n0, kBM, BN);
                                    a_band = m0 / 128;
                                    b_band = n0 / 128;
                                },
                                lane, abort_flag);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // All 32 lanes walk the loop with warp-uniform operands; the tcgen05
        // instructions are predicated on lane 0, so the same thread issues every
        // MMA and the commits that track them, without a divergent branch.
        // Ring positions advance incrementally and the descriptors of a stage
        // are one add from a base: the loop is a short dependent chain per stage.
        const uint64_t desc_ab = smem_desc(0, 16, 1024, 2);
        const uint64_t ad0 = desc_ab | (uint64_t)((smem_u32(smem + L::kOffA) >> 4) & 0x3FFFu);
        const uint64_t bd0 = desc_ab | (uint64_t)((smem_u32(smem + L::kOffB) >> 4) & 0x3FFFu);
        const uint32_t leader = lane == 0 ? 1u : 0u;
        const uint32_t ab = FMT == kGemmRuntimeTypes ? p.ab_types : 0u;
        int last_n_mma, last_n_chunk;
        stage_extent<FMT>(p.num_kt - 1, p.K, last_n_mma, last_n_chunk);
        int s = 0, slot = 0;  // stage and scale-slot ring positions
        uint32_t kg = 0;      // stages consumed
        uint32_t avail = 0;   // stages the gate warp has reported ready
        bool stop = false;
        for (int it = 0; it < n_units && !stop; ++it) {
            const KUnit U = unit_at<SPLIT>(p, worker, it);
            const uint32_t t_acc = tmem + (uint32_t)((it & 1) * L::kAccStride);
            // One stage: its MMAs, then a commit that frees the smem stage and the
            // scale slot once they have completed.
            auto run_stage = [&](int k, uint32_t acc) {
                const uint32_t t_sfa = tmem + (uint32_t)(L::kTmemSf + slot * L::kSfSlotCols);
                issue_stage<FMT, false, BN, 4 * L::kBBands>(k + 1 < p.num_kt ? 4 : last_n_mma, t_acc, ad0 + (uint64_t)(s * (L::kABytes >> 4)),
                    bd0 + (uint64_t)(s * (L::kBBytes >> 4)), t_sfa, t_sfa + 4 * F::kChunks, acc, leader, ab);
                tc_commit_if(&empty[s], leader);
                s = (s + 1 == STAGES) ? 0 : s + 1;
                slot = (slot + 1 == L::kSlots) ? 0 : slot + 1;
                ++kg;
            };
            // Two stages per iteration: the loop's own instructions then fall between
            // MMAs only every other stage.
            for (int kt = U.kb; kt < U.ke; kt += 2) {
                const bool two = kt + 1 < U.ke;
                // the gate warp publishes how many stages have their code tiles and
                // scale slots in; read it only when the stages known ready run out
                const uint32_t need = kg + (two ? 1u : 0u);
                if (need >= avail) {
                    avail = wait_counter_above(ready_count, need, p.wait_limit_ns, SITE_GEMM_MMA_READY, abort_flag);
                    if (avail == 0u) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                }
                if (kt == U.kb && it > 0) {
                    // the epilogue has released the columns this accumulator shares
                    if (!mbar_wait_bounded(acc_empty, (it - 1) & 1, p.wait_limit_ns, SITE_GEMM_MMA_ACC_EMPTY, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                }
                run_stage(kt, kt > U.kb ? 1u : 0u);
                if (two) run_stage(kt + 1, 1u);
            }
            if (!stop) tc_commit_if(&acc_full[it & 1], leader);
        }
        tc_commit_if(mma_done, leader);
        __syncwarp();
    } else if (warp == kGateWarp) {
        // ------------------------------------------------------------ gate
        gate_role<STAGES, L::kSlots>(p, full, sf_full, ready_count, unit_stages<SPLIT>(p, worker), lane, abort_flag);
    } else if (warp >= 6) {
        // ------------------------------------------------------------ scale warps
        const int q = warp & 3;
        const int my_tiles = n_units;
        float scale = 1.0f;
        if (FMT == 3) scale = gemm_ga(p) * (*p.gb);
        uint32_t amax = 0;
        // GELU: this warp's share of the shared columns of tile t (all but the
        // last tile), drained before the first wait on a stage of tile t + 1 or
        // later, whose MMAs cannot start until tile t's columns are released
        int help_next = 0;
        auto help = [&](int t) -> bool {
            int m0, n0;
            tile_coords(p, unit_at<SPLIT>(p, worker, t).tile, m0, n0, kBM, BN);
            const int b = t & 1;
            if (!mbar_wait_bounded(&acc_full[b], (t >> 1) & 1, p.wait_limit_ns, SITE_GEMM_EPI_ACC, abort_flag))
                return false;
            tc_fence_after();
            help_drain_t<BN, L::kAccStride, FMT == 3>(
                p, tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * L::kAccStride), b, m0 + 32 * q, n0, lane, amax,
                scale);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
            return true;
        };
        scale_role<L, STAGES, SPLIT>(p, smem, sfload, sfree, empty,
                                     tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)L::kTmemSf, worker, lane, abort_flag,
                                     [&](int slot) { mbar_arrive(&sf_full[slot]); },
                              [&](int kg) -> bool {
                                  if (p.epilogue != 1) return true;
                                  for (; help_next < my_tiles - 1 && kg - L::kSlots >= (help_next + 1) * p.num_kt;
                                       ++help_next)
                                      if (!help(help_next)) return false;
                                  return true;
                              });
        if (p.epilogue == 1 && !*abort_flag)
            for (; help_next < my_tiles - 1; ++help_next)
                if (!help(help_next)) break;
        // then the upper half of the columns of this CTA's last tile (its MMAs have
        // completed, so the B stage ring is free for the staging buffers)
        if (my_tiles > 0 && !*abort_flag) {
            const int it = my_tiles - 1, b = it & 1;
            const KUnit U = unit_at<SPLIT>(p, worker, it);
            int m0, n0;
            tile_coords(p, U.tile, m0, n0, kBM, BN);
            // mma_done (one phase) rather than acc_full[b]: without GELU this warp
            // may finish its slots several tiles ahead of the MMAs, and a parity
            // wait on acc_full[b], whose phases alternate every second tile,
            // could then be satisfied by an older tile's phase
            if (mbar_wait_bounded(mma_done, 0, p.wait_limit_ns, SITE_GEMM_EPI_ACC, abort_flag)) {
                tc_fence_after();
                uint8_t *bufs = smem + L::kOffB + (warp - 6) * L::kEpiBufs * kEpiChunkBytes;
                uint32_t nstore = 0;
                const uint32_t t_acc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * L::kAccStride);
                if (U.kind == kUnitPartial)
                    ks_partial_drain<BN, L::kAccStride>(p, worker, 1, 0, t_acc, b, m0 + 32 * q, n0, q, lane, false,
                                                        BN / 64, BN / 32, 1u, [] {});
                else if (U.kind == kUnitWhole ||
                         ks_finish_fold<L, STAGES>(p, smem, 2 * q + 1, U, worker, 1, 0, t_acc, m0 + 32 * q, n0, q, lane,
                                                   BN / 64, BN / 32, abort_flag))
                    epilogue_chunks<L::kEpiBufs, FMT == 3>(p, &tmC, t_acc, m0 + 32 * q, n0, BN / 64, BN / 32, lane, bufs,
                                                           nstore, amax, scale);
            }
        }
        epilogue_finish(p, lane, amax);
    } else {
        // ------------------------------------------------------------ epilogue
        // (fused: first the activation quantize, in the staging buffers' space)
        if (p.fused == 1) fused_quantize_role<FMT>(p, reinterpret_cast<FusedQuantSmem *>(smem + L::kOffEpi), threadIdx.x - 64);
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        uint8_t *bufs = smem + L::kOffEpi + (warp - 2) * L::kEpiBufs * kEpiChunkBytes;
        uint32_t amax = 0, nstore = 0;
        float scale = 1.0f;
        if (FMT == 3) scale = gemm_ga(p) * (*p.gb);
        auto release = [&] {
            if (lane == 0) mbar_arrive(acc_empty);
        };
        for (int it = 0; it < n_units; ++it) {
            const KUnit U = unit_at<SPLIT>(p, worker, it);
            int m0, n0;
            tile_coords(p, U.tile, m0, n0, kBM, BN);
            const int b = it & 1;
            if (!mbar_wait_bounded(&acc_full[b], (it >> 1) & 1, p.wait_limit_ns, SITE_GEMM_EPI_ACC, abort_flag)) break;
            tc_fence_after();
            const uint32_t t_acc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * L::kAccStride);
            const bool last = it + 1 == n_units;
            // a piece of a split tile: on the last unit the lower half of the
            // columns (the scale warp takes the upper half), else all of them
            if (U.kind == kUnitPartial) {
                ks_partial_drain<BN, L::kAccStride>(p, worker, 1, 0, t_acc, b, m0 + 32 * q, n0, q, lane, !last, 0,
                                                    last ? BN / 64 : BN / 32, last ? 1u : 2u, release);
                if (last) break;
                continue;
            }
            if (U.kind == kUnitFinish &&
                !ks_finish_fold<L, STAGES>(p, smem, 2 * q, U, worker, 1, 0, t_acc, m0 + 32 * q, n0, q, lane, 0,
                                           last ? BN / 64 : BN / 32, abort_flag))
                break;
            if (last) {
                // the last tile: the lower half of the columns (the scale warp of
                // this quadrant drains the upper half); nothing waits for its release
                epilogue_chunks<L::kEpiBufs, FMT == 3>(p, &tmC, t_acc, m0 + 32 * q, n0, 0, BN / 64, lane, bufs, nstore,
                                                       amax, scale);
                break;
            }
            epilogue_tile<BN, L::kAccStride, L::kEpiBufs, FMT == 3>(p, &tmC, t_acc, b, m0 + 32 * q, n0, lane, bufs,
                                                                     nstore, amax, scale, release);
        }
        epilogue_finish(p, lane, amax);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        // every MMA has completed once mma_done has fired
        mbar_wait_bounded(mma_done, 0, p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
        tmem_dealloc(tmem, L::kTmemCols);
    }
    // the next kernel in the stream may start its setup now (it still waits
    // for this grid's completion before reading anything)
    griddep_launch_dependents();
}

}  // namespace mx
