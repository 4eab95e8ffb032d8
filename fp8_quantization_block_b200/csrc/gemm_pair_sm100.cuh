// gemm_pair_sm100.cuh -- block-scaled GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same computation as gemm_sm100.cuh (C = A_dq * B_dq^T in bf16; page
// "Microscaling MXFP4/NVFP4 on Blackwell", section "Arquitetura Blackwell SM100
// e aceleração nativa de NVFP4"), for M > 128.  Two CTAs on neighbouring SMs
// (a cluster of 2) compute a 256 x 256 output tile with M = 256 MMAs: each CTA
// loads its own 128 rows of A and its own 128-row half of B, and the tensor
// core reads B from both CTAs' shared memory.  Per SM that is half the B
// traffic of a 128 x 256 tile for the same MMA work, which keeps the L2 -> SM
// traffic under the fabric's bandwidth at full MMA rate.  No load is multicast.
//
// Roles per CTA (10 warps), as in the single-CTA kernel:
//   warp 0     TMA producer: own A rows and B half (completion counted on the
//              leader CTA's barrier), own scale tiles (local barrier);
//   warps 6-9  scale warps: this CTA's TMEM gets the scales of its 128 A rows
//              and of all 256 B rows, via tcgen05.st, ahead of the MMAs; the
//              leader's also wait for the pair's code tiles, so the MMA thread
//              checks one barrier per stage;
//   warp 1     leader CTA only: issues the pair's MMAs; commits fan out to the
//              barriers of both CTAs;
//   warps 2-5  epilogue for this CTA's 128 rows of the tile.
// Every mbarrier wait is bounded; both CTAs meet at a cluster barrier before
// exit, so no CTA leaves while its partner may still signal it.
#pragma once

#include "gemm_sm100.cuh"

namespace mx {

template <int FMT, int STAGES>
struct PairSmem {
    using F = GemmFmt<FMT>;
    static constexpr int BN = 256;  // pair tile is 256 x 256
    static constexpr int kABytes = 128 * kStageKBytes;
    static constexpr int kBBytes = 128 * kStageKBytes;
    static constexpr int kSfaBytes = F::kChunks * 512;
    static constexpr int kSfbBytes = F::kChunks * 512 * 2;
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + STAGES * kABytes;
    static constexpr int kOffEpi = kOffB + STAGES * kBBytes;
    static constexpr int kNoEpi = STAGES * (kABytes + kBBytes + kSfaBytes + kSfbBytes) + (3 * STAGES + 4 + 2 * kSfSlots) * 8 +
                                  16 + 1024;
    static constexpr int kEpiBufs = (kNoEpi + kEpiWarps * 2 * kEpiChunkBytes <= kSmemLimit) ? 2 : 1;
    static constexpr int kOffSfa = kOffEpi + kEpiWarps * kEpiBufs * kEpiChunkBytes;
    static constexpr int kOffSfb = kOffSfa + STAGES * kSfaBytes;
    static constexpr int kOffBar = kOffSfb + STAGES * kSfbBytes;
    // full[S] (leader's counts both CTAs' code tiles), empty[S], sfload[S],
    // acc_full[2], acc_empty, mma_done, sf_full[slots], sf_empty[slots]
    static constexpr int kNumBars = 3 * STAGES + 4 + 2 * kSfSlots;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;
    // TMEM (per CTA) as in the single-CTA kernel with BN = 256.
    using T = GemmSmem<FMT, 256, 1>;
    static constexpr int kTmemCols = 512;
    static constexpr int kSfSlotCols = T::kSfSlotCols;
    static constexpr int kAccStride = T::kAccStride;
    static constexpr int kTmemSf = T::kTmemSf;
};

template <int FMT>
MX_DEVICE_INLINE uint32_t pair_idesc(uint32_t sf_id) {
    using F = GemmFmt<FMT>;
    return (sf_id << 4) | (F::kAFmt << 7) | (F::kAFmt << 10) | ((uint32_t)(256 >> 3) << 17) |
           (F::kScaleUE8M0 << 23) | ((uint32_t)(256 >> 4) << 24) | (sf_id << 29);
}

template <int FMT>
MX_DEVICE_INLINE void pair_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                               uint32_t acc) {
    if (FMT <= 1) tc_mma_pair_mxf8f6f4(d, a, b, idesc, sfa, sfb, acc);
    else if (FMT == 2) tc_mma_pair_mxf4(d, a, b, idesc, sfa, sfb, acc);
    else tc_mma_pair_nvf4(d, a, b, idesc, sfa, sfb, acc);
}

template <int FMT>
MX_DEVICE_INLINE void pair_mma_if(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                  uint32_t acc, uint32_t issue) {
    if (FMT <= 1) tc_mma_pair_mxf8f6f4_if(d, a, b, idesc, sfa, sfb, acc, issue);
    else if (FMT == 2) tc_mma_pair_mxf4_if(d, a, b, idesc, sfa, sfb, acc, issue);
    else tc_mma_pair_nvf4_if(d, a, b, idesc, sfa, sfb, acc, issue);
}

template <int FMT, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, GemmParams p) {
    using F = GemmFmt<FMT>;
    using L = PairSmem<FMT, STAGES>;
    static_assert(STAGES >= kSfSlots, "scale slots are recycled through the stage barriers");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *empty = full + STAGES;
    uint64_t *sfload = empty + STAGES;
    uint64_t *acc_full = sfload + STAGES;  // [2]
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 1;
    uint64_t *sf_full = mma_done + 1;         // [kSfSlots]
    uint64_t *sf_empty = sf_full + kSfSlots;  // [kSfSlots]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs)
    const int num_tiles = p.m_blocks * p.n_blocks;  // 256 x 256 tiles
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfload[s], 1);
        }
        mbar_init(&acc_full[0], 1);
        mbar_init(&acc_full[1], 1);
        mbar_init(acc_empty, 2 * kEpiWarps);
        mbar_init(mma_done, 1);
        for (int i = 0; i < kSfSlots; ++i) {
            mbar_init(&sf_full[i], 8);
            mbar_init(&sf_empty[i], 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (p.use_tma_store) tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, L::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before anyone signals them
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (!p.skip_producer) {
            const int n_bands_total = (p.N + 127) / 128;
            const int m_bands_total = (p.M + 127) / 128;
            int last_kg = -1;
            int kg = 0;
            bool stop = false;
            for (int tile = pair; tile < num_tiles && !stop; tile += npairs) {
                int m0, n0;
                tile_coords(tile, p.m_blocks, m0, n0, 256);
                m0 = (tile % p.m_blocks) * 256;
                const int my_m = m0 + 128 * (int)rank, my_n = n0 + 128 * (int)rank;
                const bool sfa_exists = my_m / 128 < m_bands_total;
                const int bands = min(2, n_bands_total - n0 / 128);
                const uint8_t *sfa_row = p.sfa + (int64_t)(my_m / 128) * p.sf_tiles_k * 512;
                const uint8_t *sfb_row = p.sfb + (int64_t)(n0 / 128) * p.sf_tiles_k * 512;
                for (int kt = 0; kt < p.num_kt; ++kt, ++kg) {
                    const int s = kg % STAGES, round = kg / STAGES;
                    if (!mbar_wait_bounded(&empty[s], (round & 1) ^ 1, p.wait_limit_ns, SITE_GEMM_PRODUCER_EMPTY,
                                           abort_flag)) {
                        stop = true;
                        break;
                    }
                    int n_mma, n_chunk;
                    stage_extent<FMT>(kt, p.K, n_mma, n_chunk);
                    const uint32_t sf_bytes = (uint32_t)n_chunk * 512u;
                    const int64_t sf_k = (int64_t)kt * F::kChunks * 512;
                    if (lane == 0) {
                        const uint32_t full_leader = mapa_shared(smem_u32(&full[s]), 0);
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (L::kABytes + L::kBBytes));
                        tma_load_2d_pair(smem + L::kOffA + s * L::kABytes, &tmA, kt * kStageKBytes, my_m, full_leader);
                        tma_load_2d_pair(smem + L::kOffB + s * L::kBBytes, &tmB, kt * kStageKBytes, my_n, full_leader);
                        mbar_arrive_expect_tx(&sfload[s], sf_bytes * ((sfa_exists ? 1u : 0u) + (uint32_t)bands));
                        if (sfa_exists)
                            bulk_load(smem + L::kOffSfa + s * L::kSfaBytes, sfa_row + sf_k, sf_bytes, &sfload[s]);
                        for (int h = 0; h < bands; ++h)
                            bulk_load(smem + L::kOffSfb + s * L::kSfbBytes + h * F::kChunks * 512,
                                      sfb_row + (int64_t)h * p.sf_tiles_k * 512 + sf_k, sf_bytes, &sfload[s]);
                    }
                    __syncwarp();
                    last_kg = kg;
                }
            }
            // Do not leave while copies into shared memory are in flight.  The
            // leader's full barriers count both CTAs' code tiles.
            for (int k = max(0, last_kg - STAGES + 1); k <= last_kg; ++k) {
                if (rank == 0)
                    mbar_wait_bounded(&full[k % STAGES], (k / STAGES) & 1, p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
                mbar_wait_bounded(&sfload[k % STAGES], (k / STAGES) & 1, p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // As in the single-CTA kernel: all lanes walk the loop, lane 0 issues.
        if (rank == 0) {
            const uint32_t a_base = smem_u32(smem + L::kOffA), b_base = smem_u32(smem + L::kOffB);
            const uint64_t desc_ab = smem_desc(0, 16, 1024, 2);
            const uint32_t leader = lane == 0 ? 1u : 0u;
            int kg = 0;
            bool stop = false;
            bool ready = false;  // result of the last peek at stage kg's barriers
            int it = 0;
            for (int tile = pair; tile < num_tiles && !stop; tile += npairs, ++it) {
                const uint32_t t_acc = tmem + (uint32_t)((it & 1) * L::kAccStride);
                for (int kt = 0; kt < p.num_kt; ++kt, ++kg) {
                    const int s = kg % STAGES;
                    const int slot = kg % kSfSlots;
                    // sf_full of a stage implies its code tiles have landed: the scale warps
                    // arrive only after observing the stage's load barrier.
                    if (!ready && !mbar_wait_bounded(&sf_full[slot], (kg / kSfSlots) & 1, p.wait_limit_ns,
                                                     SITE_GEMM_MMA_SF, abort_flag)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    if (kt == 0 && it > 0) {
                        if (!mbar_wait_bounded(acc_empty, (it - 1) & 1, p.wait_limit_ns, SITE_GEMM_MMA_ACC_EMPTY,
                                               abort_flag)) {
                            stop = true;
                            break;
                        }
                        tc_fence_after();
                    }
                    int n_mma, n_chunk;
                    stage_extent<FMT>(kt, p.K, n_mma, n_chunk);
                    const uint32_t a_stage = a_base + s * L::kABytes, b_stage = b_base + s * L::kBBytes;
                    const uint32_t t_sfa = tmem + (uint32_t)(L::kTmemSf + slot * L::kSfSlotCols);
                    const uint32_t t_sfb = t_sfa + 4 * F::kChunks;
                    for (int j = 0; j < n_mma; ++j) {
                        const int chunk = j / F::kMmaPerChunk;
                        const uint32_t sf_id = (uint32_t)((j % F::kMmaPerChunk) * F::kSfPerMma);
                        const uint64_t ad = desc_ab | (uint64_t)(((a_stage + 32 * j) >> 4) & 0x3FFFu);
                        const uint64_t bd = desc_ab | (uint64_t)(((b_stage + 32 * j) >> 4) & 0x3FFFu);
                        pair_mma_if<FMT>(t_acc, ad, bd, pair_idesc<FMT>(sf_id), t_sfa + 4 * chunk, t_sfb + 8 * chunk,
                                         (kt > 0 || j > 0) ? 1u : 0u, leader);
                    }
                    // frees both CTAs' smem stage and, for their scale warps, the scale slot
                    tc_commit_pair_if(&empty[s], 0x3, leader);
                    {
                        const int k1 = kg + 1;
                        ready = mbar_test_wait(&sf_full[k1 % kSfSlots], (k1 / kSfSlots) & 1);
                    }
                }
                if (!stop) tc_commit_pair_if(&acc_full[it & 1], 0x3, leader);
            }
            tc_commit_pair_if(mma_done, 0x3, leader);
            __syncwarp();
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------ scale warps
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t sf_full_leader0 = mapa_shared(smem_u32(&sf_full[0]), 0);
        int kg = 0;
        bool stop = false;
        for (int tile = pair; tile < num_tiles && !stop; tile += npairs) {
            for (int kt = 0; kt < p.num_kt; ++kt, ++kg) {
                const int s = kg % STAGES, slot = kg % kSfSlots;
                if (!mbar_wait_bounded(&sfload[s], (kg / STAGES) & 1, p.wait_limit_ns, SITE_GEMM_SF_LOAD, abort_flag) ||
                    (rank == 0 &&
                     !mbar_wait_bounded(&full[s], (kg / STAGES) & 1, p.wait_limit_ns, SITE_GEMM_SF_FULL, abort_flag))) {
                    stop = true;
                    break;
                }
                if (kg >= kSfSlots &&
                    !mbar_wait_bounded(&empty[(kg - kSfSlots) % STAGES], ((kg - kSfSlots) / STAGES) & 1,
                                       p.wait_limit_ns, SITE_GEMM_SF_EMPTY, abort_flag)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                int n_mma, n_chunk;
                stage_extent<FMT>(kt, p.K, n_mma, n_chunk);
                (void)n_chunk;  // tiles past the K tail carry stale scales the MMAs never read
                stage_scales_to_tmem<F::kChunks, 2>(smem + L::kOffSfa + s * L::kSfaBytes,
                                                    smem + L::kOffSfb + s * L::kSfbBytes,
                                                    tmem + lane_base + (uint32_t)(L::kTmemSf + slot * L::kSfSlotCols),
                                                    lane);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(sf_full_leader0 + 8u * (uint32_t)slot);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (this CTA's 128 rows)
        const int q = warp & 3;
        uint8_t *bufs = smem + L::kOffEpi + (warp - 2) * L::kEpiBufs * kEpiChunkBytes;
        const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
        uint32_t amax = 0, nstore = 0;
        float scale = 1.0f;
        if (FMT == 3) scale = (*p.ga) * (*p.gb);
        int it = 0;
        for (int tile = pair; tile < num_tiles; tile += npairs, ++it) {
            int m0, n0;
            tile_coords(tile, p.m_blocks, m0, n0, 256);
            m0 = (tile % p.m_blocks) * 256 + 128 * (int)rank;
            const int b = it & 1;
            if (!mbar_wait_bounded(&acc_full[b], (it >> 1) & 1, p.wait_limit_ns, SITE_GEMM_EPI_ACC, abort_flag)) break;
            tc_fence_after();
            const uint32_t t_acc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * L::kAccStride);
            epilogue_tile<256, L::kAccStride, L::kEpiBufs, FMT == 3>(p, &tmC, t_acc, b, m0 + 32 * q, n0, lane, bufs, nstore, amax, scale,
                                              [&] {
                                                  if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
                                              });
        }
        epilogue_finish(p, lane, amax);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        // every MMA of the pair has completed once mma_done (multicast) has fired
        mbar_wait_bounded(mma_done, 0, p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
        tmem_dealloc_pair(tmem, L::kTmemCols);
    }
    cluster_sync();
}

}  // namespace mx
