// gemm_pair_sm100.cuh -- block-scaled GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same computation as gemm_sm100.cuh (C = A_dq * B_dq^T in bf16; page
// "Microscaling MXFP4/NVFP4 on Blackwell", section "Arquitetura Blackwell SM100
// e aceleração nativa de NVFP4"), for M > 128.  Two CTAs on neighbouring SMs
// (a cluster of 2) compute a 256 x BN output tile with M = 256 MMAs: each CTA
// loads its own 128 rows of A and its own BN/2-row half of B, and the tensor
// core reads B from both CTAs' shared memory.  Per SM that is half the B
// traffic of a 128 x BN tile for the same MMA work.  No load is multicast.
// BN = 256, or 128 for the GELU epilogue: then the two accumulators and the
// scale slots fit TMEM without sharing columns, so a tile's GELU drain
// overlaps the next tile's MMAs entirely.
//
// Roles per CTA (12 warps), as in the single-CTA kernel:
//   warp 0     code-tile producer: own A rows and B half, completion counted
//              on the leader CTA's barrier;
//   warp 10    scale-tile producer: own A band and both B bands (this CTA's
//              TMEM needs the scales of all BN B rows), local barriers;
//   warps 6-9  scale warps: this CTA's TMEM slot, then an arrive on the
//              leader's slot barrier (8 arrivals: both CTAs' scale warps);
//   warp 11    leader CTA only: gate, counts the stages whose code tiles (both
//              CTAs') and scale slots (both CTAs') are in;
//   warp 1     leader CTA only: issues the pair's MMAs for the stages the gate
//              reports; commits fan out to the barriers of both CTAs;
//   warps 2-5  epilogue for this CTA's 128 rows of the tile.
// Every mbarrier wait is bounded; both CTAs meet at a cluster barrier before
// exit, so no CTA leaves while its partner may still signal it.
#pragma once

#include "gemm_sm100.cuh"

namespace mx {

// Per CTA: 128 rows of A and BN/2 rows of B in smem per stage, scale tiles of
// BN/128 B bands, a BN-column accumulator.
template <int FMT, int STAGES, int BN = 256>
using PairSmem = GemmLayout<FMT, BN / 128, BN / 2, STAGES>;

template <int FMT, int STAGES, int BN = 256, bool SPLIT = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmSfa,
                     const __grid_constant__ CUtensorMap tmSfb, GemmParams p) {
    using F = GemmFmt<FMT>;
    using L = PairSmem<FMT, STAGES, BN>;
    // with GELU the scale warps help drain the accumulator columns the next
    // tile shares, if any
    constexpr bool kHelp = gelu_help_chunks<BN, L::kAccStride>() > 0;
    static_assert(sizeof(FusedQuantSmem) <= L::kEpiAreaBytes, "fused quantize scratch in the staging buffers");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);  // leader's count both CTAs' code tiles
    uint64_t *empty = full + STAGES;
    uint64_t *sfload = empty + STAGES;          // [kSfGroups]
    uint64_t *sfree = sfload + L::kSfGroups;    // [kSfGroups]
    uint64_t *acc_full = sfree + L::kSfGroups;  // [2]
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 1;
    uint64_t *sf_full = mma_done + 1;           // [L::kSlots], leader's count both CTAs' scale warps
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
    uint32_t *ready_count = reinterpret_cast<uint32_t *>(smem + L::kOffMisc + 8);  // gate -> MMA issuer

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs)
    const int pair = (int)(blockIdx.x >> 1);        // the worker: units of 256 x BN tiles
    const int n_units = unit_count<SPLIT>(p, pair);

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
        // both CTAs' epilogue warps (with GELU, their scale warps too)
        mbar_init(acc_empty, (p.epilogue == 1 && kHelp ? 4 : 2) * kEpiWarps);
        mbar_init(mma_done, 1);
        for (int i = 0; i < L::kSlots; ++i) mbar_init(&sf_full[i], 8);
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
        tmem_alloc_pair(tmem_slot, L::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before anyone signals them
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
        if (!p.skip_producer) {
            const uint32_t full_leader0 = mapa_shared(smem_u32(&full[0]), 0);
            int used = 0, s = 0;
            uint32_t ph = 0;
            bool stop = false;
            int ready_band = -1;   // fused quantize: the last A band known to be written
            for (int u = 0; u < n_units && !stop; ++u) {
                const KUnit U = unit_at<SPLIT>(p, pair, u);
                int m0, n0;
                tile_coords(p, U.tile, m0, n0, 256, BN);
                const int my_m = m0 + 128 * (int)rank, my_n = n0 + (BN / 2) * (int)rank;
                if (p.fused && my_m / 128 != ready_band) {
                    if (!wait_band_ready(p, my_m / 128, lane, abort_flag)) break;
                    ready_band = my_m / 128;
                }
                for (int kt = U.kb; kt < U.ke; ++kt) {
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, p.wait_limit_ns, SITE_GEMM_PRODUCER_EMPTY, abort_flag)) {
                        stop = true;
                        break;
                    }
                    if (lane == 0) {
                        const uint32_t full_leader = full_leader0 + 8u * (uint32_t)s;
                        if (rank == 0)
                            mbar_arrive_expect_tx(&full[s], FMT == kGemmRuntimeTypes ? p.stage_tx
                                                                                     : 2u * (L::kABytes + L::kBBytes));
                        tma_load_2d_pair(smem + L::kOffA + s * L::kABytes, &tmA, kt * kStageKBytes, my_m, full_leader);
                        tma_load_2d_pair(smem + L::kOffB + s * L::kBBytes, &tmB, kt * kStageKBytes, my_n, full_leader);
                    }
                    __syncwarp();
                    ++used;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // Do not leave while copies into shared memory are in flight.  The
            // leader's full barriers count both CTAs' code tiles; the other CTA
            // stays until the closing cluster barrier, which the leader reaches
            // only after these waits.
            if (rank == 0)
                for (int u = max(0, used - STAGES); u < used; ++u)
                    mbar_wait_bounded(&full[u % STAGES], (uint32_t)((u / STAGES) & 1), p.wait_limit_ns, SITE_GEMM_TAIL,
                                      nullptr);
        }
    } else if (warp == kSfWarp) {
        // ------------------------------------------------------------ scale-tile producer
        if (!p.skip_producer)
            sf_producer_role<L, SPLIT>(p, &tmSfa, &tmSfb, smem, sfload, sfree, pair,
                                [&](int tile, int &a_band, int &b_band) {
                                    int m0, n0;
                                    tile_coords(p, tile, m0, n0, 256, BN);
                                    a_band = m0 / 128 + (int)rank;
                                    b_band = n0 / 128;
                                },
                                lane, abort_flag);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // As in the single-CTA kernel: all lanes walk the loop, lane 0 issues.
        if (rank == 0) {
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
                const KUnit U = unit_at<SPLIT>(p, pair, it);
                const uint32_t t_acc = tmem + (uint32_t)((it & 1) * L::kAccStride);
                // One stage: its MMAs, then a commit that frees the smem stage and the
                // scale slot once they have completed.
                auto run_stage = [&](int k, uint32_t acc) {
                    const uint32_t t_sfa = tmem + (uint32_t)(L::kTmemSf + slot * L::kSfSlotCols);
                    issue_stage<FMT, true, BN, 4 * L::kBBands>(k + 1 < p.num_kt ? 4 : last_n_mma, t_acc, ad0 + (uint64_t)(s * (L::kABytes >> 4)),
                        bd0 + (uint64_t)(s * (L::kBBytes >> 4)), t_sfa, t_sfa + 4 * F::kChunks, acc, leader, ab);
                    tc_commit_pair_if(&empty[s], 0x3, leader);
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
                if (!stop) tc_commit_pair_if(&acc_full[it & 1], 0x3, leader);
            }
            tc_commit_pair_if(mma_done, 0x3, leader);
            __syncwarp();
        }
    } else if (warp == kGateWarp) {
        // ------------------------------------------------------------ gate (leader)
        if (rank == 0) {
            gate_role<STAGES, L::kSlots>(p, full, sf_full, ready_count, unit_stages<SPLIT>(p, pair), lane, abort_flag);
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------ scale warps
        const int q = warp & 3;
        const uint32_t sf_full_leader0 = mapa_shared(smem_u32(&sf_full[0]), 0);
        const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
        const int my_tiles = n_units;
        float scale = 1.0f;
        if (FMT == 3) scale = gemm_ga(p) * (*p.gb);
        uint32_t amax = 0;
        auto rows_of = [&](int t, int &m0, int &n0) {
            tile_coords(p, unit_at<SPLIT>(p, pair, t).tile, m0, n0, 256, BN);
            m0 += 128 * (int)rank;
        };
        // GELU: this warp's share of the shared columns of tile t (all but the
        // last tile), drained before the first wait on a stage of tile t + 1 or
        // later, whose MMAs cannot start until both CTAs have released tile t's
        // columns
        int help_next = 0;
        auto help = [&](int t) -> bool {
            int m0, n0;
            rows_of(t, m0, n0);
            const int b = t & 1;
            if (!mbar_wait_bounded(&acc_full[b], (t >> 1) & 1, p.wait_limit_ns, SITE_GEMM_EPI_ACC, abort_flag))
                return false;
            tc_fence_after();
            help_drain_t<BN, L::kAccStride, FMT == 3>(
                p, tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * L::kAccStride), b, m0 + 32 * q, n0, lane, amax,
                scale);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
            return true;
        };
        scale_role<L, STAGES, SPLIT>(p, smem, sfload, sfree, empty, tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)L::kTmemSf,
                              pair, lane, abort_flag,
                              [&](int slot) { mbar_arrive_cluster(sf_full_leader0 + 8u * (uint32_t)slot); },
                              [&](int kg) -> bool {
                                  if (p.epilogue != 1 || !kHelp) return true;
                                  for (; help_next < my_tiles - 1 && kg - L::kSlots >= (help_next + 1) * p.num_kt;
                                       ++help_next)
                                      if (!help(help_next)) return false;
                                  return true;
                              });
        if (p.epilogue == 1 && kHelp && !*abort_flag)
            for (; help_next < my_tiles - 1; ++help_next)
                if (!help(help_next)) break;
        // then the upper half of the columns of this CTA's rows of the last tile
        // (the pair's MMAs have completed, so the B stage ring is free for the
        // staging buffers)
        if (my_tiles > 0 && !*abort_flag) {
            const int it = my_tiles - 1, b = it & 1;
            int m0, n0;
            rows_of(it, m0, n0);
            // mma_done (one phase) rather than acc_full[b]: without GELU this warp
            // may finish its slots several tiles ahead of the MMAs, and a parity
            // wait on acc_full[b], whose phases alternate every second tile,
            // could then be satisfied by an older tile's phase
            if (mbar_wait_bounded(mma_done, 0, p.wait_limit_ns, SITE_GEMM_EPI_ACC, abort_flag)) {
                tc_fence_after();
                uint8_t *bufs = smem + L::kOffB + (warp - 6) * L::kEpiBufs * kEpiChunkBytes;
                uint32_t nstore = 0;
                const uint32_t t_acc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * L::kAccStride);
                const KUnit U = unit_at<SPLIT>(p, pair, it);
                if (U.kind == kUnitPartial)
                    ks_partial_drain<BN, L::kAccStride>(p, pair, 2, (int)rank, t_acc, b, m0 + 32 * q, n0, q, lane,
                                                        false, BN / 64, BN / 32, 1u, [] {});
                else if (U.kind == kUnitWhole ||
                         ks_finish_fold<L, STAGES>(p, smem, 2 * q + 1, U, pair, 2, (int)rank, t_acc, m0 + 32 * q, n0,
                                                   q, lane, BN / 64, BN / 32, abort_flag))
                    epilogue_chunks<L::kEpiBufs, FMT == 3>(p, &tmC, t_acc, m0 + 32 * q, n0, BN / 64, BN / 32, lane, bufs,
                                                           nstore, amax, scale);
            }
        }
        epilogue_finish(p, lane, amax);
    } else {
        // ------------------------------------------------------------ epilogue (this CTA's 128 rows)
        // (fused: first the activation quantize, in the staging buffers' space)
        if (p.fused == 1) fused_quantize_role<FMT>(p, reinterpret_cast<FusedQuantSmem *>(smem + L::kOffEpi), threadIdx.x - 64);
        const int q = warp & 3;
        uint8_t *bufs = smem + L::kOffEpi + (warp - 2) * L::kEpiBufs * kEpiChunkBytes;
        const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
        uint32_t amax = 0, nstore = 0;
        float scale = 1.0f;
        if (FMT == 3) scale = gemm_ga(p) * (*p.gb);
        auto release = [&] {
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
        };
        for (int it = 0; it < n_units; ++it) {
            const KUnit U = unit_at<SPLIT>(p, pair, it);
            int m0, n0;
            tile_coords(p, U.tile, m0, n0, 256, BN);
            m0 += 128 * (int)rank;
            const int b = it & 1;
            if (!mbar_wait_bounded(&acc_full[b], (it >> 1) & 1, p.wait_limit_ns, SITE_GEMM_EPI_ACC, abort_flag)) break;
            tc_fence_after();
            const uint32_t t_acc = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * L::kAccStride);
            const bool last = it + 1 == n_units;
            // a piece of a split tile (this CTA's 128 rows): on the last unit
            // the lower half of the columns (the scale warp takes the upper
            // half), else all of them
            if (U.kind == kUnitPartial) {
                ks_partial_drain<BN, L::kAccStride>(p, pair, 2, (int)rank, t_acc, b, m0 + 32 * q, n0, q, lane, !last,
                                                    0, last ? BN / 64 : BN / 32, last ? 1u : 2u, release);
                if (last) break;
                continue;
            }
            if (U.kind == kUnitFinish &&
                !ks_finish_fold<L, STAGES>(p, smem, 2 * q, U, pair, 2, (int)rank, t_acc, m0 + 32 * q, n0, q, lane, 0,
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
        // every MMA of the pair has completed once mma_done (multicast) has fired
        mbar_wait_bounded(mma_done, 0, p.wait_limit_ns, SITE_GEMM_TAIL, nullptr);
        tmem_dealloc_pair(tmem, L::kTmemCols);
    }
    // the next kernel in the stream may start its setup now (it still waits
    // for this grid's completion before reading anything)
    griddep_launch_dependents();
    cluster_sync();
}

}  // namespace mx
