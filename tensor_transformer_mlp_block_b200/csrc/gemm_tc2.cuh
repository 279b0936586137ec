// Persistent tcgen05 GEMM on CTA pairs (cta_group::2), sm_100a.
//
// Same contract and epilogues as gemm_tc.cuh, but each work unit is a
// 256 × BN output tile computed by a cluster of two CTAs on two SMs:
//   - CTA r (r = 0, 1) loads rows [r·128, r·128 + 128) of the tile's A
//     k-block and columns [r·BN/2, (r+1)·BN/2) of its B k-block into its own
//     shared memory (no multicast: every byte is fetched once, by one CTA);
//   - one thread of CTA 0 (the leader) issues tcgen05.mma.cta_group::2
//     with M = 256, N = BN, which reads both CTAs' shared memory and writes
//     rows [r·128, +128) of the accumulator into CTA r's tensor memory;
//   - both CTAs' epilogue warps drain their own tensor memory.
// Per SM this halves the B operand's share of shared-memory fill and L2
// traffic relative to the one-CTA kernel at the same tile per SM.
//
// Barriers: full[s] lives in the leader and counts both CTAs' TMA bytes;
// empty[s] and tfull[b] live in both CTAs and are completed by the leader's
// tcgen05.commit multicast to both; tempty[b] lives in the leader and
// collects the epilogue warps of both CTAs. All waits are bounded.
#pragma once

#include "gemm_tc.cuh"

namespace tpmlp {

// DBL: two epilogue staging slots per warp, paid for with one ring stage (5
// instead of 6).
template <int BN, bool DBL = false>
struct Tile2Cfg {
    static_assert(BN == 128 || BN == 256, "pair tiles use BN = 128 or 256");
    static constexpr int A_BYTES = kBM * kBK * 2;         // this CTA's 128 rows
    static constexpr int B_BYTES = (BN / 2) * kBK * 2;    // this CTA's BN/2 columns
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // per CTA
    static constexpr int RING_BYTES = DBL ? 163840 : 196608;
    static constexpr int STAGES = (RING_BYTES / STAGE_BYTES) > 8 ? 8 : (RING_BYTES / STAGE_BYTES);
    static constexpr int STAGING_BYTES = (DBL ? 2 : 1) * kEpiStagingBytes;
    static constexpr int TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
    // barriers: ring (2·STAGES), accumulators (4), drain, relay (8), item
    // queue (2·kQueue); then the TMEM address, the abort flag, the queue's items
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5 + 8 + 2 * kQueue) + 16 + 4 * kQueue;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STAGING_BYTES + BAR_BYTES;
};

constexpr int kPairM = 2 * kBM;  // 256 rows per pair tile

// LONG: the variant for long products (bf16 outputs, ≥ 64 k-blocks per tile,
// ≥ 4 waves of tiles): double epilogue staging (Tile2Cfg's DBL), and the only
// variant that can run the dynamic schedule (g.dyn_counter non-null). The
// other variants compile the static schedule alone: a run-time choice between
// the two in their loops costs the short products (12–24 k-blocks per tile)
// 6–9% per launch, measured on B200.
template <int BN, bool A_MN, bool B_MN, int EPI, bool RELAY, bool LONG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                    const GemmArgs g) {
    using C = Tile2Cfg<BN, LONG>;
    constexpr int STAGES = C::STAGES;
    constexpr uint32_t IDESC = idesc_bf16_f32(kPairM, BN, A_MN, B_MN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * C::A_BYTES;
    uint8_t* sEpi = sB + STAGES * C::B_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + C::STAGING_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 2;
    uint64_t* drain = bars + 2 * STAGES + 4;
    uint64_t* xfull = bars + 2 * STAGES + 5;   // relay hand-off, 4 pairs
    uint64_t* xempty = bars + 2 * STAGES + 9;
    uint64_t* qfull = bars + 2 * STAGES + 13;  // item queue (dynamic schedule)
    uint64_t* qempty = qfull + kQueue;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qempty + kQueue);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* qitems = reinterpret_cast<int*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = (rank == 0);
    const int pair = static_cast<int>(cluster_id_x());
    const int npairs = static_cast<int>(num_clusters_x());

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tfull[b]), 1);
            mbar_init(smem_u32(&tempty[b]), 2 * kEpiWarps);
        }
        mbar_init(smem_u32(drain), 1);
        for (int x = 0; x < 4; ++x) {
            mbar_init(smem_u32(&xfull[x]), 32);
            mbar_init(smem_u32(&xempty[x]), 32);
        }
        if constexpr (LONG) {
            // readers of each queue slot: the leader's MMA thread and 8 epilogue
            // warps, the other CTA's producer and 8 epilogue warps
            for (int x = 0; x < kQueue; ++x) {
                mbar_init(smem_u32(&qfull[x]), 1);
                mbar_init(smem_u32(&qempty[x]), 2 + 2 * kEpiWarps);
            }
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // launched as a programmatic dependent: the prologue above overlaps the
    // predecessor's last CTAs; its outputs are read only after this wait
    grid_dep_wait();
    grid_dep_launch();

    const uint64_t limit = g.wait_limit_ns;  // num_m_blocks counts 256-row blocks
    if (warp == 0) zero_later_counters(g, lane);
    const bool dyn = LONG && g.dyn_counter != nullptr;  // constant false in the other variants
    const PairQueue queue{smem_u32(qitems), smem_u32(qfull), smem_u32(qempty), leader};

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            if (g.second) {
                tma_prefetch_desc(&tmA2);
                tma_prefetch_desc(&tmB2);
            }
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            const int a_row0 = static_cast<int>(rank) * kBM;
            const int b_col0 = static_cast<int>(rank) * (BN / 2);
            UnitCursor cur = unit_cursor(pair, npairs, dyn);
            WorkUnit w;
            bool qok = true;
            while (ok && (leader ? cursor_next<true, false>(g, npairs, cur, w, &queue, qok, abort, limit)
                                 : cursor_next<false, false>(g, npairs, cur, w, &queue, qok, abort, limit))) {
                const int mb = w.mb, nb = w.nb;
                const int kb0 = w.kb0, kb1 = w.kb1;
                const CUtensorMap* mA = w.prob ? &tmA2 : &tmA;
                const CUtensorMap* mB = w.prob ? &tmB2 : &tmB;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, abort, limit)) {
                        raise_timeout(abort);
                        ok = false;
                        break;
                    }
                    const uint32_t fb_local = smem_u32(&full[stage]);
                    if (leader) mbar_arrive_expect_tx(fb_local, 2 * C::STAGE_BYTES);
                    const uint32_t fb = mapa_shared(fb_local, 0);
                    const uint32_t a_dst = smem_u32(sA + stage * C::A_BYTES);
                    const uint32_t b_dst = smem_u32(sB + stage * C::B_BYTES);
                    const int m0 = mb * kPairM + a_row0;
                    const int n0 = nb * BN + b_col0;
                    if constexpr (!A_MN) {
                        tma_load_2d_pair(a_dst, mA, fb, kb * kBK, m0);
                    } else {
                        tma_load_2d_pair(a_dst, mA, fb, m0, kb * kBK);
                        tma_load_2d_pair(a_dst + 8192, mA, fb, m0 + 64, kb * kBK);
                    }
                    if constexpr (!B_MN) {
                        tma_load_2d_pair(b_dst, mB, fb, kb * kBK, n0);
                    } else {
#pragma unroll
                        for (int j = 0; j < BN / 128; ++j)
                            tma_load_2d_pair(b_dst + j * 8192, mB, fb, n0 + j * 64, kb * kBK);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!qok) {
                raise_timeout(abort);
                ok = false;
            }
            if (dyn && leader && ok) {
                // every pair has drawn past the end once it arrives here: the
                // last one puts the counters back to zero for the next launch
                __threadfence();
                if (atomicAdd(g.dyn_counter + 1, 1) == npairs - 1) {
                    atomicExch(g.dyn_counter, 0);
                    atomicExch(g.dyn_counter + 1, 0);
                }
            }
            if (ok && !*abort) {
                // Producer tail: every slot released by the leader's MMAs.
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < STAGES && ok; ++i) {
                    if (!mbar_wait_bounded(smem_u32(&empty[s]), ph ^ 1u, abort, limit)) {
                        raise_timeout(abort);
                        ok = false;
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if ((!ok || *abort) && leader) {
                // Wind down: wait (bounded) for the copies of the last slots issued.
                int s = stage;
                uint32_t ph = phase;
                const int n = issued < STAGES ? issued : STAGES;
                for (int i = 0; i < n; ++i) {
                    if (--s < 0) {
                        s = STAGES - 1;
                        ph ^= 1u;
                    }
                    volatile int never = 0;
                    mbar_wait_bounded(smem_u32(&full[s]), ph, &never, limit);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            UnitCursor cur = unit_cursor(pair, npairs, dyn);
            WorkUnit w;
            bool qok = true;
            for (int local = 0;
                 ok && cursor_next<false, false>(g, npairs, cur, w, &queue, qok, abort, limit); ++local) {
                const int kb0 = w.kb0, kb1 = w.kb1;
                const int buf = local & 1;
                const uint32_t aphase = (local >> 1) & 1;
                if (!mbar_wait_bounded(smem_u32(&tempty[buf]), aphase ^ 1u, abort, limit)) {
                    raise_timeout(abort);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&full[stage]), phase, abort, limit)) {
                        raise_timeout(abort);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
                    const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        const uint64_t ad = A_MN ? smem_desc_sw128(a_base + k * 2048, 8192, 1024)
                                                 : smem_desc_sw128(a_base + k * 32, 16, 1024);
                        const uint64_t bd = B_MN ? smem_desc_sw128(b_base + k * 2048, 8192, 1024)
                                                 : smem_desc_sw128(b_base + k * 32, 16, 1024);
                        umma_bf16_pair(d_tmem, ad, bd, IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit_pair(smem_u32(&empty[stage]), 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit_pair(smem_u32(&tfull[buf]), 0x3);
            }
            if (!qok) {
                raise_timeout(abort);
                ok = false;
            }
            if (!ok || *abort) {
                umma_commit_pair(smem_u32(drain), 0x1);
                volatile int never = 0;
                mbar_wait_bounded(smem_u32(drain), 0, &never, limit);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue warps (both CTAs)
        epilogue_role<BN, EPI, true, RELAY, LONG>(g, &tmO0, &tmO1, tmem_base, tfull, tempty, xfull, xempty, sEpi,
                                            pair, npairs, kPairM, static_cast<int>(rank) * kBM, abort,
                                            limit, warp, lane, dyn ? &queue : nullptr);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA frees or exits while its pair still uses it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace tpmlp
