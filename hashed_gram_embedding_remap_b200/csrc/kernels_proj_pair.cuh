// Step 4 of the lookup on CTA pairs: the same projections and epilogue as proj_kernel, with
// every MMA spanning the two CTAs of a cluster (tcgen05 cta_group::2).  A work unit is a
// 256-token x 256-channel tile; CTA rank r of the pair loads A rows [128r, 128r + 128) of the
// tile and B rows [128r, 128r + 128) of the 256 channels, and its tensor memory holds its 128
// tokens x all 256 channels of the accumulator.  Per k-block of 64 each SM's shared memory
// thus takes 16 KB of A and 16 KB of B (the single-CTA 128 x 256 tile takes 16 + 32 KB for
// half the MMA work), so the tensor cores read half the B bytes per flop and the stage ring
// holds six k-blocks instead of four.
//
// Roles in each CTA: warp 0 lane 0 loads its CTA's tiles into its own shared memory with the
// cta_group::2 TMA forms, whose bytes are counted on the EVEN CTA's full barrier (no
// multicast; the even CTA's expect_tx covers both halves); warp 1 lane 0 of the even CTA
// waits for the stage and issues the MMAs, committing stage and accumulator releases to the
// barriers of both CTAs (tcgen05.commit with a CTA mask: an arrival, not a data multicast);
// warps 2-5 drain their CTA's accumulator rows (the epilogue of proj_kernel) and hand the
// accumulator back to the even CTA.  Every wait is bounded; the CTAs leave only together
// (cluster barrier), after the last MMA.
#pragma once
#include "kernels_proj.cuh"

namespace engram {

constexpr int kPairBN = 256;   // channels per unit (N of one pair MMA)
constexpr int kPairRows = 2 * kBM;

struct PairCfg {
    static constexpr int kATile = kBM * kBK * 2;              // 16 KB: this CTA's 128 rows of A
    static constexpr int kBTile = (kPairBN / 2) * kBK * 2;    // 16 KB: this CTA's 128 rows of B
    static constexpr int kStageBytes = kATile + kBTile;
    static constexpr int kStages = 6;
    static constexpr int kAccum = 2;
    static constexpr int kTmemCols = kAccum * kPairBN;        // 512: all of tensor memory
    // dynamic smem: [align pad][stages x A][stages x B][split-K transpose tiles][full, empty,
    //               tmem_full, tmem_empty, drain][tmem addr]
    static constexpr int kBarBytes = (2 * kStages + 2 * kAccum + 1) * 8;
    static constexpr int kTrStride = 36;                          // split-K transpose (as ProjCfg)
    static constexpr int kTrBytes = 4 * 32 * kTrStride * 4;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kTrBytes + kBarBytes + 16;
};

__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// p.m_tiles counts 256-token tiles; p.n_tiles = (M + 1) * d_h / 256.  SPLIT: units are
// (k split, 256-token tile, 256-channel slice), n fastest, and their raw fp32 partial
// accumulators go to p.acc_out exactly as proj_kernel's split-K units write them (the rows of
// each CTA through a per-warp shared-memory transpose), to be finished by the same kernels.
// map_wk / map_wv: the row-major weights (boxes of 128 rows), or with packed weights map_wk
// spans the packed copy as [tiles * k_blocks * 256 rows, 64 columns] (boxes of 128 rows, no
// swizzle: the bytes are already in the tensor cores' layout) and map_wv is unused.
template <bool SPLIT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kProjThreads, 1)
    proj_pair_kernel(const __grid_constant__ CUtensorMap map_m, const __grid_constant__ CUtensorMap map_wk,
                     const __grid_constant__ CUtensorMap map_wv, const __grid_constant__ ProjParams p) {
    using Cfg = PairCfg;
    constexpr int S = Cfg::kStages;
    constexpr int NACC = Cfg::kAccum;
    constexpr int BN = kPairBN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + S * Cfg::kATile;
    float *s_tr = reinterpret_cast<float *>(smem + S * Cfg::kStageBytes);
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + S * Cfg::kStageBytes + Cfg::kTrBytes);
    uint64_t *empty_bar = full_bar + S;
    uint64_t *tfull_bar = empty_bar + S;      // MMA -> epilogue of both CTAs
    uint64_t *tempty_bar = tfull_bar + NACC;  // epilogues of both CTAs -> MMA (even CTA's copy)
    uint64_t *drain_bar = tempty_bar + NACC;  // even CTA: all MMAs issued so far are done
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(drain_bar + 1);
    __shared__ int s_abort;

    pdl_launch_dependents();
    const uint64_t lim = p.wait_limit_ns ? p.wait_limit_ns : ENGRAM_WAIT_TIMEOUT_NS;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();   // 0: issues the MMAs; 1: its partner
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int mn_tiles = p.m_tiles * p.n_tiles;
    const int total = mn_tiles * p.k_splits;   // units: (k split, 256-token tile, 256-channel slice), n fastest
    // unit t -> (k split, 256-token tile, channel slice) and its k-block range
    auto unit = [&](int t, int &ks, int &mt, int &nt, int &kb0, int &kb1) {
        ks = t / mn_tiles;
        const int tmn = t - ks * mn_tiles;
        mt = tmn / p.n_tiles;
        nt = tmn - mt * p.n_tiles;
        kb0 = ks * p.kb_per_split;
        kb1 = min(p.k_blocks, kb0 + p.kb_per_split);
    };
    const int key_tiles = p.M * (p.d_h / BN);
    const int kpb = p.d_h / BN;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);    // even CTA: its producer's expect_tx arrival (both halves' bytes)
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < NACC; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 8);   // four epilogue warps in each CTA
        }
        mbar_init(drain_bar, 1);
        fence_barrier_init();
        tma_prefetch_desc(&map_m);
        tma_prefetch_desc(&map_wk);
        tma_prefetch_desc(&map_wv);
    }
    if (warp == 1) {
        tmem_alloc_pair(s_tmem, Cfg::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();   // both CTAs' barriers initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    constexpr uint32_t kTxBytes = 2 * Cfg::kStageBytes;   // both CTAs' A and B halves, on the even CTA's barrier
    const uint32_t full_cluster = mapa_shared(full_bar, 0);

    if (warp == 0) {
        if (lane == 0 && !p.stall) {
            auto load_b = [&](int s, int nt, int kb) {
                if (p.w_packed != nullptr)   // this CTA's 128 rows of the pre-swizzled 256 x 64 tile: 16 KB
                    tma_load_2d_pair(sB + s * Cfg::kBTile, &map_wk, full_cluster + s * 8, 0,
                                     (nt * p.k_blocks + kb) * BN + static_cast<int>(rank) * (BN / 2));
                else {
                    const bool is_key = nt < key_tiles;
                    tma_load_2d_pair(sB + s * Cfg::kBTile, is_key ? &map_wk : &map_wv, full_cluster + s * 8, kb * kBK,
                                     (is_key ? nt : nt - key_tiles) * BN + static_cast<int>(rank) * (BN / 2));
                }
            };
            int pre = 0;
            if (pair < total) {   // weight tiles of the first stages: independent of the previous kernel
                int ks, mt, nt, kb0, kb1;
                unit(pair, ks, mt, nt, kb0, kb1);
                pre = min(S, kb1 - kb0);
                for (int q = 0; q < pre; ++q) {
                    if (rank == 0) mbar_arrive_expect_tx(&full_bar[q], kTxBytes);
                    load_b(q, nt, kb0 + q);
                }
            }
            pdl_wait();
            int it = 0, issued = pre;
            for (int t = pair; t < total && !s_abort; t += npairs) {
                int ks, mt, nt, kb0, kb1;
                unit(t, ks, mt, nt, kb0, kb1);
                const int m0 = mt * kPairRows + static_cast<int>(rank) * kBM;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S;
                    if (it < pre) {
                        tma_load_2d_pair(sA + s * Cfg::kATile, &map_m, full_cluster + s * 8, kb * kBK, m0);
                        continue;
                    }
                    if (!mbar_wait(&empty_bar[s], ((it / S) & 1) ^ 1, &s_abort, lim)) break;
                    if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], kTxBytes);
                    tma_load_2d_pair(sA + s * Cfg::kATile, &map_m, full_cluster + s * 8, kb * kBK, m0);
                    load_b(s, nt, kb);
                    issued = it + 1;
                }
            }
            if (s_abort && rank == 0) {   // every issued copy lands before shared memory is released
                volatile int never = 0;
                for (int k = issued - S > 0 ? issued - S : 0; k < issued; ++k)
                    if (!mbar_wait(&full_bar[k % S], (k / S) & 1, &never, lim)) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------------------ MMA issue (even CTA)
            constexpr uint32_t idesc = idesc_bf16_f32(kPairRows, BN);
            int it = 0, li = 0;
            bool issued_any = false;
            for (int t = pair; t < total && !s_abort; t += npairs, ++li) {
                const int acc = li % NACC;
                const uint32_t use = li / NACC;
                if (!mbar_wait_cluster(&tempty_bar[acc], (use & 1) ^ 1, &s_abort, lim)) break;
                tc_fence_after();
                const uint32_t dst = tmem_base + acc * BN;
                int ks, mt, nt, kb0, kb1;
                unit(t, ks, mt, nt, kb0, kb1);
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(&full_bar[s], (it / S) & 1, &s_abort, lim)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = sdesc_kmajor_sw128(sA + s * Cfg::kATile);
                    const uint64_t bdesc = sdesc_kmajor_sw128(sB + s * Cfg::kBTile);
#pragma unroll
                    for (int k = 0; k < kBK / kUmmaK; ++k) {
                        const uint64_t koff = static_cast<uint64_t>((k * kUmmaK * 2) >> 4);
                        umma_bf16_ss_pair(dst, adesc + koff, bdesc + koff, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    issued_any = true;
                    umma_commit_pair(&empty_bar[s], 0x3);   // frees stage s in both CTAs
                }
                if (!ok) break;
                umma_commit_pair(&tfull_bar[acc], 0x3);     // accumulator rows ready in both CTAs
            }
            if (s_abort) {
                // wait for the MMAs already issued, then release every waiting role of both CTAs
                if (issued_any) {
                    volatile int never = 0;
                    umma_commit_pair(drain_bar, 0x1);
                    mbar_wait(drain_bar, 0, &never, lim);
                }
                st_cluster_u32(mapa_shared(&s_abort, 1), 1);
                for (int a = 0; a < NACC; ++a) {
                    mbar_arrive(&tfull_bar[a]);
                    mbar_arrive_cluster(mapa_shared(&tfull_bar[a], 1));
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const uint32_t leader_tempty = mapa_shared(tempty_bar, 0);
        int li = 0;
        for (int t = pair; t < total; t += npairs, ++li) {
            const int acc = li % NACC;
            const uint32_t use = li / NACC;
            bool ok = true;
            if (lane == 0) ok = mbar_wait_cluster(&tfull_bar[acc], use & 1, &s_abort, lim) && !s_abort;
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            tc_fence_after();
            int ks, mt, nt, kb0, kb1;
            unit(t, ks, mt, nt, kb0, kb1);
            const bool is_key = nt < key_tiles;
            const int br = is_key ? nt / kpb : 0;
            const int c0 = (is_key ? nt - br * kpb : nt - key_tiles) * BN;
            const int64_t rows0 = static_cast<int64_t>(mt) * kPairRows + static_cast<int>(rank) * kBM;
            const int64_t n = rows0 + row;
            const bool valid = n < p.n_tok;
            const uint32_t taddr = tmem_base + acc * BN + (static_cast<uint32_t>(sub * 32) << 16);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f;
            for (int cc = 0; cc < BN; cc += 32) {
                float accv[32];
                tmem_ld32(taddr + cc, accv);
                if constexpr (SPLIT) {
                    // raw partial accumulator, stored through the warp's 32 x 32 transpose tile so
                    // that each store instruction writes whole 128-byte row segments
                    float *tr = s_tr + sub * (32 * Cfg::kTrStride);
                    float4 *mine = reinterpret_cast<float4 *>(tr + lane * Cfg::kTrStride);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        mine[q] = make_float4(accv[4 * q], accv[4 * q + 1], accv[4 * q + 2], accv[4 * q + 3]);
                    __syncwarp();
                    const int c4 = (lane & 7) * 4;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = i * 4 + (lane >> 3);
                        const int64_t nr = rows0 + sub * 32 + r;
                        if (nr < p.n_tok)
                            *reinterpret_cast<float4 *>(p.acc_out + (static_cast<int64_t>(ks) * p.n_tok + nr) *
                                                                        (p.n_tiles * BN) + nt * BN + cc + c4) =
                                *reinterpret_cast<const float4 *>(tr + r * Cfg::kTrStride + c4);
                    }
                    __syncwarp();
                    continue;
                }
                if (valid) epilogue_chunk(p, accv, n, br, c0 + cc, is_key, a0, a1, a2);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty + acc * 8);   // to the even CTA's copy
            if constexpr (!SPLIT) {
                if (valid) p.part[n * p.n_tiles + nt] = make_float4(a0, a1, a2, 0.f);
            }
        }
    }
    tc_fence_before();
    cluster_sync();   // neither CTA leaves while the other may still reach its memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace engram
