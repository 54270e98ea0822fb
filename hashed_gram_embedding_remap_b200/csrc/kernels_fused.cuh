// Prefill steps 4-6 in ONE persistent tcgen05 kernel: projections, gate, RMSNorm, dilated
// depthwise conv (kernel 4, dilation 3), SiLU and residual.
//
// Work unit = a 128-row block of the flattened token axis that starts 9 rows before the
// block's first output token: rows 0..8 are the conv halo (the inputs u at t-9..t-1 that the
// block's first outputs need), rows 9..127 are outputs.  Consecutive units therefore advance
// by 119 tokens and recompute 9 rows (7.6% more MMA work) instead of exchanging the halo
// between CTAs.
//
// Per unit the MMA warp walks the 2*d_h/BN tiles of [k~ | v] -- key tiles first -- into two
// TMEM accumulators.  Eight epilogue warps (two per TMEM lane quarter, each taking half of
// the tile's columns) drain every tile:
//   key tile   -> per-row running sums S0 = sum h^2, S1 = sum h gamma_q gamma_k k~, S2 = sum k~^2
//   value tile -> per-row running sum S3 = sum v^2, and v (fp32) to the CTA's scratch
// After the last tile of a unit every row knows g = sigmoid(S1 / (rms_h rms_k sqrt d)) and
// beta = g / rms_U.  The conv pass of that unit then runs in 32-channel chunks interleaved
// with the tile drains of the CTA's NEXT unit (so the tensor cores keep working): for each
// chunk every thread writes u = beta v gamma_c of its row to shared memory, and after a
// named barrier computes c = sum_i w_i u[row - 3i] (zero before the sequence start),
// Delta = g v + c sigmoid(c) and out = bf16(h + Delta) for its output rows.
//
// Roles: warp 0 = TMA producer, warp 1 = TMEM owner + MMA issuer, warps 2..9 = epilogue.
// Every pipeline wait is bounded (see ptx.cuh).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "engram.h"
#include "kernels_gate.cuh"
#include "ptx.cuh"

namespace engram {

constexpr int kFusedHalo = 9;                    // (kernel 4 - 1) * dilation 3
constexpr int kFusedRows = kBM - kFusedHalo;     // output tokens per unit
constexpr int kFusedEpiWarps = 8;
constexpr int kFusedThreads = 64 + 32 * kFusedEpiWarps;
constexpr int kFusedChunk = 32;                  // channels per conv-pass chunk
constexpr int kFusedBarId = 1;                   // named barrier among the epilogue warps

template <int BN>
struct FusedCfg {
    static constexpr int kATile = kBM * kBK * 2;
    static constexpr int kBTile = BN * kBK * 2;
    static constexpr int kStageBytes = kATile + kBTile;
    static constexpr int kStages = (192 * 1024) / kStageBytes > 8 ? 8 : (192 * 1024) / kStageBytes;
    static constexpr int kTmemCols = 2 * BN;
    static constexpr int kUBytes = kBM * kFusedChunk * 4;               // u exchange buffer
    static constexpr int kStatBytes = 2 * 4 * kBM * 4;                  // two halves x S0..S3
    static constexpr int kBarBytes = (2 * kStages + 4) * 8;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kUBytes + kStatBytes + kBarBytes + 16;
};

struct FusedParams {
    const uint16_t *h;        // [n_tok, d_h]
    const uint16_t *gamma_q, *gamma_k, *gamma_c;   // [d_h]
    const uint16_t *conv_w;   // [d_h, 4]
    uint16_t *out;            // [n_tok, d_h]
    float *delta;             // [n_tok, d_h] or null
    float *vbuf;              // [gridDim.x, 2, d_h, 128] fp32 scratch (channel-major per unit)
    int64_t n_tok;
    int32_t T;                // tokens per sequence (positions restart every T tokens)
    int32_t d_m, d_h;
    int32_t k_blocks;
    int32_t n_units;
    float eps, inv_sqrt_d;
};

__device__ __forceinline__ void epi_bar_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kFusedBarId), "n"(32 * kFusedEpiWarps) : "memory");
}

// Named-barrier OR over the epilogue warps: true if any of them passes `pred`.  Used so that
// a failed (timed-out) wait ends the epilogue loop in every epilogue warp at the same point.
__device__ __forceinline__ bool epi_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "n"(kFusedBarId), "n"(32 * kFusedEpiWarps)
        : "memory");
    return r != 0;
}

template <int BN>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_proj_gate_kernel(const __grid_constant__ CUtensorMap map_m, const __grid_constant__ CUtensorMap map_wk,
                           const __grid_constant__ CUtensorMap map_wv, const __grid_constant__ FusedParams p) {
    using Cfg = FusedCfg<BN>;
    constexpr int S = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + S * Cfg::kATile;
    float *s_u = reinterpret_cast<float *>(smem + S * Cfg::kStageBytes);            // [32][128]
    float *s_stat = s_u + kBM * kFusedChunk;                                          // [2][4][128]
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(s_stat + 2 * 4 * kBM);
    uint64_t *empty_bar = full_bar + S;
    uint64_t *tfull_bar = empty_bar + S;
    uint64_t *tempty_bar = tfull_bar + 2;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(tempty_bar + 2);
    __shared__ int s_abort;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int key_tiles = p.d_h / BN;
    const int n_tiles = 2 * key_tiles;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], kFusedEpiWarps);
        }
        fence_barrier_init();
        tma_prefetch_desc(&map_m);
        tma_prefetch_desc(&map_wk);
        tma_prefetch_desc(&map_wv);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (warp == 0) {
        if (lane == 0) {
            int it = 0, issued = 0;
            for (int u = blockIdx.x; u < p.n_units && !s_abort; u += gridDim.x) {
                const int y0 = u * kFusedRows - kFusedHalo;     // first row of the block (may be < 0)
                for (int nt = 0; nt < n_tiles && !s_abort; ++nt) {
                    const bool is_key = nt < key_tiles;
                    const CUtensorMap *map_w = is_key ? &map_wk : &map_wv;
                    const int c0 = (is_key ? nt : nt - key_tiles) * BN;
                    for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                        const int s = it % S;
                        const uint32_t ph = (it / S) & 1;
                        if (!mbar_wait(&empty_bar[s], ph ^ 1, &s_abort)) break;
                        mbar_arrive_expect_tx(&full_bar[s], Cfg::kStageBytes);
                        tma_load_2d(sA + s * Cfg::kATile, &map_m, &full_bar[s], kb * kBK, y0);
                        tma_load_2d(sB + s * Cfg::kBTile, map_w, &full_bar[s], kb * kBK, c0);
                        issued = it + 1;
                    }
                }
            }
            if (s_abort) {
                volatile int never = 0;
                for (int k = issued - S > 0 ? issued - S : 0; k < issued; ++k)
                    if (!mbar_wait(&full_bar[k % S], (k / S) & 1, &never)) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
            int it = 0, li = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < p.n_units && ok && !s_abort; u += gridDim.x) {
                for (int nt = 0; nt < n_tiles && ok; ++nt, ++li) {
                    const int acc = li & 1;
                    const uint32_t use = li >> 1;
                    if (!mbar_wait(&tempty_bar[acc], (use & 1) ^ 1, &s_abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t dst = tmem_base + acc * BN;
                    for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                        const int s = it % S;
                        const uint32_t ph = (it / S) & 1;
                        if (!mbar_wait(&full_bar[s], ph, &s_abort)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t adesc = sdesc_kmajor_sw128(sA + s * Cfg::kATile);
                        const uint64_t bdesc = sdesc_kmajor_sw128(sB + s * Cfg::kBTile);
#pragma unroll
                        for (int k = 0; k < kBK / kUmmaK; ++k) {
                            const uint64_t koff = static_cast<uint64_t>((k * kUmmaK * 2) >> 4);
                            umma_bf16_ss(dst, adesc + koff, bdesc + koff, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                        }
                        umma_commit(&empty_bar[s]);
                    }
                    if (!ok) break;
                    umma_commit(&tfull_bar[acc]);
                }
            }
            if (s_abort) {
                for (int a = 0; a < 2; ++a) mbar_arrive(&tfull_bar[a]);
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue
        const int ew = warp - 2;                 // 0..7
        const int sub = warp & 3;                // TMEM lane quarter
        const int half = ew >> 2;                // which half of the tile's columns
        const int row = sub * 32 + lane;         // row of the block this thread drains
        const int etid = ew * 32 + lane;         // 0..255, conv-pass thread index
        const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
        float *vbuf0 = p.vbuf + static_cast<int64_t>(blockIdx.x) * 2 * kBM * p.d_h;
        // conv pass: thread etid handles row crow = etid & 127 and 16 channels (chalf) of a chunk
        const int crow = etid & (kBM - 1);
        const int chalf = etid >> 7;
        const int n_chunks = p.d_h / kFusedChunk;

        // state of the unit whose conv pass is pending
        int pend_unit = -1, pend_buf = 0;
        float pend_g = 0.f, pend_beta = 0.f;      // for row crow of the pending unit
        int next_chunk = 0;

        // one chunk of the pending unit's conv pass (all 256 epilogue threads take part)
        int pend_t = 0;                           // position of row crow of the pending unit in its sequence
        bool pend_ok = false;                     // row crow of the pending unit is a real token
        auto conv_chunk = [&](int ch) {
            const int cbase = ch * kFusedChunk + chalf * 16;
            const int64_t y0 = static_cast<int64_t>(pend_unit) * kFusedRows - kFusedHalo;
            const int64_t n = y0 + crow;
            // every load of the chunk is issued before the first use
            const float *vr = vbuf0 + (static_cast<int64_t>(pend_buf) * p.d_h + cbase) * kBM + crow;
            float vv[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) vv[e] = pend_ok ? vr[e * kBM] : 0.f;
            const uint4 *gcp = reinterpret_cast<const uint4 *>(p.gamma_c + cbase);
            const uint4 gc0 = __ldg(gcp), gc1 = __ldg(gcp + 1);
            const uint4 *cwp = reinterpret_cast<const uint4 *>(p.conv_w + cbase * 4);   // 16 channels x 4 taps
            uint4 cw[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) cw[q] = __ldg(cwp + q);
            const bool out_row = crow >= kFusedHalo && pend_ok;
            uint4 hw0 = make_uint4(0, 0, 0, 0), hw1 = hw0;
            if (out_row) {
                hw0 = __ldg(reinterpret_cast<const uint4 *>(p.h + n * p.d_h + cbase));
                hw1 = __ldg(reinterpret_cast<const uint4 *>(p.h + n * p.d_h + cbase + 8));
            }
            const uint32_t gcu[8] = {gc0.x, gc0.y, gc0.z, gc0.w, gc1.x, gc1.y, gc1.z, gc1.w};
            // s_u is [32 channels][128 rows]: consecutive rows (threads) hit consecutive banks
            float *ucol = s_u + (chalf * 16) * kBM + crow;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ucol[(2 * e) * kBM] = pend_beta * vv[2 * e] * bf16_lo(gcu[e]);
                ucol[(2 * e + 1) * kBM] = pend_beta * vv[2 * e + 1] * bf16_hi(gcu[e]);
            }
            epi_bar_sync();
            if (out_row) {
                const int t = pend_t;
                const uint32_t hu[8] = {hw0.x, hw0.y, hw0.z, hw0.w, hw1.x, hw1.y, hw1.z, hw1.w};
                const uint32_t cwu[16] = {cw[0].x, cw[0].y, cw[0].z, cw[0].w, cw[1].x, cw[1].y, cw[1].z, cw[1].w,
                                          cw[2].x, cw[2].y, cw[2].z, cw[2].w, cw[3].x, cw[3].y, cw[3].z, cw[3].w};
                const uint32_t cwv[16] = {cw[4].x, cw[4].y, cw[4].z, cw[4].w, cw[5].x, cw[5].y, cw[5].z, cw[5].w,
                                          cw[6].x, cw[6].y, cw[6].z, cw[6].w, cw[7].x, cw[7].y, cw[7].z, cw[7].w};
                uint32_t ob[8];
                float dl[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    // channel e's taps are words 2e and 2e+1 of the 16-channel block
                    const uint32_t wa = e < 8 ? cwu[2 * e] : cwv[2 * e - 16];
                    const uint32_t wb = e < 8 ? cwu[2 * e + 1] : cwv[2 * e + 1 - 16];
                    const float *uc = s_u + (chalf * 16 + e) * kBM + crow;
                    float c = bf16_lo(wa) * uc[0];
                    if (t >= 3) c = fmaf(bf16_hi(wa), uc[-3], c);
                    if (t >= 6) c = fmaf(bf16_lo(wb), uc[-6], c);
                    if (t >= 9) c = fmaf(bf16_hi(wb), uc[-9], c);
                    dl[e] = fmaf(pend_g, vv[e], c * fast_sigmoid(c));
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t lo = f32_to_bf16_bits(bf16_lo(hu[e]) + dl[2 * e]);
                    const uint32_t hi = f32_to_bf16_bits(bf16_hi(hu[e]) + dl[2 * e + 1]);
                    ob[e] = lo | (hi << 16);
                }
                uint4 *op = reinterpret_cast<uint4 *>(p.out + n * p.d_h + cbase);
                op[0] = make_uint4(ob[0], ob[1], ob[2], ob[3]);
                op[1] = make_uint4(ob[4], ob[5], ob[6], ob[7]);
                if (p.delta != nullptr) {
                    float4 *dp = reinterpret_cast<float4 *>(p.delta + n * p.d_h + cbase);
#pragma unroll
                    for (int q = 0; q < 4; ++q) dp[q] = make_float4(dl[4 * q], dl[4 * q + 1], dl[4 * q + 2], dl[4 * q + 3]);
                }
            }
            epi_bar_sync();   // s_u is rewritten by the next chunk
        };

        int li = 0;
        int local = 0;          // index of the unit within this CTA (selects the v scratch buffer)
        bool alive = true;
        for (int u = blockIdx.x; u < p.n_units && alive; u += gridDim.x, ++local) {
            const int64_t y0 = static_cast<int64_t>(u) * kFusedRows - kFusedHalo;
            const int64_t n = y0 + row;
            const bool valid = n >= 0 && n < p.n_tok;
            const int buf = local & 1;
            float *vcol = vbuf0 + static_cast<int64_t>(buf) * p.d_h * kBM + row;   // [d_h][128]
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            // chunks of the pending conv pass to run after each tile drain of this unit
            const int per_tile = (n_chunks + n_tiles - 1) / n_tiles;
            for (int nt = 0; nt < n_tiles; ++nt, ++li) {
                const int acc = li & 1;
                const uint32_t use = li >> 1;
                const bool got = mbar_wait(&tfull_bar[acc], use & 1, &s_abort);
                if (epi_any(!got)) { alive = false; break; }
                tc_fence_after();
                const bool is_key = nt < key_tiles;
                const int c0 = (is_key ? nt : nt - key_tiles) * BN + half * (BN / 2);
                const uint32_t taddr = tmem_base + acc * BN + half * (BN / 2) + lane_off;
                for (int cc = 0; cc < BN / 2; cc += 32) {
                    uint4 hq[4], gqq[4], gkq[4];
                    if (is_key && valid) {     // issue the loads first; they overlap the TMEM read
                        const uint4 *hp = reinterpret_cast<const uint4 *>(p.h + n * p.d_h + c0 + cc);
                        const uint4 *gq = reinterpret_cast<const uint4 *>(p.gamma_q + c0 + cc);
                        const uint4 *gk = reinterpret_cast<const uint4 *>(p.gamma_k + c0 + cc);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            hq[q] = __ldg(hp + q);
                            gqq[q] = __ldg(gq + q);
                            gkq[q] = __ldg(gk + q);
                        }
                    }
                    float accv[32];
                    tmem_ld32(taddr + cc, accv);
                    if (!valid) continue;
                    if (is_key) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 hw = hq[q], qw = gqq[q], kw = gkq[q];
                            const uint32_t h4[4] = {hw.x, hw.y, hw.z, hw.w};
                            const uint32_t q4[4] = {qw.x, qw.y, qw.z, qw.w};
                            const uint32_t k4[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = q * 8 + e * 2;
                                const float h0 = bf16_lo(h4[e]), h1 = bf16_hi(h4[e]);
                                const float k0 = accv[j], k1 = accv[j + 1];
                                a0 = fmaf(h0, h0, fmaf(h1, h1, a0));
                                a1 = fmaf(h0 * bf16_lo(q4[e]) * bf16_lo(k4[e]), k0,
                                          fmaf(h1 * bf16_hi(q4[e]) * bf16_hi(k4[e]), k1, a1));
                                a2 = fmaf(k0, k0, fmaf(k1, k1, a2));
                            }
                        }
                    } else {
                        float *vp = vcol + static_cast<int64_t>(c0 + cc) * kBM;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {   // a warp stores 32 consecutive rows of one channel
                            vp[j * kBM] = accv[j];
                            a3 = fmaf(accv[j], accv[j], a3);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty_bar[acc]);
                // interleave the pending unit's conv pass with this unit's MMAs
                if (pend_unit >= 0) {
                    for (int k = 0; k < per_tile && next_chunk < n_chunks; ++k) conv_chunk(next_chunk++);
                }
            }
            if (!alive) break;
            if (pend_unit >= 0) {                 // finish the previous unit's conv pass
                while (next_chunk < n_chunks) conv_chunk(next_chunk++);
            }
            // combine the two column halves' sums for each row, then the gate scalars of row crow
            s_stat[(half * 4 + 0) * kBM + row] = a0;
            s_stat[(half * 4 + 1) * kBM + row] = a1;
            s_stat[(half * 4 + 2) * kBM + row] = a2;
            s_stat[(half * 4 + 3) * kBM + row] = a3;
            __threadfence_block();                // v scratch writes visible to the conv pass
            epi_bar_sync();
            {
                const float s0 = s_stat[0 * kBM + crow] + s_stat[4 * kBM + crow];
                const float s1 = s_stat[1 * kBM + crow] + s_stat[5 * kBM + crow];
                const float s2 = s_stat[2 * kBM + crow] + s_stat[6 * kBM + crow];
                const float s3 = s_stat[3 * kBM + crow] + s_stat[7 * kBM + crow];
                const float inv_d = 1.f / static_cast<float>(p.d_h);
                const float rms_h = sqrtf(s0 * inv_d + p.eps);
                const float rms_k = sqrtf(s2 * inv_d + p.eps);
                pend_g = fast_sigmoid(s1 / (rms_h * rms_k) * p.inv_sqrt_d);
                pend_beta = pend_g / sqrtf(pend_g * pend_g * s3 * inv_d + p.eps);
            }
            epi_bar_sync();                       // s_stat is rewritten by the next unit
            pend_unit = u;
            pend_buf = buf;
            next_chunk = 0;
            {
                const int64_t nc = static_cast<int64_t>(u) * kFusedRows - kFusedHalo + crow;
                pend_ok = nc >= 0 && nc < p.n_tok;
                pend_t = pend_ok ? static_cast<int>(nc % p.T) : 0;
            }
        }
        if (alive && pend_unit >= 0) {
            while (next_chunk < n_chunks) conv_chunk(next_chunk++);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

}  // namespace engram
