// Step 4 of the lookup: the key and value projections [k~ | v] = m [W_k ; W_v]^T on the
// tcgen05 tensor cores, with the gate's per-token partial sums reduced in the epilogue.
//
// proj_kernel: persistent (grid = #SMs); CTA i takes work units i, i + grid, ...  A unit is
// a 128-token x BN-channel tile of [k~_0 | .. | k~_{M-1} | v] (the key tiles of the M branches
// first, branch-major, then the value tiles), or for decode-sized batches a K-slice of such a
// tile (split-K).  Warp 0 streams 128x64 tiles of m and BNx64 tiles of W
// with TMA (128-byte swizzle, no cluster multicast) through an S-stage shared-memory ring;
// warp 1 owns TMEM and issues tcgen05.mma (M=128, N=BN, K=16) into one of two accumulators;
// warps 2-5 drain the other accumulator with tcgen05.ld while the next unit's MMAs run.  The
// epilogue never writes k~: for a key tile it reduces, per token, S0 = sum h^2,
// S1 = sum h gamma_q gamma_k k~ and S2 = sum k~^2 over the tile's channels; for a value tile it
// writes v (fp16; S3 = sum v^2 from the fp32 values).  Split-K units write raw fp32 partial accumulators and
// splitk_reduce_kernel produces the same per-tile outputs.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "engram.h"
#include "ptx.cuh"

namespace engram {

constexpr int kBM = 128;          // tokens per tile (UMMA M)
constexpr int kBK = 64;           // K elements per stage: one 128-byte swizzle row
constexpr int kUmmaK = 16;        // K per tcgen05.mma for 16-bit inputs
constexpr int kProjThreads = 192; // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue

template <int BN>
struct ProjCfg {
    static constexpr int kATile = kBM * kBK * 2;                 // 16 KB
    static constexpr int kBTile = BN * kBK * 2;
    static constexpr int kStageBytes = kATile + kBTile;
    static constexpr int kStages = (200 * 1024) / kStageBytes > 8 ? 8 : (200 * 1024) / kStageBytes;
    static constexpr int kAccum = 2;                              // TMEM accumulators (double buffer)
    static constexpr int kTmemCols = kAccum * BN;                 // fp32 columns, power of two
    // split-K epilogue: one 32 x 32 fp32 transpose tile per epilogue warp (rows padded to 36
    // floats: 16-byte row starts, conflict-free quarter-warp phases)
    static constexpr int kTrStride = 36;
    static constexpr int kTrBytes = 4 * 32 * kTrStride * 4;
    // dynamic smem: [align pad][stages x A][stages x B][transpose tiles]
    //               [full, empty, tmem_full, tmem_empty][tmem addr]
    static constexpr int kBarBytes = (2 * kStages + 2 * kAccum) * 8;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kTrBytes + kBarBytes + 16;
};

struct ProjParams {
    const uint16_t *h;         // [n_tok, M, d_h] bf16
    const uint16_t *gamma_q;   // [d_h]
    const uint16_t *gamma_k;   // [d_h]
    uint16_t *v;               // [n_tok, d_h] fp16 out (rounded from the fp32 accumulator)
    float4 *part;              // [n_tok, n_tiles] partial sums out
    int64_t n_tok;
    int32_t d_m, d_h;
    int32_t n_tiles;           // (M + 1) * d_h / BN: key tiles (branch-major), then value tiles
    int32_t M;                 // branches (key projections)
    int32_t k_blocks;          // ceil(d_m / kBK)
    int32_t m_tiles;           // ceil(n_tok / kBM)
    int32_t k_splits;          // > 1: split-K, raw fp32 partial accumulators go to acc_out
    int32_t kb_per_split;      // k-blocks per split
    float *acc_out;            // [k_splits, n_tok, (M+1)*d_h] when k_splits > 1
    const uint8_t *w_packed;   // non-null: B tiles come as 32 KB pre-swizzled blocks (BN = 256)
    uint64_t wait_limit_ns;    // bound of every pipeline wait (0: ENGRAM_WAIT_TIMEOUT_NS)
    int32_t stall;             // self-test of the bounded waits: issue no loads at all, so that
                               // the first wait for a stage runs out and the kernel unwinds
};

// Packs [W_k ; W_v] into pre-swizzled 256 x 64 tiles (the layout engram_pack_weights
// documents): one thread per 16-byte chunk of the packed copy.
__global__ void pack_weights_kernel(const uint16_t *__restrict__ w_k, const uint16_t *__restrict__ w_v,
                                    int64_t key_rows, int32_t d_m, int32_t k_blocks, int64_t n_chunks,
                                    uint4 *__restrict__ packed) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_chunks;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t tile = i >> 11;                  // 2048 chunks of 16 B per 32 KB tile
        const int within = static_cast<int>(i & 2047);
        const int r = within >> 3, jp = within & 7;    // row in the tile, stored chunk position
        const int j = jp ^ (r & 7);                    // source chunk (8 columns)
        const int64_t t = tile / k_blocks;
        const int b = static_cast<int>(tile - t * k_blocks);
        const int64_t row = t * 256 + r;
        const int col = b * 64 + j * 8;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (col < d_m) {
            const uint16_t *src = row < key_rows ? w_k + row * d_m : w_v + (row - key_rows) * d_m;
            val = __ldg(reinterpret_cast<const uint4 *>(src + col));
        }
        packed[i] = val;
    }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}
// two floats -> two bf16 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Storage format of the value projection v between the projection and the gate kernels:
// IEEE fp16 (11 significant bits; v is a projection of bf16 rows by bf16 weights, orders of
// magnitude inside fp16's range).  Two values per 32-bit word, lo in the low half.
__device__ __forceinline__ uint32_t pack_v2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float v_lo(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
}
__device__ __forceinline__ float v_hi(uint32_t w) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
}

// Whole-K epilogue of one 32-column chunk of a token's accumulator row: for a key tile the
// gate's partial sums S0 = sum h^2, S1 = sum h gamma_q gamma_k k~, S2 = sum k~^2 over the
// chunk's channels; for a value tile the fp16 store of v and S3 = sum v^2 (in a0).
__device__ __forceinline__ void epilogue_chunk(const ProjParams &p, const float (&accv)[32], int64_t n, int br,
                                               int ch, bool is_key, float &a0, float &a1, float &a2) {
    if (is_key) {
        const uint4 *hp = reinterpret_cast<const uint4 *>(p.h + (n * p.M + br) * p.d_h + ch);
        const uint4 *gq = reinterpret_cast<const uint4 *>(p.gamma_q + ch);
        const uint4 *gk = reinterpret_cast<const uint4 *>(p.gamma_k + ch);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 hw = __ldg(hp + q), qw = __ldg(gq + q), kw = __ldg(gk + q);
            const uint32_t h4[4] = {hw.x, hw.y, hw.z, hw.w};
            const uint32_t q4[4] = {qw.x, qw.y, qw.z, qw.w};
            const uint32_t k4[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = q * 8 + e * 2;
                const float h0 = bf16_lo(h4[e]), h1 = bf16_hi(h4[e]);
                const float g0 = bf16_lo(q4[e]) * bf16_lo(k4[e]);
                const float g1 = bf16_hi(q4[e]) * bf16_hi(k4[e]);
                const float k0 = accv[j], k1 = accv[j + 1];
                a0 = fmaf(h0, h0, a0);
                a0 = fmaf(h1, h1, a0);
                a1 = fmaf(h0 * g0, k0, a1);
                a1 = fmaf(h1 * g1, k1, a1);
                a2 = fmaf(k0, k0, a2);
                a2 = fmaf(k1, k1, a2);
            }
        }
    } else {
        // S3 from the fp32 accumulator; v itself is stored as fp16
        uint4 *vp = reinterpret_cast<uint4 *>(p.v + n * p.d_h + ch);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float x0 = accv[8 * q + 2 * e], x1 = accv[8 * q + 2 * e + 1];
                a0 = fmaf(x0, x0, fmaf(x1, x1, a0));
                wv[e] = pack_v2(x0, x1);
            }
            vp[q] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
    }
}

// Persistent: grid = min(#tiles, #SMs); CTA i takes tiles i, i + grid, ...  Tile t covers
// tokens [128*(t / n_tiles), +128) and channel slice t % n_tiles, so the CTAs running at
// one time share a few 128-token blocks of m (re-read from L2) and stream all of W.
// Roles: warp 0 = TMA producer, warp 1 = TMEM owner + MMA issuer, warps 2-5 = epilogue.
// Two TMEM accumulators: the epilogue drains tile i while the MMAs of tile i+1 run.
// SPLIT: compiled for split-K work units (p.k_splits > 1, raw partial accumulators out) or
// for whole-K tiles only, so that neither epilogue costs the other registers.
template <int BN, bool SPLIT>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_kernel(const __grid_constant__ CUtensorMap map_m, const __grid_constant__ CUtensorMap map_wk,
                const __grid_constant__ CUtensorMap map_wv, const __grid_constant__ ProjParams p) {
    using Cfg = ProjCfg<BN>;
    constexpr int S = Cfg::kStages;
    constexpr int NACC = Cfg::kAccum;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + S * Cfg::kATile;
    float *s_tr = reinterpret_cast<float *>(smem + S * Cfg::kStageBytes);
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + S * Cfg::kStageBytes + Cfg::kTrBytes);
    uint64_t *empty_bar = full_bar + S;
    uint64_t *tfull_bar = empty_bar + S;      // MMA -> epilogue, one per accumulator
    uint64_t *tempty_bar = tfull_bar + NACC;  // epilogue -> MMA, one per accumulator
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(tempty_bar + NACC);
    __shared__ int s_abort;

    pdl_launch_dependents();   // the kernel after this one may load its independent inputs now
    const uint64_t lim = p.wait_limit_ns ? p.wait_limit_ns : ENGRAM_WAIT_TIMEOUT_NS;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int mn_tiles = p.m_tiles * p.n_tiles;
    const int total = mn_tiles * p.k_splits;   // work units: (k split, m tile, n tile), n fastest
    const int key_tiles = p.M * (p.d_h / BN);   // all branches
    const int kpb = p.d_h / BN;                 // key tiles per branch

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < NACC; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 4);   // one arrival per epilogue warp
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

    constexpr uint32_t kTxBytes = Cfg::kStageBytes;   // TMA bytes per stage: A + B
    if (warp == 0) {
        if (lane == 0 && !p.stall) {
            // unit t -> (k split, m tile, n tile) and the weight tile it streams
            auto unit = [&](int t, int &ks, int &mt, int &nt, int &kb0, int &kb1) {
                ks = t / mn_tiles;
                const int tmn = t - ks * mn_tiles;
                mt = tmn / p.n_tiles;
                nt = tmn - mt * p.n_tiles;
                kb0 = ks * p.kb_per_split;
                kb1 = min(p.k_blocks, kb0 + p.kb_per_split);
            };
            auto load_b = [&](int s, int nt, int kb) {
                const bool is_key = nt < key_tiles;
                if (BN == 256 && p.w_packed != nullptr)   // one linear 32 KB copy of the pre-swizzled tile
                    bulk_load_1d(sB + s * Cfg::kBTile, p.w_packed + (static_cast<int64_t>(nt) * p.k_blocks + kb) * Cfg::kBTile,
                                 Cfg::kBTile, &full_bar[s]);
                else   // row of the stacked W_k, or of W_v
                    tma_load_2d(sB + s * Cfg::kBTile, is_key ? &map_wk : &map_wv, &full_bar[s], kb * kBK,
                                (is_key ? nt : nt - key_tiles) * BN);
            };
            // The weight tiles of this CTA's first stages do not depend on the previous kernel on
            // the stream: they are issued before waiting for it (programmatic dependent launch);
            // the m tiles, which that kernel writes, follow the wait.
            int pre = 0;
            if (blockIdx.x < total) {
                int ks, mt, nt, kb0, kb1;
                unit(blockIdx.x, ks, mt, nt, kb0, kb1);
                pre = min(S, kb1 - kb0);
                for (int q = 0; q < pre; ++q) {   // fresh stages: nothing to wait for
                    mbar_arrive_expect_tx(&full_bar[q], kTxBytes);
                    load_b(q, nt, kb0 + q);
                }
            }
            pdl_wait();
            int it = 0, issued = pre;
            for (int t = blockIdx.x; t < total && !s_abort; t += gridDim.x) {
                int ks, mt, nt, kb0, kb1;
                unit(t, ks, mt, nt, kb0, kb1);
                const int m0 = mt * kBM;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S;
                    if (it < pre) {   // weight tile and byte count already issued
                        tma_load_2d(sA + s * Cfg::kATile, &map_m, &full_bar[s], kb * kBK, m0);
                        continue;
                    }
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait(&empty_bar[s], ph ^ 1, &s_abort, lim)) break;
                    mbar_arrive_expect_tx(&full_bar[s], kTxBytes);
                    tma_load_2d(sA + s * Cfg::kATile, &map_m, &full_bar[s], kb * kBK, m0);
                    load_b(s, nt, kb);
                    issued = it + 1;
                }
            }
            if (s_abort) {
                // Every issued copy must land before the CTA's shared memory is released.
                volatile int never = 0;
                for (int k = issued - S > 0 ? issued - S : 0; k < issued; ++k)
                    if (!mbar_wait(&full_bar[k % S], (k / S) & 1, &never, lim)) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
            int it = 0, li = 0;
            for (int t = blockIdx.x; t < total && !s_abort; t += gridDim.x, ++li) {
                const int acc = li % NACC;
                const uint32_t use = li / NACC;
                if (!mbar_wait(&tempty_bar[acc], (use & 1) ^ 1, &s_abort, lim)) break;
                tc_fence_after();
                const uint32_t dst = tmem_base + acc * BN;
                const int ks = t / mn_tiles;
                const int kb0 = ks * p.kb_per_split, kb1 = min(p.k_blocks, kb0 + p.kb_per_split);
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait(&full_bar[s], ph, &s_abort, lim)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = sdesc_kmajor_sw128(sA + s * Cfg::kATile);
                    const uint64_t bdesc = sdesc_kmajor_sw128(sB + s * Cfg::kBTile);
#pragma unroll
                    for (int k = 0; k < kBK / kUmmaK; ++k) {
                        const uint64_t koff = static_cast<uint64_t>((k * kUmmaK * 2) >> 4);
                        umma_bf16_ss(dst, adesc + koff, bdesc + koff, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty_bar[s]);   // frees the stage once these MMAs have read it
                }
                if (!ok) break;
                umma_commit(&tfull_bar[acc]);     // accumulator ready for the epilogue
            }
            if (s_abort) {
                for (int a = 0; a < NACC; ++a) mbar_arrive(&tfull_bar[a]);   // release waiting epilogue warps
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int sub = warp & 3;                      // TMEM lane quarter this warp may access
        const int row = sub * 32 + lane;
        int li = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++li) {
            const int acc = li % NACC;
            const uint32_t use = li / NACC;
            if (!mbar_wait(&tfull_bar[acc], use & 1, &s_abort, lim) || s_abort) break;
            tc_fence_after();
            const int ks = t / mn_tiles, tmn = t - ks * mn_tiles;
            const int mt = tmn / p.n_tiles, nt = tmn - mt * p.n_tiles;
            const bool is_key = nt < key_tiles;
            const int br = is_key ? nt / kpb : 0;                       // branch of a key tile
            const int c0 = (is_key ? nt - br * kpb : nt - key_tiles) * BN;   // channel within d_h
            const int64_t n = static_cast<int64_t>(mt) * kBM + row;
            const bool valid = n < p.n_tok;
            const uint32_t taddr = tmem_base + acc * BN + (static_cast<uint32_t>(sub * 32) << 16);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f;
            for (int cc = 0; cc < BN; cc += 32) {
                float accv[32];
                tmem_ld32(taddr + cc, accv);
                if constexpr (SPLIT) {
                    // split-K: raw partial accumulator; the reduction finishes the tile.  Each
                    // lane holds 32 columns of its own row: the warp's 32 x 32 block goes through
                    // shared memory so that every store instruction writes 4 whole 128-byte
                    // row segments instead of 32 scattered 16-byte pieces.
                    float *tr = s_tr + sub * (32 * Cfg::kTrStride);
                    float4 *mine = reinterpret_cast<float4 *>(tr + lane * Cfg::kTrStride);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        mine[q] = make_float4(accv[4 * q], accv[4 * q + 1], accv[4 * q + 2], accv[4 * q + 3]);
                    __syncwarp();
                    const int c4 = (lane & 7) * 4;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = i * 4 + (lane >> 3);                      // row within the warp's 32
                        const int64_t nr = static_cast<int64_t>(mt) * kBM + sub * 32 + r;
                        if (nr < p.n_tok)
                            *reinterpret_cast<float4 *>(p.acc_out + (static_cast<int64_t>(ks) * p.n_tok + nr) *
                                                                        (p.n_tiles * BN) + nt * BN + cc + c4) =
                                *reinterpret_cast<const float4 *>(tr + r * Cfg::kTrStride + c4);
                    }
                    __syncwarp();   // the tile is rewritten by the next column block
                    continue;
                }
                if (valid) epilogue_chunk(p, accv, n, br, c0 + cc, is_key, a0, a1, a2);
            }
            // the accumulator has been read: hand it back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[acc]);
            if constexpr (!SPLIT) {
                if (valid) p.part[n * p.n_tiles + nt] = make_float4(a0, a1, a2, 0.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

// Finishes a split-K projection: sums the k_splits partial accumulators of one token and one
// BN-wide tile, then produces exactly what the unsplit epilogue produces for that tile --
// (S0, S1, S2) for a key tile, v and S3 for a value tile.  Grid: (n_tiles, n_tok); block:
// kReduceThreads threads x 2 channels; fixed-order sums (deterministic).
constexpr int kReduceThreads = 128;

__global__ void __launch_bounds__(kReduceThreads) splitk_reduce_kernel(const __grid_constant__ ProjParams p, int BN) {
    __shared__ float s_red[3][kReduceThreads / 32];
    const int nt = blockIdx.x;
    const int64_t n = blockIdx.y;
    const int kpb = p.d_h / BN;
    const int key_tiles = p.M * kpb;
    const bool is_key = nt < key_tiles;
    const int br = is_key ? nt / kpb : 0;
    const int c0 = (is_key ? nt - br * kpb : nt - key_tiles) * BN;
    const int64_t row_len = static_cast<int64_t>(p.n_tiles) * BN;
    const int64_t stride_split = p.n_tok * row_len;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f;
    for (int j = threadIdx.x * 2; j < BN; j += kReduceThreads * 2) {
        const float *src = p.acc_out + n * row_len + nt * BN + j;
        float x0 = 0.f, x1 = 0.f;
        for (int ks = 0; ks < p.k_splits; ++ks) {
            const float2 q = __ldg(reinterpret_cast<const float2 *>(src + ks * stride_split));
            x0 += q.x;
            x1 += q.y;
        }
        if (is_key) {
            const uint32_t hw = __ldg(reinterpret_cast<const uint32_t *>(p.h + (n * p.M + br) * p.d_h + c0 + j));
            const uint32_t qw = __ldg(reinterpret_cast<const uint32_t *>(p.gamma_q + c0 + j));
            const uint32_t kw = __ldg(reinterpret_cast<const uint32_t *>(p.gamma_k + c0 + j));
            const float h0 = bf16_lo(hw), h1 = bf16_hi(hw);
            a0 = fmaf(h0, h0, fmaf(h1, h1, a0));
            a1 = fmaf(h0 * bf16_lo(qw) * bf16_lo(kw), x0, fmaf(h1 * bf16_hi(qw) * bf16_hi(kw), x1, a1));
            a2 = fmaf(x0, x0, fmaf(x1, x1, a2));
        } else {
            *reinterpret_cast<uint32_t *>(p.v + n * p.d_h + c0 + j) = pack_v2(x0, x1);
            a0 = fmaf(x0, x0, fmaf(x1, x1, a0));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a0 += __shfl_xor_sync(0xffffffffu, a0, o);
        a1 += __shfl_xor_sync(0xffffffffu, a1, o);
        a2 += __shfl_xor_sync(0xffffffffu, a2, o);
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0) {
        s_red[0][warp] = a0;
        s_red[1][warp] = a1;
        s_red[2][warp] = a2;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float b0 = 0.f, b1 = 0.f, b2 = 0.f;
        for (int w = 0; w < kReduceThreads / 32; ++w) {
            b0 += s_red[0][w];
            b1 += s_red[1][w];
            b2 += s_red[2][w];
        }
        p.part[n * p.n_tiles + nt] = make_float4(b0, b1, b2, 0.f);
    }
}

}  // namespace engram
