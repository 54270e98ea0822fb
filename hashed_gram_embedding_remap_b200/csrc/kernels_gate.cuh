// Steps 4-6 of the lookup.
//
// (a) proj_kernel: the value and key projections [k~ | v] = m [W_k ; W_v]^T on the tcgen05
//     tensor cores.  One CTA computes a 128-token x BN-channel tile: a TMA producer warp
//     streams 128x64 tiles of m and BNx64 tiles of W (128-byte swizzle) through an S-stage
//     shared-memory ring, one thread issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM
//     accumulator, and four epilogue warps read the accumulator back with tcgen05.ld.  The
//     epilogue never writes k~: for a key tile it reduces, per token, the three partial sums
//     the gate needs over the tile's channels --
//         S0 = sum h^2,  S1 = sum h * gamma_q * gamma_k * k~,  S2 = sum k~^2
//     -- and for a value tile it writes v (fp32) and S3 = sum v^2.  The gate kernel combines
//     the partials of all tiles in a fixed order (deterministic, no atomics).
// (b) gate_conv_kernel: per token, g = sigmoid(S1 / (rms_h rms_k sqrt(d))), with
//     rms_h = sqrt(S0/d + eps), rms_k = sqrt(S2/d + eps); U = g v; u = U / rms_U * gamma_c with
//     rms_U = sqrt(g^2 S3 / d + eps); c_t = sum_i w_i u_{t - i*dil}; Delta = U + c sigmoid(c);
//     out = bf16_rne(h + Delta).  Each thread owns 4 channels and walks the tokens of one
//     residue class modulo the dilation, so the dilated conv becomes a dense 4-tap shift
//     register in registers.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

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
    static constexpr int kTmemCols = BN;                          // fp32 accumulator columns
    // dynamic smem: [align pad][stages x A][stages x B][barriers][gamma_qk BN floats][tmem addr]
    static constexpr int kBarBytes = (2 * kStages + 1) * 8;
    static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes + BN * 4 + 16;
};

struct ProjParams {
    const uint16_t *h;         // [n_tok, d_h] bf16
    const uint16_t *gamma_q;   // [d_h]
    const uint16_t *gamma_k;   // [d_h]
    float *v;                  // [n_tok, d_h] fp32 out
    float4 *part;              // [n_tok, n_tiles] partial sums out
    int64_t n_tok;
    int32_t d_m, d_h;
    int32_t n_tiles;           // 2 * d_h / BN: key tiles first, then value tiles
    int32_t k_blocks;          // ceil(d_m / kBK)
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

template <int BN>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_kernel(const __grid_constant__ CUtensorMap map_m, const __grid_constant__ CUtensorMap map_wk,
                const __grid_constant__ CUtensorMap map_wv, const __grid_constant__ ProjParams p) {
    using Cfg = ProjCfg<BN>;
    constexpr int S = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + S * Cfg::kATile;
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + S * Cfg::kStageBytes);
    uint64_t *empty_bar = full_bar + S;
    uint64_t *accum_bar = empty_bar + S;
    float *s_gqk = reinterpret_cast<float *>(accum_bar + 1);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(s_gqk + BN);
    __shared__ int s_abort;

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int tile_n = blockIdx.x;                 // which BN-wide slice of [k~ | v]
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
    const bool is_key = tile_n * BN < p.d_h;
    const int c0 = is_key ? tile_n * BN : tile_n * BN - p.d_h;   // channel offset in d_h

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(accum_bar, 1);
        fence_barrier_init();
        tma_prefetch_desc(&map_m);
        tma_prefetch_desc(is_key ? &map_wk : &map_wv);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, Cfg::kTmemCols);
        tmem_relinquish();
    }
    if (warp >= 2) {
        for (int c = threadIdx.x - 64; c < BN; c += 128)
            s_gqk[c] = is_key ? bf16_bits_to_f32(p.gamma_q[c0 + c]) * bf16_bits_to_f32(p.gamma_k[c0 + c]) : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;

    if (warp == 0) {
        if (lane == 0) {
            const CUtensorMap *map_w = is_key ? &map_wk : &map_wv;
            int issued = 0;
            for (int kb = 0; kb < p.k_blocks; ++kb) {
                const int s = kb % S;
                const uint32_t ph = (kb / S) & 1;
                if (!mbar_wait(&empty_bar[s], ph ^ 1, &s_abort)) break;
                mbar_arrive_expect_tx(&full_bar[s], Cfg::kStageBytes);
                tma_load_2d(sA + s * Cfg::kATile, &map_m, &full_bar[s], kb * kBK, static_cast<int>(m0));
                tma_load_2d(sB + s * Cfg::kBTile, map_w, &full_bar[s], kb * kBK, c0);
                ++issued;
            }
            if (s_abort) {
                // Every issued copy must land before the CTA's shared memory is released.
                volatile int never = 0;
                for (int kb = issued - S > 0 ? issued - S : 0; kb < issued; ++kb)
                    if (!mbar_wait(&full_bar[kb % S], (kb / S) & 1, &never)) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
            bool ok = true;
            for (int kb = 0; kb < p.k_blocks; ++kb) {
                const int s = kb % S;
                const uint32_t ph = (kb / S) & 1;
                if (!mbar_wait(&full_bar[s], ph, &s_abort)) { ok = false; break; }
                tc_fence_after();
                const uint64_t adesc = sdesc_kmajor_sw128(sA + s * Cfg::kATile);
                const uint64_t bdesc = sdesc_kmajor_sw128(sB + s * Cfg::kBTile);
#pragma unroll
                for (int k = 0; k < kBK / kUmmaK; ++k) {
                    // advance 16 elements (32 bytes) along K inside the swizzled row
                    const uint64_t koff = static_cast<uint64_t>((k * kUmmaK * 2) >> 4);
                    umma_bf16_ss(tmem_base, adesc + koff, bdesc + koff, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&empty_bar[s]);  // frees the stage once these MMAs have read it
            }
            if (ok) umma_commit(accum_bar);
            else mbar_arrive(accum_bar);    // release the epilogue; it sees s_abort
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int sub = warp & 3;                      // TMEM lane quarter this warp may access
        const int row = sub * 32 + lane;
        const int64_t n = m0 + row;
        const bool valid = n < p.n_tok;
        const bool got = mbar_wait(accum_bar, 0, &s_abort) && !s_abort;
        tc_fence_after();
        float a0 = 0.f, a1 = 0.f, a2 = 0.f;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sub * 32) << 16);
        if (got) {
            for (int cc = 0; cc < BN; cc += 32) {
                float acc[32];
                tmem_ld32(taddr + cc, acc);
                if (!valid) continue;
                if (is_key) {
                    const uint4 *hp = reinterpret_cast<const uint4 *>(p.h + n * p.d_h + c0 + cc);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 hw = __ldg(hp + q);
                        const uint32_t w4[4] = {hw.x, hw.y, hw.z, hw.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = q * 8 + e * 2;
                            const float h0 = bf16_lo(w4[e]), h1 = bf16_hi(w4[e]);
                            const float k0 = acc[j], k1 = acc[j + 1];
                            a0 = fmaf(h0, h0, a0);
                            a0 = fmaf(h1, h1, a0);
                            a1 = fmaf(h0 * s_gqk[cc + j], k0, a1);
                            a1 = fmaf(h1 * s_gqk[cc + j + 1], k1, a1);
                            a2 = fmaf(k0, k0, a2);
                            a2 = fmaf(k1, k1, a2);
                        }
                    }
                } else {
                    float4 *vp = reinterpret_cast<float4 *>(p.v + n * p.d_h + c0 + cc);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 x = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
                        vp[q] = x;
                        a0 = fmaf(x.x, x.x, a0);
                        a0 = fmaf(x.y, x.y, a0);
                        a0 = fmaf(x.z, x.z, a0);
                        a0 = fmaf(x.w, x.w, a0);
                    }
                }
            }
            if (valid) p.part[n * p.n_tiles + tile_n] = make_float4(a0, a1, a2, 0.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

struct GateParams {
    const uint16_t *h;        // [n_tok, d_h]
    const float *v;           // [n_tok, d_h]
    const float4 *part;       // [n_tok, n_tiles]
    const uint16_t *gamma_c;  // [d_h]
    const uint16_t *conv_w;   // [d_h, ksize]
    uint16_t *conv_state;     // [B, state_len, d_h] or null
    uint16_t *out;            // [n_tok, d_h]
    float *delta;             // [n_tok, d_h] or null
    int32_t B, T;
    int32_t d_h;
    int32_t n_tiles;          // total tiles; the first n_key_tiles are key tiles
    int32_t n_key_tiles;
    int32_t ksize, dil, state_len;
    int32_t tok_chunk;        // tokens per CTA (T when a conv state is carried)
    float eps;
    float inv_sqrt_d;
};

__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + __expf(-z)); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

constexpr int kGateThreads = 128;

// Grid: (token chunks, B, channel slices of 4 * kGateThreads).  One thread per 4 channels.
// Dynamic smem: 2 floats (g, g/rms_U) per token of [t0 - state_len, t1).
__global__ void __launch_bounds__(kGateThreads) gate_conv_kernel(const __grid_constant__ GateParams p) {
    extern __shared__ float s_scal[];   // [2][tok_chunk + state_len]
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * p.tok_chunk;
    if (t0 >= p.T) return;
    const int t1 = min(p.T, t0 + p.tok_chunk);
    const int lo = t0 - p.state_len;           // first token whose conv input is needed
    const int span = t1 - lo;
    float *s_g = s_scal;
    float *s_beta = s_scal + span;
    const float inv_d = 1.f / static_cast<float>(p.d_h);

    // per-token scalars from the projection partials (fixed summation order)
    for (int i = threadIdx.x; i < span; i += blockDim.x) {
        const int t = lo + i;
        float g = 0.f, beta = 0.f;
        if (t >= 0) {
            const float4 *pp = p.part + (static_cast<int64_t>(b) * p.T + t) * p.n_tiles;
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
            for (int j = 0; j < p.n_key_tiles; ++j) {
                const float4 q = pp[j];
                s0 += q.x;
                s1 += q.y;
                s2 += q.z;
            }
            for (int j = p.n_key_tiles; j < p.n_tiles; ++j) s3 += pp[j].x;
            const float rms_h = sqrtf(s0 * inv_d + p.eps);
            const float rms_k = sqrtf(s2 * inv_d + p.eps);
            g = sigmoidf_(s1 / (rms_h * rms_k) * p.inv_sqrt_d);
            const float rms_u = sqrtf(g * g * s3 * inv_d + p.eps);
            beta = g / rms_u;
        }
        s_g[i] = g;
        s_beta[i] = beta;
    }
    __syncthreads();

    const int nq = p.d_h / 4;
    const int q = blockIdx.z * blockDim.x + threadIdx.x;
    if (q < nq) {
        const int c = q * 4;
        float gc[4], w[4][8];
        {
            const uint2 gw = *reinterpret_cast<const uint2 *>(p.gamma_c + c);
            gc[0] = bf16_lo(gw.x); gc[1] = bf16_hi(gw.x); gc[2] = bf16_lo(gw.y); gc[3] = bf16_hi(gw.y);
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    w[e][i] = i < p.ksize ? bf16_bits_to_f32(p.conv_w[(c + e) * p.ksize + i]) : 0.f;
        }
        for (int r = 0; r < p.dil; ++r) {
            // shift register over the chain lo+r, lo+r+dil, ...: hist[i] holds u at t - i*dil
            float hist[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) hist[i][e] = 0.f;
            for (int t = lo + r; t < t1; t += p.dil) {
                float u[4], vv[4];
                const int si = t - lo;
                if (t >= 0) {
                    const int64_t n = static_cast<int64_t>(b) * p.T + t;
                    const float4 v4 = *reinterpret_cast<const float4 *>(p.v + n * p.d_h + c);
                    vv[0] = v4.x; vv[1] = v4.y; vv[2] = v4.z; vv[3] = v4.w;
                    const float beta = s_beta[si];
#pragma unroll
                    for (int e = 0; e < 4; ++e) u[e] = beta * vv[e] * gc[e];
                } else if (p.conv_state != nullptr) {
                    const uint2 sw = *reinterpret_cast<const uint2 *>(
                        p.conv_state + (static_cast<int64_t>(b) * p.state_len + p.state_len + t) * p.d_h + c);
                    u[0] = bf16_lo(sw.x); u[1] = bf16_hi(sw.x); u[2] = bf16_lo(sw.y); u[3] = bf16_hi(sw.y);
                    vv[0] = vv[1] = vv[2] = vv[3] = 0.f;
                } else {
                    u[0] = u[1] = u[2] = u[3] = 0.f;
                    vv[0] = vv[1] = vv[2] = vv[3] = 0.f;
                }
#pragma unroll
                for (int i = 7; i > 0; --i)
#pragma unroll
                    for (int e = 0; e < 4; ++e) hist[i][e] = hist[i - 1][e];
#pragma unroll
                for (int e = 0; e < 4; ++e) hist[0][e] = u[e];
                if (t < t0) continue;
                const int64_t n = static_cast<int64_t>(b) * p.T + t;
                const float g = s_g[si];
                const uint2 hw = *reinterpret_cast<const uint2 *>(p.h + n * p.d_h + c);
                const float hv[4] = {bf16_lo(hw.x), bf16_hi(hw.x), bf16_lo(hw.y), bf16_hi(hw.y)};
                float dl[4];
                uint16_t ob[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float acc = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (i < p.ksize) acc = fmaf(w[e][i], hist[i][e], acc);
                    dl[e] = g * vv[e] + acc * sigmoidf_(acc);
                    ob[e] = f32_to_bf16_bits(hv[e] + dl[e]);
                }
                uint2 o;
                o.x = static_cast<uint32_t>(ob[0]) | (static_cast<uint32_t>(ob[1]) << 16);
                o.y = static_cast<uint32_t>(ob[2]) | (static_cast<uint32_t>(ob[3]) << 16);
                *reinterpret_cast<uint2 *>(p.out + n * p.d_h + c) = o;
                if (p.delta != nullptr)
                    *reinterpret_cast<float4 *>(p.delta + n * p.d_h + c) = make_float4(dl[0], dl[1], dl[2], dl[3]);
            }
        }
        if (p.conv_state != nullptr) {
            // new state slot s <- conv input at position T - state_len + s (this CTA covers
            // the whole sequence).  Increasing s reads slot s + T >= s before it is rewritten.
            for (int s = 0; s < p.state_len; ++s) {
                const int t = p.T - p.state_len + s;
                uint2 o;
                if (t >= 0) {
                    const int64_t n = static_cast<int64_t>(b) * p.T + t;
                    const float4 v4 = *reinterpret_cast<const float4 *>(p.v + n * p.d_h + c);
                    const float beta = s_beta[t - lo];
                    const uint16_t u0 = f32_to_bf16_bits(beta * v4.x * gc[0]);
                    const uint16_t u1 = f32_to_bf16_bits(beta * v4.y * gc[1]);
                    const uint16_t u2 = f32_to_bf16_bits(beta * v4.z * gc[2]);
                    const uint16_t u3 = f32_to_bf16_bits(beta * v4.w * gc[3]);
                    o.x = static_cast<uint32_t>(u0) | (static_cast<uint32_t>(u1) << 16);
                    o.y = static_cast<uint32_t>(u2) | (static_cast<uint32_t>(u3) << 16);
                } else {
                    o = *reinterpret_cast<const uint2 *>(
                        p.conv_state + (static_cast<int64_t>(b) * p.state_len + p.state_len + t) * p.d_h + c);
                }
                *reinterpret_cast<uint2 *>(p.conv_state + (static_cast<int64_t>(b) * p.state_len + s) * p.d_h + c) = o;
            }
        }
    }
}

}  // namespace engram
