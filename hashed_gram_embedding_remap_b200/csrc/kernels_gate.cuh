// Steps 5-6 of the lookup (and the finishing of step 4's gate statistics): per-token gate
// scalars g = sigmoid(S1 / (rms_h rms_k sqrt(d))) and beta = g / rms_U from the projection
// partials; u = beta v gamma_c; c_t = sum_i w_i u_{t - i*dil}; Delta = g v + c sigmoid(c);
// out = bf16_rne(h + Delta).  Kernels: a generic one (any conv shape, optional carried
// state), the kernel-4 dilation-3 chain kernel for prefill and short stateful calls, the
// one-token decode kernels (with a carried conv state), and the fused split-K reduce + decode
// gate.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "engram.h"
#include "kernels_proj.cuh"
#include "ptx.cuh"

namespace engram {

struct GateParams {
    const uint16_t *h;        // [n_tok, M, d_h]
    const uint16_t *v;        // [n_tok, d_h] fp16 (pack_v2 / v_lo / v_hi), shared by the branches
    const float4 *part;       // [n_tok, n_tiles]
    const uint16_t *gamma_c;  // [d_h]
    const uint16_t *conv_w;   // [d_h, ksize]
    uint16_t *conv_state;     // [B, M, state_len, d_h] or null
    uint16_t *out;            // [n_tok, M, d_h]
    float *delta;             // [n_tok, M, d_h] or null
    int32_t B, T;
    int32_t d_h;
    int32_t n_tiles;          // (M + 1) * n_key_tiles: the key tiles of branch b are
                              // [b * n_key_tiles, (b + 1) * n_key_tiles), then the value tiles
    int32_t n_key_tiles;      // key tiles per branch
    int32_t M;                // branches
    int32_t ksize, dil, state_len;
    int32_t tok_chunk;        // tokens per CTA (T when a conv state is carried)
    float eps;
    float inv_sqrt_d;
    const float2 *scal;       // [n_tok] (g, beta) from gate_scalars_kernel, or null
    int32_t *history;         // decode_fused_kernel: [B, hist_len] hash history to advance, or null
    const int32_t *xr;        // with history: [B] remapped ids of this step
    int32_t hist_len;
};

__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + __expf(-z)); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

constexpr int kGateThreads = 128;

// Grid: (token chunks, B, channel slices of 4 * kGateThreads x M branches, branch fastest).
// One thread per 4 channels of one branch.  Dynamic smem: 2 floats (g, g/rms_U) per token of
// [t0 - state_len, t1).
__global__ void __launch_bounds__(kGateThreads) gate_conv_kernel(const __grid_constant__ GateParams p) {
    extern __shared__ float s_scal[];   // [2][tok_chunk + state_len]
    const int b = blockIdx.y;
    const int br = static_cast<int>(blockIdx.z % p.M);
    const int slice = static_cast<int>(blockIdx.z / p.M);
    const int64_t hrow = static_cast<int64_t>(p.M);   // rows of h / out per token
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
            for (int j = br * p.n_key_tiles; j < (br + 1) * p.n_key_tiles; ++j) {
                const float4 q = pp[j];
                s0 += q.x;
                s1 += q.y;
                s2 += q.z;
            }
            for (int j = p.M * p.n_key_tiles; j < p.n_tiles; ++j) s3 += pp[j].x;
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
    const int q = slice * blockDim.x + threadIdx.x;
    const int64_t sbase = (static_cast<int64_t>(b) * p.M + br) * p.state_len;   // conv state rows of (b, br)
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
                    const uint2 v4 = *reinterpret_cast<const uint2 *>(p.v + n * p.d_h + c);
                    vv[0] = v_lo(v4.x); vv[1] = v_hi(v4.x); vv[2] = v_lo(v4.y); vv[3] = v_hi(v4.y);
                    const float beta = s_beta[si];
#pragma unroll
                    for (int e = 0; e < 4; ++e) u[e] = beta * vv[e] * gc[e];
                } else if (p.conv_state != nullptr) {
                    const uint2 sw = *reinterpret_cast<const uint2 *>(
                        p.conv_state + (sbase + p.state_len + t) * p.d_h + c);
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
                const int64_t nr = n * hrow + br;   // row of (token, branch) in h / out / delta
                const float g = s_g[si];
                const uint2 hw = *reinterpret_cast<const uint2 *>(p.h + nr * p.d_h + c);
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
                *reinterpret_cast<uint2 *>(p.out + nr * p.d_h + c) = o;
                if (p.delta != nullptr)
                    *reinterpret_cast<float4 *>(p.delta + nr * p.d_h + c) = make_float4(dl[0], dl[1], dl[2], dl[3]);
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
                    const uint2 v4 = *reinterpret_cast<const uint2 *>(p.v + n * p.d_h + c);
                    const float beta = s_beta[t - lo];
                    const uint16_t u0 = f32_to_bf16_bits(beta * v_lo(v4.x) * gc[0]);
                    const uint16_t u1 = f32_to_bf16_bits(beta * v_hi(v4.x) * gc[1]);
                    const uint16_t u2 = f32_to_bf16_bits(beta * v_lo(v4.y) * gc[2]);
                    const uint16_t u3 = f32_to_bf16_bits(beta * v_hi(v4.y) * gc[3]);
                    o.x = static_cast<uint32_t>(u0) | (static_cast<uint32_t>(u1) << 16);
                    o.y = static_cast<uint32_t>(u2) | (static_cast<uint32_t>(u3) << 16);
                } else {
                    o = *reinterpret_cast<const uint2 *>(p.conv_state + (sbase + p.state_len + t) * p.d_h + c);
                }
                *reinterpret_cast<uint2 *>(p.conv_state + (sbase + s) * p.d_h + c) = o;
            }
        }
    }
}

// Per-(token, branch) gate scalars from the projection partials: scal[n*M + b] =
// (g_b, g_b / rms(U_b)).  Eight lanes per (token, branch) take every eighth of the branch's
// key tiles followed by the value tiles; a fixed-order butterfly over the eight lanes finishes
// the sums (deterministic).
__global__ void __launch_bounds__(256) gate_scalars_kernel(const float4 *__restrict__ part, int64_t n_tok,
                                                           int32_t n_tiles, int32_t n_key_tiles, int32_t M,
                                                           int32_t d_h, float eps, float inv_sqrt_d,
                                                           float2 *__restrict__ scal) {
    const int64_t gt = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t item = gt >> 3;          // (token, branch)
    const int sub = static_cast<int>(gt & 7);
    const int64_t n = item / M;
    const int br = static_cast<int>(item - n * M);
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    if (n < n_tok) {
        const float4 *pp = part + n * n_tiles;
        for (int j = sub; j < 2 * n_key_tiles; j += 8) {
            if (j < n_key_tiles) {
                const float4 q = __ldg(pp + br * n_key_tiles + j);
                s0 += q.x;
                s1 += q.y;
                s2 += q.z;
            } else {
                s3 += __ldg(pp + M * n_key_tiles + (j - n_key_tiles)).x;
            }
        }
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        s3 += __shfl_xor_sync(0xffffffffu, s3, o);
    }
    if (n < n_tok && sub == 0) {
        const float inv_d = 1.f / static_cast<float>(d_h);
        const float rms_h = sqrtf(s0 * inv_d + eps);
        const float rms_k = sqrtf(s2 * inv_d + eps);
        const float g = 1.f / (1.f + __expf(-(s1 / (rms_h * rms_k) * inv_sqrt_d)));
        scal[item] = make_float2(g, g / sqrtf(g * g * s3 * inv_d + eps));
    }
}

// x * sigmoid(x) = h + h * tanh(h) with h = x / 2, on the hardware tanh approximation
// (relative error about 2^-11).
__device__ __forceinline__ float silu_fast(float x) {
    const float h = 0.5f * x;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
}

// Fast path for the pages' conv shape (kernel 4, dilation 3): prefill, and decode with a
// carried conv state when one chunk covers the whole call (T <= 3*CH).
// Same arithmetic as gate_conv_kernel, organised for memory-level parallelism: a CTA covers
// 3*CH tokens of one sequence and 2*kGateFastThreads channels; each thread owns 2 channels
// and, for each residue r of the tokens mod 3, first issues every load of its chain -- CH + 3
// value rows (3 of them the conv halo) and CH hidden rows -- and only then computes, so a
// thread keeps ~35 independent loads in flight instead of walking a dependent chain.
constexpr int kGateFastThreads = 256;

__device__ __forceinline__ float fast_sigmoid(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

template <int CH>
__global__ void __launch_bounds__(kGateFastThreads, 3) gate_conv_k4d3_kernel(const __grid_constant__ GateParams p) {
    constexpr int KS = 4, DIL = 3, HALO = (KS - 1) * DIL, TC = CH * DIL;
    __shared__ float s_g[TC + HALO];
    __shared__ float s_beta[TC + HALO];
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * TC;
    if (t0 >= p.T) return;
    const int t1 = min(p.T, t0 + TC);
    const int lo = t0 - HALO;
    const float inv_d = 1.f / static_cast<float>(p.d_h);
    const int64_t row0 = static_cast<int64_t>(b) * p.T;

    // per-token scalars: precomputed by gate_scalars_kernel when p.scal is set, else one warp
    // per token reduces the tiles here
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (p.scal != nullptr) {
        for (int i = threadIdx.x; i < TC + HALO; i += kGateFastThreads) {
            const int t = lo + i;
            float2 sc = make_float2(0.f, 0.f);
            if (t >= 0 && t < t1) sc = __ldg(p.scal + row0 + t);
            s_g[i] = sc.x;
            s_beta[i] = sc.y;
        }
    }
    for (int i = warp; i < TC + HALO && p.scal == nullptr; i += kGateFastThreads / 32) {
        const int t = lo + i;
        float g = 0.f, beta = 0.f;
        if (t >= 0 && t < t1) {
            const float4 *pp = p.part + (row0 + t) * p.n_tiles;
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
            for (int j = lane; j < p.n_tiles; j += 32) {
                const float4 q = __ldg(pp + j);
                if (j < p.n_key_tiles) {
                    s0 += q.x;
                    s1 += q.y;
                    s2 += q.z;
                } else {
                    s3 += q.x;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s0 += __shfl_xor_sync(0xffffffffu, s0, o);
                s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                s2 += __shfl_xor_sync(0xffffffffu, s2, o);
                s3 += __shfl_xor_sync(0xffffffffu, s3, o);
            }
            const float rms_h = sqrtf(s0 * inv_d + p.eps);
            const float rms_k = sqrtf(s2 * inv_d + p.eps);
            g = fast_sigmoid(s1 / (rms_h * rms_k) * p.inv_sqrt_d);
            beta = g / sqrtf(g * g * s3 * inv_d + p.eps);
        }
        if (lane == 0) {
            s_g[i] = g;
            s_beta[i] = beta;
        }
    }
    __syncthreads();

    const int q = blockIdx.z * blockDim.x + threadIdx.x;
    if (q >= p.d_h / 2) return;
    const int c = q * 2;
    float gc[2], w[2][KS];
    {
        const uint32_t gw = __ldg(reinterpret_cast<const uint32_t *>(p.gamma_c + c));
        gc[0] = bf16_lo(gw);
        gc[1] = bf16_hi(gw);
        const uint2 *wp = reinterpret_cast<const uint2 *>(p.conv_w + c * KS);   // 2 channels x 4 taps
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const uint2 ww = __ldg(wp + e);
            w[e][0] = bf16_lo(ww.x); w[e][1] = bf16_hi(ww.x); w[e][2] = bf16_lo(ww.y); w[e][3] = bf16_hi(ww.y);
        }
    }
#pragma unroll 1
    for (int r = 0; r < DIL; ++r) {
        // raw bf16 pairs: v for positions in the call, the carried conv input u for positions
        // before it (decode), zero otherwise; every load is issued before any is used
        uint32_t vv[CH + KS - 1];
        uint32_t hh[CH];
#pragma unroll
        for (int j = 0; j < CH + KS - 1; ++j) {
            const int t = lo + r + DIL * j;
            const bool in_call = t >= 0 && t < t1;
            const bool carried = t < 0 && p.conv_state != nullptr;
            const uint16_t *src = in_call ? p.v + (row0 + t) * p.d_h + c
                                          : p.conv_state + (static_cast<int64_t>(b) * HALO + HALO + t) * p.d_h + c;
            vv[j] = (in_call || carried) ? *reinterpret_cast<const uint32_t *>(src) : 0u;
        }
#pragma unroll
        for (int j = 0; j < CH; ++j) {
            const int t = t0 + r + DIL * j;
            hh[j] = t < t1 ? __ldg(reinterpret_cast<const uint32_t *>(p.h + (row0 + t) * p.d_h + c)) : 0u;
        }
        float u[KS][2];   // u[i] holds the conv input i chain steps back
#pragma unroll
        for (int i = 0; i < KS; ++i) u[i][0] = u[i][1] = 0.f;
#pragma unroll
        for (int j = 0; j < CH + KS - 1; ++j) {
            const int si = r + DIL * j;            // index into s_g / s_beta
            const float beta = s_beta[si];
            const bool in_seq = lo + si >= 0;
            // positions in the call hold v (fp16); positions before it hold the carried u (bf16)
            const float vj[2] = {in_seq ? v_lo(vv[j]) : 0.f, in_seq ? v_hi(vv[j]) : 0.f};
#pragma unroll
            for (int i = KS - 1; i > 0; --i) {
                u[i][0] = u[i - 1][0];
                u[i][1] = u[i - 1][1];
            }
            if (in_seq) {
                u[0][0] = beta * vj[0] * gc[0];
                u[0][1] = beta * vj[1] * gc[1];
            } else {
                u[0][0] = bf16_lo(vv[j]);
                u[0][1] = bf16_hi(vv[j]);
            }
            if (j < KS - 1) continue;
            const int t = lo + si;
            if (t >= t1) continue;
            const float g = s_g[si];
            const uint32_t hw = hh[j - (KS - 1)];
            const float hv[2] = {bf16_lo(hw), bf16_hi(hw)};
            float dl[2];
            uint32_t ob[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < KS; ++i) acc = fmaf(w[e][i], u[i][e], acc);
                dl[e] = fmaf(g, vj[e], silu_fast(acc));
                ob[e] = f32_to_bf16_bits(hv[e] + dl[e]);
            }
            const int64_t n = row0 + t;
            *reinterpret_cast<uint32_t *>(p.out + n * p.d_h + c) = ob[0] | (ob[1] << 16);
            if (p.delta != nullptr)
                *reinterpret_cast<float2 *>(p.delta + n * p.d_h + c) = make_float2(dl[0], dl[1]);
        }
    }
    if (p.conv_state != nullptr) {
        // new state slot s <- conv input at position T - HALO + s; this CTA covers the whole
        // call (T <= TC), and each thread rewrites only its own channels, after reading them.
#pragma unroll 1
        for (int sl = 0; sl < HALO; ++sl) {
            const int t = p.T - HALO + sl;
            uint32_t o;
            if (t >= 0) {
                const uint32_t vw = __ldg(reinterpret_cast<const uint32_t *>(p.v + (row0 + t) * p.d_h + c));
                const float2 vt = make_float2(v_lo(vw), v_hi(vw));
                const float beta = s_beta[t - lo];
                o = static_cast<uint32_t>(f32_to_bf16_bits(beta * vt.x * gc[0])) |
                    (static_cast<uint32_t>(f32_to_bf16_bits(beta * vt.y * gc[1])) << 16);
            } else {
                o = *reinterpret_cast<const uint32_t *>(
                    p.conv_state + (static_cast<int64_t>(b) * HALO + HALO + t) * p.d_h + c);
            }
            *reinterpret_cast<uint32_t *>(p.conv_state + (static_cast<int64_t>(b) * HALO + sl) * p.d_h + c) = o;
        }
    }
}

// Prefill, kernel 4 / dilation 3, streaming form: a CTA owns 9*G consecutive tokens of one
// (sequence, branch) and 512 channels (4 per thread); each thread walks its tokens in order.
// Two 9-slot register rings replace a per-residue (t mod 3) decomposition: `ur` holds the
// conv inputs u of the last 9 positions (slot = position mod 9, so the taps t-3, t-6, t-9 sit
// in static slots of the unrolled loop), and the load ring holds (v, h) of the next 9
// positions -- the slot of token t is refilled with token t+9 as soon as t has read it, so
// every thread keeps 9 tokens of loads in flight instead of alternating load and compute
// phases.  The first group of 9 is the conv halo before the chunk (conv inputs only).
// Channel pairs go through the packed fp32x2 pipe (FFMA2 / FMUL2 / FADD2), about 8
// instructions per element; gamma_c is folded into the conv taps (u' = beta v, taps
// w_i gamma_c).  The kernel is issue- and latency-bound at 4 resident CTAs per SM (128
// registers).  Needs the per-(token, branch) scalars of gate_scalars_kernel.
constexpr int kStreamThreads = 128;
constexpr int kStreamMinBlocks = 4;

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 half2_to_f2(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&w));
}
__device__ __forceinline__ float2 bf162_to_f2(uint32_t w) { return make_float2(bf16_lo(w), bf16_hi(w)); }
// x * sigmoid(x) = h + h * tanh(h), h = x / 2, per pair (hardware tanh approximation)
__device__ __forceinline__ float2 silu2(float2 x) {
    const float2 h = __fmul2_rn(x, f2(0.5f));
    float2 t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t.x) : "f"(h.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(t.y) : "f"(h.y));
    return __ffma2_rn(h, t, h);
}

// One thread's walk over its CTA's tokens (see gate_stream_kernel).  FULL: the CTA's chunk is
// whole (t1 == t0 + 9G), so no token of the walk needs a bounds check.  Each load and store
// address advances by a fixed stride per token instead of being recomputed.
template <int G, bool DELTA, bool FULL>
__device__ __forceinline__ void gate_stream_walk(const GateParams &p, const float2 *s_sc, const float2 (&w)[4][2],
                                                 const uint16_t *vbase, const uint16_t *hbase, uint16_t *obase,
                                                 float *dbase, int lo, int t0, int t1) {
    constexpr int R = 9;
    const int64_t vstride = p.d_h;                               // elements per token of v
    const int64_t hstride = static_cast<int64_t>(p.M) * p.d_h;   // h / out / delta token stride
    uint2 lv[R], lh[R];     // load ring: (v, h) of the token in each slot
    float2 ur[R][2];        // conv-input ring: u' of the last 9 positions, slot = position mod 9
#pragma unroll
    for (int j = 0; j < R; ++j) {
        const int t = lo + j;   // halo: conv inputs only
        lv[j] = (t >= 0) ? __ldg(reinterpret_cast<const uint2 *>(vbase + static_cast<int64_t>(t) * vstride))
                         : make_uint2(0u, 0u);
        lh[j] = make_uint2(0u, 0u);
        ur[j][0] = ur[j][1] = make_float2(0.f, 0.f);
    }
    // next tokens to load: t0 (the first output token) onwards
    const uint16_t *vp = vbase + static_cast<int64_t>(t0) * vstride;
    const uint16_t *hp = hbase + static_cast<int64_t>(t0) * hstride;
    uint16_t *op = obase + static_cast<int64_t>(t0) * hstride;
    float *dp = DELTA ? dbase + static_cast<int64_t>(t0) * hstride : nullptr;
#pragma unroll 1
    for (int gi = 0; gi <= G; ++gi) {
        const int tb = lo + R * gi;
#pragma unroll
        for (int j = 0; j < R; ++j) {
            const int t = tb + j;
            const uint2 vw = lv[j], hw = lh[j];
            // refill the slot with token t + 9 (the next group)
            if (gi < G) {
                const bool in = FULL || t + R < t1;
                lv[j] = in ? __ldg(reinterpret_cast<const uint2 *>(vp)) : make_uint2(0u, 0u);
                lh[j] = in ? __ldg(reinterpret_cast<const uint2 *>(hp)) : make_uint2(0u, 0u);
                vp += vstride;
                hp += hstride;
            }
            const float2 sc = s_sc[t - lo];
            const float2 vj[2] = {half2_to_f2(vw.x), half2_to_f2(vw.y)};
            const float2 un[2] = {__fmul2_rn(f2(sc.y), vj[0]), __fmul2_rn(f2(sc.y), vj[1])};
            if (gi > 0) {
                if (FULL || t < t1) {
                    const uint32_t hh[2] = {hw.x, hw.y};
                    float2 dl[2];
                    uint32_t ob[2];
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        float2 acc = __fmul2_rn(w[0][k], un[k]);
                        acc = __ffma2_rn(w[1][k], ur[(j + 6) % R][k], acc);   // t - 3
                        acc = __ffma2_rn(w[2][k], ur[(j + 3) % R][k], acc);   // t - 6
                        acc = __ffma2_rn(w[3][k], ur[j][k], acc);             // t - 9
                        dl[k] = __ffma2_rn(f2(sc.x), vj[k], silu2(acc));     // U + SiLU(conv)
                        const float2 o = __fadd2_rn(bf162_to_f2(hh[k]), dl[k]);
                        ob[k] = pack_bf16x2(o.x, o.y);
                    }
                    *reinterpret_cast<uint2 *>(op) = make_uint2(ob[0], ob[1]);
                    if constexpr (DELTA)
                        *reinterpret_cast<float4 *>(dp) = make_float4(dl[0].x, dl[0].y, dl[1].x, dl[1].y);
                }
                op += hstride;
                if constexpr (DELTA) dp += hstride;
            }
            ur[j][0] = un[0];
            ur[j][1] = un[1];
        }
    }
}

template <int G, bool DELTA>
__global__ void __launch_bounds__(kStreamThreads, kStreamMinBlocks) gate_stream_kernel(const __grid_constant__ GateParams p) {
    constexpr int R = 9;                       // ring length = conv halo (kernel 4, dilation 3)
    constexpr int TC = R * G;                  // tokens per CTA
    __shared__ float2 s_sc[TC + R];            // (g, beta) per token of [t0 - 9, t0 + TC)
    // blockIdx.x = (chunk, branch, channel slice), slice fastest
    const int n_slices = (p.d_h / 4 + kStreamThreads - 1) / kStreamThreads;
    const int slice = static_cast<int>(blockIdx.x % n_slices);
    const int bx = static_cast<int>(blockIdx.x / n_slices);
    const int b = blockIdx.y;
    const int br = bx % p.M;
    const int t0 = (bx / p.M) * TC;
    if (t0 >= p.T) return;
    const int t1 = min(p.T, t0 + TC);
    const int lo = t0 - R;
    const int64_t row0 = static_cast<int64_t>(b) * p.T;
    for (int i = threadIdx.x; i < TC + R; i += kStreamThreads) {
        const int t = lo + i;
        s_sc[i] = (t >= 0 && t < t1) ? __ldg(p.scal + (row0 + t) * p.M + br) : make_float2(0.f, 0.f);
    }
    __syncthreads();
    const int q = slice * kStreamThreads + threadIdx.x;
    if (q >= p.d_h / 4) return;
    const int c = q * 4;
    float2 w[4][2];   // [tap][channel pair] = conv tap x gamma_c
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint32_t gw = __ldg(reinterpret_cast<const uint32_t *>(p.gamma_c + c + 2 * k));
        const uint4 ww = __ldg(reinterpret_cast<const uint4 *>(p.conv_w + (c + 2 * k) * 4));   // 2 channels x 4 taps
        const float g0 = bf16_lo(gw), g1 = bf16_hi(gw);
        w[0][k] = make_float2(bf16_lo(ww.x) * g0, bf16_lo(ww.z) * g1);
        w[1][k] = make_float2(bf16_hi(ww.x) * g0, bf16_hi(ww.z) * g1);
        w[2][k] = make_float2(bf16_lo(ww.y) * g0, bf16_lo(ww.w) * g1);
        w[3][k] = make_float2(bf16_hi(ww.y) * g0, bf16_hi(ww.w) * g1);
    }
    const uint16_t *vbase = p.v + row0 * p.d_h + c;
    const int64_t hoff = (row0 * p.M + br) * p.d_h + c;
    float *dbase = DELTA ? p.delta + hoff : nullptr;
    if (t1 - t0 == TC)
        gate_stream_walk<G, DELTA, true>(p, s_sc, w, vbase, p.h + hoff, p.out + hoff, dbase, lo, t0, t1);
    else
        gate_stream_walk<G, DELTA, false>(p, s_sc, w, vbase, p.h + hoff, p.out + hoff, dbase, lo, t0, t1);
}

// Decode step (T = 1) with a carried conv state, kernel 4 / dilation 3: the conv taps of the
// new token read state slots 6, 3 and 0 (positions t-3, t-6, t-9); the new state is slots
// 1..8 followed by u_t.  One CTA per (sequence, 512-channel slice); each thread loads all of
// its 2 channels' data (9 state slots, v, h) in one round trip, then computes and writes.
constexpr int kDecodeThreads = 256;

__global__ void __launch_bounds__(kDecodeThreads) gate_conv_decode_kernel(const __grid_constant__ GateParams p) {
    constexpr int S = 9;
    __shared__ float s_gb[2];
    pdl_launch_dependents();   // the history update may be scheduled now (it waits for this kernel)
    const int b = blockIdx.y;
    const float inv_d = 1.f / static_cast<float>(p.d_h);
    // this thread's loads that do not depend on the projection first
    const int q = blockIdx.x * blockDim.x + threadIdx.x;
    const bool active = q < p.d_h / 2;
    const int c = q * 2;
    uint32_t st[S];
    float2 v = make_float2(0.f, 0.f);
    uint32_t hw = 0, gw = 0;
    uint2 w0 = make_uint2(0, 0), w1 = make_uint2(0, 0);
    uint16_t *state = p.conv_state + static_cast<int64_t>(b) * S * p.d_h + c;
    if (active) {
#pragma unroll
        for (int k = 0; k < S; ++k) st[k] = *reinterpret_cast<const uint32_t *>(state + k * p.d_h);
        hw = __ldg(reinterpret_cast<const uint32_t *>(p.h + static_cast<int64_t>(b) * p.d_h + c));
        gw = __ldg(reinterpret_cast<const uint32_t *>(p.gamma_c + c));
        w0 = __ldg(reinterpret_cast<const uint2 *>(p.conv_w + c * 4));
        w1 = __ldg(reinterpret_cast<const uint2 *>(p.conv_w + (c + 1) * 4));
    }
    pdl_wait();   // v and the gate sums come from the projection kernel before this one
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const float4 *pp = p.part + static_cast<int64_t>(b) * p.n_tiles;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        for (int j = lane; j < p.n_tiles; j += 32) {
            const float4 e = __ldg(pp + j);
            if (j < p.n_key_tiles) {
                s0 += e.x;
                s1 += e.y;
                s2 += e.z;
            } else {
                s3 += e.x;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s0 += __shfl_xor_sync(0xffffffffu, s0, o);
            s1 += __shfl_xor_sync(0xffffffffu, s1, o);
            s2 += __shfl_xor_sync(0xffffffffu, s2, o);
            s3 += __shfl_xor_sync(0xffffffffu, s3, o);
        }
        if (lane == 0) {
            const float rms_h = sqrtf(s0 * inv_d + p.eps);
            const float rms_k = sqrtf(s2 * inv_d + p.eps);
            const float g = fast_sigmoid(s1 / (rms_h * rms_k) * p.inv_sqrt_d);
            s_gb[0] = g;
            s_gb[1] = g / sqrtf(g * g * s3 * inv_d + p.eps);
        }
    }
    if (active) {
        const uint32_t vw = __ldg(reinterpret_cast<const uint32_t *>(p.v + static_cast<int64_t>(b) * p.d_h + c));
        v = make_float2(v_lo(vw), v_hi(vw));
    }
    __syncthreads();
    if (!active) return;
    const float g = s_gb[0], beta = s_gb[1];
    const float u0 = beta * v.x * bf16_lo(gw), u1 = beta * v.y * bf16_hi(gw);
    // taps: i = 0 current, 1 -> slot 6 (t-3), 2 -> slot 3 (t-6), 3 -> slot 0 (t-9)
    const float c0 = fmaf(bf16_lo(w0.x), u0, fmaf(bf16_hi(w0.x), bf16_lo(st[6]),
                     fmaf(bf16_lo(w0.y), bf16_lo(st[3]), bf16_hi(w0.y) * bf16_lo(st[0]))));
    const float c1 = fmaf(bf16_lo(w1.x), u1, fmaf(bf16_hi(w1.x), bf16_hi(st[6]),
                     fmaf(bf16_lo(w1.y), bf16_hi(st[3]), bf16_hi(w1.y) * bf16_hi(st[0]))));
    const float d0 = fmaf(g, v.x, c0 * fast_sigmoid(c0));
    const float d1 = fmaf(g, v.y, c1 * fast_sigmoid(c1));
    const uint32_t o = static_cast<uint32_t>(f32_to_bf16_bits(bf16_lo(hw) + d0)) |
                       (static_cast<uint32_t>(f32_to_bf16_bits(bf16_hi(hw) + d1)) << 16);
    *reinterpret_cast<uint32_t *>(p.out + static_cast<int64_t>(b) * p.d_h + c) = o;
    if (p.delta != nullptr)
        *reinterpret_cast<float2 *>(p.delta + static_cast<int64_t>(b) * p.d_h + c) = make_float2(d0, d1);
#pragma unroll
    for (int k = 0; k < S - 1; ++k) *reinterpret_cast<uint32_t *>(state + k * p.d_h) = st[k + 1];
    *reinterpret_cast<uint32_t *>(state + (S - 1) * p.d_h) =
        static_cast<uint32_t>(f32_to_bf16_bits(u0)) | (static_cast<uint32_t>(f32_to_bf16_bits(u1)) << 16);
}

// Decode step (T = 1) after a split-K projection, fully fused: one CTA per token sums the
// k_splits partial accumulators of its [k~ | v] row, reduces S0..S3 across the block, then
// applies gate, conv (kernel 4, dilation 3, taps from the carried state or zeros), SiLU,
// residual and the state shift, and advances the token's hash history.  Replaces
// splitk_reduce_kernel + the gate kernel for decode.  d_h / 8 threads, 8 consecutive channels
// each, so that every access is 16 bytes wide (the 9 carried state slots, h, the gains, the
// taps, out and the new state as bf16 x 8; the split accumulators as fp32 x 4): about 25 wide
// loads per thread in one round trip, instead of ~80 narrow ones, which the load queues
// throttled.
constexpr int kFusedDecodeMaxThreads = 512;   // d_h <= 8 * 512 = 4096
// MAXT: the largest block this instantiation runs; 320 (d_h <= 2560) keeps two CTAs per SM
// (<= 102 registers), so a 256-sequence decode step runs in one wave.

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &w, float (&f)[8]) {
    f[0] = bf16_lo(w.x); f[1] = bf16_hi(w.x); f[2] = bf16_lo(w.y); f[3] = bf16_hi(w.y);
    f[4] = bf16_lo(w.z); f[5] = bf16_hi(w.z); f[6] = bf16_lo(w.w); f[7] = bf16_hi(w.w);
}

template <int MAXT>
__global__ void __launch_bounds__(MAXT, MAXT <= 320 ? 2 : 1) decode_fused_kernel(const __grid_constant__ ProjParams pp,
                                                                                const __grid_constant__ GateParams p) {
    constexpr int S = 9;
    __shared__ float s_red[4][MAXT / 32];
    __shared__ float s_gb[2];
    // dependents (the next step's kernels) may be scheduled now; the hash history, when given,
    // is advanced below by this kernel itself, after pdl_wait
    pdl_launch_dependents();
    const int b = blockIdx.x;
    const int d_h = p.d_h;
    const int c = threadIdx.x * 8;   // blockDim.x == d_h / 8, a multiple of 32
    const int64_t split_stride = pp.n_tok * (2 * d_h);
    const float *acc = pp.acc_out + static_cast<int64_t>(b) * (2 * d_h) + c;
    // Everything that does not depend on the projection first: the carried state, h, the
    // gains and the conv taps.  The state shift (slot j <- slot j + 1 for j < 8) needs only
    // the old state, so it is stored here too; only the three conv taps (slots 6, 3, 0 =
    // positions t-3, t-6, t-9) stay in registers across the wait.
    uint4 tap6 = make_uint4(0, 0, 0, 0), tap3 = tap6, tap0 = tap6;
    uint16_t *state = p.conv_state != nullptr ? p.conv_state + static_cast<int64_t>(b) * S * d_h + c : nullptr;
    if (state != nullptr) {
        uint4 st[S];
#pragma unroll
        for (int j = 0; j < S; ++j) st[j] = *reinterpret_cast<const uint4 *>(state + j * d_h);
        tap6 = st[6];
        tap3 = st[3];
        tap0 = st[0];
#pragma unroll
        for (int j = 0; j < S - 1; ++j) *reinterpret_cast<uint4 *>(state + j * d_h) = st[j + 1];
    }
    const uint4 hw = __ldg(reinterpret_cast<const uint4 *>(pp.h + static_cast<int64_t>(b) * d_h + c));
    const uint4 gqw = __ldg(reinterpret_cast<const uint4 *>(pp.gamma_q + c));
    const uint4 gkw = __ldg(reinterpret_cast<const uint4 *>(pp.gamma_k + c));
    const uint4 gcw = __ldg(reinterpret_cast<const uint4 *>(p.gamma_c + c));
    uint4 ww[4];   // conv taps: ww[q] holds channel c + 2q (x, y) and channel c + 2q + 1 (z, w)
#pragma unroll
    for (int q = 0; q < 4; ++q) ww[q] = __ldg(reinterpret_cast<const uint4 *>(p.conv_w + c * 4) + q);
    pdl_wait();   // the split accumulators come from the projection kernel before this one
    if (p.history != nullptr && threadIdx.x == 0) {
        // the step's hash history update (T = 1): drop the oldest id, append this step's.
        // The lookup that read the history finished before the projection did.
        int32_t *hb = p.history + static_cast<int64_t>(b) * p.hist_len;
        for (int s = 0; s + 1 < p.hist_len; ++s) hb[s] = hb[s + 1];
        hb[p.hist_len - 1] = p.xr[b];
    }
    float kt[8], v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) kt[e] = v[e] = 0.f;
    // in split order; unrolled by three so that the loads of three splits issue together
#pragma unroll 3
    for (int ks = 0; ks < pp.k_splits; ++ks) {
        const float4 *src = reinterpret_cast<const float4 *>(acc + ks * split_stride);
        const float4 k0 = __ldg(src), k1 = __ldg(src + 1);
        const float4 v0 = __ldg(src + d_h / 4), v1 = __ldg(src + d_h / 4 + 1);
        kt[0] += k0.x; kt[1] += k0.y; kt[2] += k0.z; kt[3] += k0.w;
        kt[4] += k1.x; kt[5] += k1.y; kt[6] += k1.z; kt[7] += k1.w;
        v[0] += v0.x; v[1] += v0.y; v[2] += v0.z; v[3] += v0.w;
        v[4] += v1.x; v[5] += v1.y; v[6] += v1.z; v[7] += v1.w;
    }
    float hf[8];
    bf16x8_to_f32(hw, hf);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    {
        float gq[8], gk[8];
        bf16x8_to_f32(gqw, gq);
        bf16x8_to_f32(gkw, gk);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            a0 = fmaf(hf[e], hf[e], a0);
            a1 = fmaf(hf[e] * gq[e] * gk[e], kt[e], a1);
            a2 = fmaf(kt[e], kt[e], a2);
            a3 = fmaf(v[e], v[e], a3);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a0 += __shfl_xor_sync(0xffffffffu, a0, o);
        a1 += __shfl_xor_sync(0xffffffffu, a1, o);
        a2 += __shfl_xor_sync(0xffffffffu, a2, o);
        a3 += __shfl_xor_sync(0xffffffffu, a3, o);
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0) {
        s_red[0][warp] = a0;
        s_red[1][warp] = a1;
        s_red[2][warp] = a2;
        s_red[3][warp] = a3;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        for (int w = 0; w < static_cast<int>(blockDim.x / 32); ++w) {
            s0 += s_red[0][w];
            s1 += s_red[1][w];
            s2 += s_red[2][w];
            s3 += s_red[3][w];
        }
        const float inv_d = 1.f / static_cast<float>(d_h);
        const float rms_h = sqrtf(s0 * inv_d + p.eps);
        const float rms_k = sqrtf(s2 * inv_d + p.eps);
        const float g = fast_sigmoid(s1 / (rms_h * rms_k) * p.inv_sqrt_d);
        s_gb[0] = g;
        s_gb[1] = g / sqrtf(g * g * s3 * inv_d + p.eps);
    }
    __syncthreads();
    const float g = s_gb[0], beta = s_gb[1];
    float gc[8], s6[8], s3f[8], s0f[8];
    bf16x8_to_f32(gcw, gc);
    bf16x8_to_f32(tap6, s6);    // position t-3
    bf16x8_to_f32(tap3, s3f);   // t-6
    bf16x8_to_f32(tap0, s0f);   // t-9
    float u[8], d[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {   // channel pairs
        const float w0[4] = {bf16_lo(ww[q].x), bf16_hi(ww[q].x), bf16_lo(ww[q].y), bf16_hi(ww[q].y)};
        const float w1[4] = {bf16_lo(ww[q].z), bf16_hi(ww[q].z), bf16_lo(ww[q].w), bf16_hi(ww[q].w)};
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const int e = 2 * q + e2;
            const float *w = e2 == 0 ? w0 : w1;
            u[e] = beta * v[e] * gc[e];
            const float cv = fmaf(w[0], u[e], fmaf(w[1], s6[e], fmaf(w[2], s3f[e], w[3] * s0f[e])));
            d[e] = fmaf(g, v[e], cv * fast_sigmoid(cv));
        }
    }
    uint4 o;
    o.x = pack_bf16x2(hf[0] + d[0], hf[1] + d[1]);
    o.y = pack_bf16x2(hf[2] + d[2], hf[3] + d[3]);
    o.z = pack_bf16x2(hf[4] + d[4], hf[5] + d[5]);
    o.w = pack_bf16x2(hf[6] + d[6], hf[7] + d[7]);
    *reinterpret_cast<uint4 *>(p.out + static_cast<int64_t>(b) * d_h + c) = o;
    if (p.delta != nullptr) {
        float4 *dp = reinterpret_cast<float4 *>(p.delta + static_cast<int64_t>(b) * d_h + c);
        dp[0] = make_float4(d[0], d[1], d[2], d[3]);
        dp[1] = make_float4(d[4], d[5], d[6], d[7]);
    }
    if (state != nullptr)   // the new slot 8: this token's conv input (slots 0..7 were shifted above)
        *reinterpret_cast<uint4 *>(state + (S - 1) * d_h) =
            make_uint4(pack_bf16x2(u[0], u[1]), pack_bf16x2(u[2], u[3]), pack_bf16x2(u[4], u[5]), pack_bf16x2(u[6], u[7]));
}

}  // namespace engram
