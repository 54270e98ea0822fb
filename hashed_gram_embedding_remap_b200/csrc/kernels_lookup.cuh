// Steps 1-3 of the lookup: remap + n-gram hashing (one fused kernel), row gather into the
// concatenated memory vector, and the decode-history update.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "engram.h"

#include "status.cuh"

namespace engram {

struct HashParams {
    uint64_t mult[ENGRAM_MAX_TABLES][ENGRAM_MAX_ORDERS];  // a_{o,j,i}, i = 0 is the current token
    uint64_t prime[ENGRAM_MAX_TABLES];
    int32_t order[ENGRAM_MAX_TABLES];                     // n-gram order of table h
    int32_t H;
    int32_t max_order;
    int32_t hist_len;
    int32_t pad_id;
    int32_t vocab_in;
    int32_t B, T;
};

// MurmurHash3's 64-bit finaliser (Appleby, public domain).
__device__ __forceinline__ uint64_t fmix64(uint64_t k) {
    k ^= k >> 33;
    k *= 0xFF51AFD7ED558CCDull;
    k ^= k >> 33;
    k *= 0xC4CEB9FE1A85EC53ull;
    k ^= k >> 33;
    return k;
}

// One thread per token.  Reads the token and the (max_order - 1) before it (remapping each
// through `remap` when given), then for every table h forms the gram of its order and writes
// idx[n, h] = fmix64(XOR_i (x'_{t-i} + 1) * a_{h,i}) mod P_h.
// Token ids outside [0, vocab_in) read as the pad id and raise ENGRAM_STATUS_BAD_TOKEN.
__global__ void __launch_bounds__(256) hash_kernel(const int32_t *__restrict__ ids,
                                                   const int32_t *__restrict__ remap,
                                                   const int32_t *__restrict__ history,
                                                   uint32_t *__restrict__ idx,
                                                   int32_t *__restrict__ xr_out,
                                                   const __grid_constant__ HashParams p) {
    const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t n_tok = static_cast<int64_t>(p.B) * p.T;
    if (n >= n_tok) return;
    const int32_t b = static_cast<int32_t>(n / p.T);
    const int32_t t = static_cast<int32_t>(n - static_cast<int64_t>(b) * p.T);

    uint64_t xp1[ENGRAM_MAX_ORDERS];  // x'_{t-i} + 1
#pragma unroll
    for (int i = 0; i < ENGRAM_MAX_ORDERS; ++i) {
        if (i >= p.max_order) break;
        const int32_t pos = t - i;
        int32_t x;
        if (pos >= 0) {
            int32_t raw = __ldg(ids + (n - i));
            if (remap != nullptr) {
                if (raw >= 0 && raw < p.vocab_in) {
                    x = __ldg(remap + raw);
                } else {
                    x = p.pad_id;
                    if (i == 0) atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_TOKEN);
                }
            } else {
                x = raw;
            }
        } else if (history != nullptr && -pos <= p.hist_len) {
            x = __ldg(history + static_cast<int64_t>(b) * p.hist_len + p.hist_len + pos);
        } else {
            x = p.pad_id;
        }
        if (i == 0 && xr_out != nullptr) xr_out[n] = x;
        xp1[i] = static_cast<uint64_t>(static_cast<int64_t>(x)) + 1ull;
    }
    uint32_t *row = idx + n * p.H;
    for (int h = 0; h < p.H; ++h) {
        const int o = p.order[h];
        uint64_t s = 0;
#pragma unroll
        for (int i = 0; i < ENGRAM_MAX_ORDERS; ++i)
            if (i < o) s ^= xp1[i] * p.mult[h][i];
        row[h] = static_cast<uint32_t>(fmix64(s) % p.prime[h]);
    }
}

// Plain remap (step 1 on its own).
__global__ void remap_kernel(const int32_t *__restrict__ ids, int64_t n, const int32_t *__restrict__ remap,
                             int32_t vocab_in, int32_t pad_id, int32_t *__restrict__ out) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t x = ids[i];
        int32_t y;
        if (x >= 0 && x < vocab_in) {
            y = __ldg(remap + x);
        } else {
            y = pad_id;
            atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_TOKEN);
        }
        out[i] = y;
    }
}

// history[b] <- last hist_len ids of (history[b] ++ xr[b, :]).  One thread per sequence;
// slots are rewritten in increasing order, each read slot lies at or after its target.
__global__ void advance_history_kernel(const int32_t *__restrict__ xr, int32_t B, int32_t T,
                                       int32_t *history, int32_t hist_len) {
    const int32_t b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    int32_t *hb = history + static_cast<int64_t>(b) * hist_len;
    for (int32_t s = 0; s < hist_len; ++s) {
        const int32_t pos = T - hist_len + s;
        hb[s] = pos >= 0 ? xr[static_cast<int64_t>(b) * T + pos] : hb[hist_len + pos];
    }
}

struct GatherParams {
    const uint16_t *table[ENGRAM_MAX_TABLES];
    uint64_t rows[ENGRAM_MAX_TABLES];
    int32_t H;
    int32_t chunks_per_row;  // d_e / 8  (16-byte chunks)
    int32_t chunks_per_tok;  // H * d_e / 8
    int64_t n_tok;
};

// m[n, h*d_e + c] = table_h[idx[n, h], c], copied as 16-byte chunks.  Consecutive threads
// take consecutive chunks of m, so stores are fully coalesced and each table row is read
// as contiguous 16-byte pieces.  Each thread keeps UNROLL independent chunks in flight.
template <int UNROLL>
__global__ void __launch_bounds__(256) gather_kernel(const uint32_t *__restrict__ idx, uint4 *__restrict__ m,
                                                     const __grid_constant__ GatherParams p) {
    const int64_t total = p.n_tok * p.chunks_per_tok;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < total;
         base += stride * UNROLL) {
        uint32_t row[UNROLL];
        int32_t hh[UNROLL], cc[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t i = base + u * stride;
            row[u] = 0xFFFFFFFFu;
            hh[u] = 0;
            cc[u] = 0;
            if (i < total) {
                const int64_t n = i / p.chunks_per_tok;
                const int32_t r = static_cast<int32_t>(i - n * p.chunks_per_tok);
                const int32_t h = r / p.chunks_per_row;
                hh[u] = h;
                cc[u] = r - h * p.chunks_per_row;
                row[u] = __ldg(idx + n * p.H + h);
            }
        }
        uint4 val[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t i = base + u * stride;
            val[u] = make_uint4(0, 0, 0, 0);
            if (i < total) {
                if (row[u] < p.rows[hh[u]]) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(p.table[hh[u]]) +
                                       static_cast<int64_t>(row[u]) * p.chunks_per_row + cc[u];
                    val[u] = __ldg(src);
                } else {
                    atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_ROW);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t i = base + u * stride;
            if (i < total) m[i] = val[u];
        }
    }
}

}  // namespace engram
