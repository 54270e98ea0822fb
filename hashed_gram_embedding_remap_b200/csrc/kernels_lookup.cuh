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
    uint64_t barrett[ENGRAM_MAX_TABLES];                  // floor(2^64 / P_h)
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

// s mod P for a 64-bit s and P < 2^32, exactly, by Barrett reduction: with M = floor(2^64 / P)
// the estimate q = floor(s * M / 2^64) is at most 2 below floor(s / P), so the remainder
// s - q P lies in [0, 3P) and at most two subtractions finish it.
__device__ __forceinline__ uint32_t mod_prime(uint64_t s, uint64_t P, uint64_t M) {
    const uint64_t q = __umul64hi(s, M);
    uint64_t r = s - q * P;
    if (r >= P) r -= P;
    if (r >= P) r -= P;
    return static_cast<uint32_t>(r);
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
        row[h] = mod_prime(fmix64(s), p.prime[h], p.barrett[h]);
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

// Steps 1-3 fused for device-resident tables: one warp per (token, table) row.  Lane 0
// remaps the gram's ids and hashes them (same arithmetic as hash_kernel), the row id is
// broadcast to the warp, and the 32 lanes copy the row into m as 16-byte chunks.  Used by
// engram_forward: the row ids never round-trip through memory (the remapped current id is
// still written for the decode-history update).
struct LookupParams {
    HashParams hash;
    const uint16_t *table[ENGRAM_MAX_TABLES];
    int32_t chunks_per_row;  // d_e / 8
    int32_t warps_per_row;   // each warp copies up to kLookupChunksPerWarp chunks of a row
};
constexpr int kLookupChunksPerWarp = 64;

__global__ void __launch_bounds__(256) lookup_kernel(const int32_t *__restrict__ ids,
                                                     const int32_t *__restrict__ remap,
                                                     const int32_t *__restrict__ history,
                                                     int32_t *__restrict__ xr_out, uint4 *__restrict__ m,
                                                     const __grid_constant__ LookupParams p) {
    const HashParams &hp = p.hash;
    const int64_t n_tok = static_cast<int64_t>(hp.B) * hp.T;
    const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    const int64_t row_id = gw / p.warps_per_row;            // (token, table) row
    const int part = static_cast<int>(gw - row_id * p.warps_per_row);
    const int64_t n = row_id / hp.H;
    if (n >= n_tok) return;
    const int h = static_cast<int>(row_id - n * hp.H);
    uint32_t row = 0;
    if (lane == 0) {
        const int32_t b = static_cast<int32_t>(n / hp.T);
        const int32_t t = static_cast<int32_t>(n - static_cast<int64_t>(b) * hp.T);
        const int o = hp.order[h];
        uint64_t s = 0;
        for (int i = 0; i < o; ++i) {
            const int32_t pos = t - i;
            int32_t x;
            if (pos >= 0) {
                const int32_t raw = __ldg(ids + (n - i));
                if (remap != nullptr) {
                    if (raw >= 0 && raw < hp.vocab_in) {
                        x = __ldg(remap + raw);
                    } else {
                        x = hp.pad_id;
                        if (i == 0) atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_TOKEN);
                    }
                } else {
                    x = raw;
                }
            } else if (history != nullptr && -pos <= hp.hist_len) {
                x = __ldg(history + static_cast<int64_t>(b) * hp.hist_len + hp.hist_len + pos);
            } else {
                x = hp.pad_id;
            }
            if (i == 0 && h == 0 && part == 0 && xr_out != nullptr) xr_out[n] = x;
            s ^= (static_cast<uint64_t>(static_cast<int64_t>(x)) + 1ull) * hp.mult[h][i];
        }
        row = mod_prime(fmix64(s), hp.prime[h], hp.barrett[h]);
    }
    row = __shfl_sync(0xffffffffu, row, 0);
    const uint4 *src = reinterpret_cast<const uint4 *>(p.table[h]) + static_cast<int64_t>(row) * p.chunks_per_row;
    uint4 *dst = m + (n * hp.H + h) * p.chunks_per_row;
    const int c_end = min(p.chunks_per_row, (part + 1) * kLookupChunksPerWarp);
    uint4 val[kLookupChunksPerWarp / 32];
#pragma unroll
    for (int k = 0; k < kLookupChunksPerWarp / 32; ++k) {
        const int c = part * kLookupChunksPerWarp + k * 32 + lane;
        if (c < c_end) val[k] = __ldg(src + c);
    }
#pragma unroll
    for (int k = 0; k < kLookupChunksPerWarp / 32; ++k) {
        const int c = part * kLookupChunksPerWarp + k * 32 + lane;
        if (c < c_end) dst[c] = val[k];
    }
}

// ---------------------------------------------------------------- host-resident tables
// A step's row ids are known before its compute starts, so the rows a batch needs can be
// fetched from host memory ahead of use.  stage_dedup_kernel (one CTA per table) sorts the
// batch's row ids with their positions in shared memory (bitonic), marks the first of each
// run of equal ids, and assigns slots in sorted order: unique[h][s] is the s-th distinct row
// id and staged_idx[n, h] the slot of token n.  stage_copy_kernel then copies only the
// distinct rows from the (pinned, mapped) host tables into device staging, many CTAs wide so
// that enough reads are in flight to fill the host link.
constexpr int kStageMaxTok = 8192;
constexpr int kDedupThreads = 1024;

__global__ void __launch_bounds__(kDedupThreads) stage_dedup_kernel(const uint32_t *__restrict__ idx, int32_t n,
                                                                    int32_t H, int32_t capacity,
                                                                    uint32_t *__restrict__ staged_idx,
                                                                    uint32_t *__restrict__ unique_rows,
                                                                    int32_t *__restrict__ n_unique) {
    extern __shared__ uint32_t s_dd[];
    int N = 1;
    while (N < n) N <<= 1;
    uint32_t *key = s_dd;
    uint32_t *pos = s_dd + N;
    __shared__ int32_t s_count[kDedupThreads / 32];
    const int h = blockIdx.x;
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        key[i] = i < n ? idx[static_cast<int64_t>(i) * H + h] : 0xFFFFFFFFu;
        pos[i] = static_cast<uint32_t>(i);
    }
    __syncthreads();
    // bitonic sort of (key, pos) pairs, ascending; positions break ties (stable order)
    for (int k = 2; k <= N; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < N; i += blockDim.x) {
                const int l = i ^ j;
                if (l > i) {
                    const bool up = (i & k) == 0;
                    const uint64_t a = (static_cast<uint64_t>(key[i]) << 32) | pos[i];
                    const uint64_t b = (static_cast<uint64_t>(key[l]) << 32) | pos[l];
                    if ((a > b) == up) {
                        key[i] = static_cast<uint32_t>(b >> 32);
                        pos[i] = static_cast<uint32_t>(b);
                        key[l] = static_cast<uint32_t>(a >> 32);
                        pos[l] = static_cast<uint32_t>(a);
                    }
                }
            }
            __syncthreads();
        }
    }
    // each thread owns a contiguous segment; count run heads, block-scan the counts
    const int per = (N + blockDim.x - 1) / blockDim.x;
    const int beg = threadIdx.x * per;
    const int end = min(n, beg + per);
    int cnt = 0;
    for (int i = beg; i < end; ++i) cnt += (i == 0 || key[i] != key[i - 1]);
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_count[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < blockDim.x / 32 ? s_count[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        if (lane < blockDim.x / 32) s_count[lane] = wi - w;   // exclusive warp offsets
        if (lane == 31) n_unique[h] = wi;
    }
    __syncthreads();
    int slot = s_count[warp] + incl - cnt;   // exclusive offset of this thread's first head
    for (int i = beg; i < end; ++i) {
        const bool head = (i == 0 || key[i] != key[i - 1]);
        if (head) {
            unique_rows[static_cast<int64_t>(h) * capacity + slot] = key[i];
            ++slot;
        }
        staged_idx[static_cast<int64_t>(pos[i]) * H + h] = static_cast<uint32_t>(slot - 1);
    }
}

struct StageParams {
    const uint16_t *table[ENGRAM_MAX_TABLES];  // host-mapped
    uint16_t *staging[ENGRAM_MAX_TABLES];      // device, [capacity, d_e]
    uint64_t rows[ENGRAM_MAX_TABLES];
    const uint32_t *unique_rows;               // [H, capacity]
    const int32_t *n_unique;                   // [H]
    int32_t H, capacity, chunks_per_row;
};

template <int UNROLL>
__global__ void __launch_bounds__(256) stage_copy_kernel(const __grid_constant__ StageParams p) {
    const int64_t per_table = static_cast<int64_t>(p.capacity) * p.chunks_per_row;
    const int64_t total = per_table * p.H;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < total;
         base += stride * UNROLL) {
        uint4 val[UNROLL];
        int64_t dst[UNROLL];
        int hh[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t i = base + u * stride;
            dst[u] = -1;
            hh[u] = 0;
            if (i < total) {
                const int h = static_cast<int>(i / per_table);
                const int64_t r = i - h * per_table;
                const int32_t s = static_cast<int32_t>(r / p.chunks_per_row);
                const int32_t c = static_cast<int32_t>(r - static_cast<int64_t>(s) * p.chunks_per_row);
                if (s < __ldg(p.n_unique + h)) {
                    const uint32_t row = __ldg(p.unique_rows + static_cast<int64_t>(h) * p.capacity + s);
                    hh[u] = h;
                    dst[u] = r;
                    if (row < p.rows[h]) {
                        val[u] = reinterpret_cast<const uint4 *>(p.table[h])[static_cast<int64_t>(row) * p.chunks_per_row + c];
                    } else {
                        val[u] = make_uint4(0, 0, 0, 0);
                        atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_ROW);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
            if (dst[u] >= 0) reinterpret_cast<uint4 *>(p.staging[hh[u]])[dst[u]] = val[u];
    }
}

}  // namespace engram
