// Steps 1-3 of the lookup: remap + n-gram hashing (one fused kernel), row gather into the
// concatenated memory vector, and the decode-history update.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

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

// ---------------------------------------------------------------- FP8 (e4m3) tables
// A table may hold e4m3 codes with one dequantisation scale per table; the gathered value is
// the bf16 nearest to decode(code) * scale_h (ties to even), rounded once from the exact
// product.  decode() is exact in fp16 (cvt.rn.f16x2.e4m3x2) and in fp32; the fp32 product
// a*s is rounded, but fma(a, s, -a*s) recovers its error exactly, and a double rounding
// (fp32, then bf16) can only go wrong when the fp32 product sits exactly on a bf16 midpoint,
// where the sign of that error decides.

// bf16 pattern of the correctly rounded product a * s (finite a, s; no underflow).
__device__ __forceinline__ uint32_t bf16_of_product(float a, float s) {
    const float hi = __fmul_rn(a, s);
    const float lo = __fmaf_rn(a, s, -hi);
    const uint32_t u = __float_as_uint(hi);
    if ((u & 0xFFFFu) == 0x8000u && lo != 0.0f) return (lo > 0.0f) == (hi > 0.0f) ? (u >> 16) + 1u : (u >> 16);
    if ((u & 0x7F800000u) == 0x7F800000u) return (u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u);  // inf / NaN
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

// Two e4m3 codes (low byte = first element) -> two dequantised bf16 packed in 32 bits.
__device__ __forceinline__ uint32_t dequant_e4m3x2(uint32_t two_codes, float scale) {
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes), __NV_E4M3);
    const float2 f = __half22float2(__half2(hr));
    return bf16_of_product(f.x, scale) | (bf16_of_product(f.y, scale) << 16);
}

// Eight codes (8 bytes) -> eight bf16 (16 bytes).
__device__ __forceinline__ uint4 dequant_e4m3x8(uint2 w, float scale) {
    return make_uint4(dequant_e4m3x2(w.x & 0xFFFFu, scale), dequant_e4m3x2(w.x >> 16, scale),
                      dequant_e4m3x2(w.y & 0xFFFFu, scale), dequant_e4m3x2(w.y >> 16, scale));
}

struct GatherParams {
    const void *table[ENGRAM_MAX_TABLES];
    uint64_t rows[ENGRAM_MAX_TABLES];
    float scale[ENGRAM_MAX_TABLES];  // FP8 tables only
    int32_t H;
    int32_t chunks_per_row;  // d_e / 8  (16-byte chunks of m)
    int32_t chunks_per_tok;  // H * d_e / 8
    int64_t n_tok;
};

// One 16-byte chunk of m (8 values) from chunk c of row `row` of table h: 16 bytes of a bf16
// table, or 8 bytes of an e4m3 table dequantised on the fly.
template <bool FP8>
__device__ __forceinline__ uint4 load_row_chunk(const void *table, float scale, uint32_t row, int32_t chunks_per_row,
                                                int32_t c) {
    const int64_t off = static_cast<int64_t>(row) * chunks_per_row + c;
    if constexpr (FP8) {
        return dequant_e4m3x8(__ldg(reinterpret_cast<const uint2 *>(table) + off), scale);
    } else {
        return __ldg(reinterpret_cast<const uint4 *>(table) + off);
    }
}

// m[n, h*d_e + c] = table_h[idx[n, h], c], copied as 16-byte chunks of m.  Consecutive
// threads take consecutive chunks of m, so stores are fully coalesced and each table row is
// read as contiguous pieces.  Each thread keeps UNROLL independent chunks in flight.
template <int UNROLL, bool FP8>
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
                    val[u] = load_row_chunk<FP8>(p.table[hh[u]], p.scale[hh[u]], row[u], p.chunks_per_row, cc[u]);
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
    const void *table[ENGRAM_MAX_TABLES];
    float scale[ENGRAM_MAX_TABLES];  // FP8 tables only
    int32_t chunks_per_row;  // d_e / 8 (16-byte chunks of m)
    int32_t warps_per_row;   // each warp copies up to kLookupChunksPerWarp chunks of a row
};
constexpr int kLookupChunksPerWarp = 64;

template <bool FP8>
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
    uint4 *dst = m + (n * hp.H + h) * p.chunks_per_row;
    const int c_end = min(p.chunks_per_row, (part + 1) * kLookupChunksPerWarp);
    uint4 val[kLookupChunksPerWarp / 32];
#pragma unroll
    for (int k = 0; k < kLookupChunksPerWarp / 32; ++k) {
        const int c = part * kLookupChunksPerWarp + k * 32 + lane;
        if (c < c_end) val[k] = load_row_chunk<FP8>(p.table[h], p.scale[h], row, p.chunks_per_row, c);
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
    const void *table[ENGRAM_MAX_TABLES];  // host-mapped
    void *staging[ENGRAM_MAX_TABLES];      // device, [capacity, d_e] of the table's element type
    uint64_t rows[ENGRAM_MAX_TABLES];
    const uint32_t *unique_rows;           // [H, capacity]
    const int32_t *n_unique;               // [H]
    int32_t H, capacity, chunks_per_row;   // 16-byte chunks of a stored row (any element type)
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
