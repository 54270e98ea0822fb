// Steps 1-3 of the lookup: remap + n-gram hashing (one fused kernel), row gather into the
// concatenated memory vector, and the decode-history update.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "engram.h"

#include "ptx.cuh"
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

// The row ids of token n for every table: row[h] = fmix64(XOR_i (x'_{t-i} + 1) * a_{h,i}) mod
// P_h, reading the token and the (max_order - 1) before it (through `remap` when given; the
// history, then the pad id, before the sequence start).  xr_out[n] = x'_t when given.
__device__ __forceinline__ void hash_token(const int32_t *__restrict__ ids, const int32_t *__restrict__ remap,
                                           const int32_t *__restrict__ history, uint32_t *row,
                                           int32_t *__restrict__ xr_out, const HashParams &p, int64_t n) {
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
    for (int h = 0; h < p.H; ++h) {
        const int o = p.order[h];
        uint64_t s = 0;
#pragma unroll
        for (int i = 0; i < ENGRAM_MAX_ORDERS; ++i)
            if (i < o) s ^= xp1[i] * p.mult[h][i];
        row[h] = mod_prime(fmix64(s), p.prime[h], p.barrett[h]);
    }
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
    hash_token(ids, remap, history, idx + n * p.H, xr_out, p, n);
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
    pdl_wait();   // launched early behind the gate kernel: xr and history belong to earlier kernels
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
// product.  decode() is exact in fp16 (cvt.rn.f16x2.e4m3x2) and in fp32.  The product is
// first rounded to odd at fp32 precision: truncated toward zero (mul.rz), with its last bit
// set when the truncation was inexact (fma recovers the exact remainder).  Rounding a
// round-to-odd value with p >= q + 2 bits to q bits is the correctly rounded q-bit result,
// so one hardware RNE conversion to bf16 (24 >= 8 + 2) finishes it.  Scales are limited to
// [2^-100, 2^100] on the host, so every product of a finite code is a normal fp32 value.

// Round-to-odd fp32 pattern of a * s.
__device__ __forceinline__ float product_round_to_odd(float a, float s) {
    const float t = __fmul_rz(a, s);
    const float r = __fmaf_rn(a, s, -t);
    return __uint_as_float(__float_as_uint(t) | (r != 0.0f ? 1u : 0u));
}

// Two e4m3 codes (low byte = first element) -> two dequantised bf16 packed in 32 bits.
__device__ __forceinline__ uint32_t dequant_e4m3x2(uint32_t two_codes, float scale) {
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes), __NV_E4M3);
    const float2 f = __half22float2(__half2(hr));
    const __nv_bfloat162 b =
        __floats2bfloat162_rn(product_round_to_odd(f.x, scale), product_round_to_odd(f.y, scale));
    return *reinterpret_cast<const uint32_t *>(&b);
}

// Eight codes (8 bytes) -> eight bf16 (16 bytes).
__device__ __forceinline__ uint4 dequant_e4m3x8(uint2 w, float scale) {
    return make_uint4(dequant_e4m3x2(w.x & 0xFFFFu, scale), dequant_e4m3x2(w.x >> 16, scale),
                      dequant_e4m3x2(w.y & 0xFFFFu, scale), dequant_e4m3x2(w.y >> 16, scale));
}

// Unsigned 32-bit division by a divisor fixed for a launch (Granlund and Montgomery,
// "Division by Invariant Integers using Multiplication", PLDI 1994, the unsigned method of
// section 4): with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1,
// n / d = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0), where t = mulhi(m, n).
struct FastDivU32 {
    uint32_t d, m, s1, s2;
};

inline FastDivU32 make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while (l < 32 && (1ull << l) < d) ++l;
    FastDivU32 f;
    f.d = d;
    f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - d)) / d + 1);
    f.s1 = l < 1 ? l : 1;
    f.s2 = l > 1 ? l - 1 : 0;
    return f;
}

__device__ __forceinline__ uint32_t fastdiv(uint32_t n, const FastDivU32 &f) {
    const uint32_t t = __umulhi(f.m, n);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

struct GatherParams {
    const void *table[ENGRAM_MAX_TABLES];
    uint64_t rows[ENGRAM_MAX_TABLES];
    float scale[ENGRAM_MAX_TABLES];  // FP8 tables only
    int32_t H;
    int32_t chunks_per_row;  // d_e / 8  (16-byte chunks of m)
    int32_t chunks_per_tok;  // H * d_e / 8
    int64_t n_tok;
    FastDivU32 div_row, div_tok;  // by chunks_per_row, chunks_per_tok (32-bit index launches)
    FastDivU32 div_h;             // by H (row-ordered gather: list item -> table)
};

// The stored bytes behind one 16-byte chunk of m (8 values): 16 bytes of a bf16 row, or 8
// bytes of an e4m3 row.  Loads and conversions are kept apart (all of a thread's loads are
// issued before the first conversion), so that the conversions do not serialise the loads.
template <bool FP8> struct RowChunk { using type = uint4; };
template <> struct RowChunk<true> { using type = uint2; };

template <bool FP8>
__device__ __forceinline__ typename RowChunk<FP8>::type load_row_chunk(const void *table, uint32_t row,
                                                                       int32_t chunks_per_row, int32_t c) {
    const int64_t off = static_cast<int64_t>(row) * chunks_per_row + c;
    return __ldg(reinterpret_cast<const typename RowChunk<FP8>::type *>(table) + off);
}

__device__ __forceinline__ uint4 chunk_to_m(uint4 raw, float) { return raw; }
__device__ __forceinline__ uint4 chunk_to_m(uint2 raw, float scale) { return dequant_e4m3x8(raw, scale); }

template <bool FP8>
__device__ __forceinline__ typename RowChunk<FP8>::type zero_chunk() {
    typename RowChunk<FP8>::type z;
    memset(&z, 0, sizeof z);
    return z;
}

// m[n, h*d_e + c] = table_h[idx[n, h], c], copied as 16-byte chunks of m.  Consecutive
// threads take consecutive chunks of m, so stores are fully coalesced and each table row is
// read as contiguous pieces.  Each thread keeps UNROLL independent chunks in flight.
// Idx = uint32_t when every chunk index of the launch (plus one grid stride) fits in 32 bits:
// the chunk -> (token, table, column) split then runs on multiply-high divisions.
template <int UNROLL, bool FP8, typename Idx>
__global__ void __launch_bounds__(256) gather_kernel(const uint32_t *__restrict__ idx, uint4 *__restrict__ m,
                                                     const __grid_constant__ GatherParams p) {
    pdl_launch_dependents();   // the projection may prefetch its weight tiles while this drains
    const Idx total = static_cast<Idx>(p.n_tok * p.chunks_per_tok);
    const Idx stride = static_cast<Idx>(gridDim.x) * blockDim.x;
    for (Idx base = static_cast<Idx>(blockIdx.x) * blockDim.x + threadIdx.x; base < total; base += stride * UNROLL) {
        uint32_t row[UNROLL];
        int32_t hh[UNROLL], cc[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const Idx i = base + u * stride;
            row[u] = 0xFFFFFFFFu;
            hh[u] = 0;
            cc[u] = 0;
            if (i < total) {
                int64_t n;
                int32_t r, h;
                if constexpr (sizeof(Idx) == 4) {
                    const uint32_t n32 = fastdiv(i, p.div_tok);
                    r = static_cast<int32_t>(i - n32 * p.div_tok.d);
                    h = static_cast<int32_t>(fastdiv(static_cast<uint32_t>(r), p.div_row));
                    n = n32;
                } else {
                    n = i / p.chunks_per_tok;
                    r = static_cast<int32_t>(i - n * p.chunks_per_tok);
                    h = r / p.chunks_per_row;
                }
                hh[u] = h;
                cc[u] = r - h * p.chunks_per_row;
                row[u] = __ldg(idx + n * p.H + h);
            }
        }
        typename RowChunk<FP8>::type val[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const Idx i = base + u * stride;
            val[u] = zero_chunk<FP8>();
            if (i < total) {
                if (row[u] < p.rows[hh[u]]) {
                    val[u] = load_row_chunk<FP8>(p.table[hh[u]], row[u], p.chunks_per_row, cc[u]);
                } else {
                    atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_ROW);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const Idx i = base + u * stride;
            if (i < total) m[i] = chunk_to_m(val[u], p.scale[hh[u]]);
        }
    }
}

// m[n, h*d_e : (h+1)*d_e] = table_h[idx[n, h]] for bf16 rows, as bulk (TMA) copies staged in
// shared memory: list item i = n * H + h is the i-th row-sized piece of m, so a CTA that takes
// the consecutive items [c0, c1) fills one contiguous stretch of m.  One warp per CTA: the lanes
// fetch the row ids 32 at a time, lane 0 issues a bulk load of each row into a ring of S slots
// (bytes counted on the slot's mbarrier) and, L items behind, a bulk store of the landed row
// into m; before a slot is refilled, the store that read it has finished reading (bulk
// async-group wait).  No per-chunk index arithmetic, no register staging: the rows move
// global -> shared -> global in one instruction each.  Rows beyond the table are written as
// zeros and flagged (ENGRAM_STATUS_BAD_ROW); every wait is bounded.
template <int S, int L>
__global__ void __launch_bounds__(32) gather_bulk_kernel(const uint32_t *__restrict__ idx, uint8_t *__restrict__ m,
                                                        const __grid_constant__ GatherParams p, int64_t per_cta) {
    static_assert(L >= 1 && L < S, "lag");
    extern __shared__ __align__(128) uint8_t g_smem[];
    __shared__ uint64_t full[S];
    __shared__ int s_abort;
    pdl_launch_dependents();   // the projection may prefetch its weight tiles while this drains
    const int lane = threadIdx.x;
    const uint32_t rb = static_cast<uint32_t>(p.chunks_per_row) * 16u;   // row bytes
    const int64_t n_items = p.n_tok * p.H;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * per_cta;
    const int64_t c1 = min(n_items, c0 + per_cta);
    if (c0 >= c1) return;
    const int count = static_cast<int>(c1 - c0);
    if (lane == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
    int issued = 0;       // lane 0: items whose slot was filled or armed so far
    uint32_t batch = 0;   // lane l: row id of item c0 + 32 * (k / 32) + l
    for (int k = 0; k < count + L; ++k) {
        if (k < count) {
            if ((k & 31) == 0) {
                const int64_t it = c0 + k + lane;
                batch = it < c1 ? __ldg(idx + it) : 0u;
            }
            const uint32_t row = __shfl_sync(0xffffffffu, batch, k & 31);
            if (lane == 0 && !s_abort) {
                const int s = k % S;
                uint8_t *slot = g_smem + static_cast<int64_t>(s) * rb;
                if (k >= S) bulk_wait_group_read<S - L - 1>();   // the store of item k - S has read the slot
                const uint32_t i = static_cast<uint32_t>(c0 + k);
                const uint32_t h = i - fastdiv(i, p.div_h) * p.div_h.d;
                if (row < p.rows[h]) {
                    mbar_arrive_expect_tx(&full[s], rb);
                    bulk_load_1d(slot, static_cast<const uint8_t *>(p.table[h]) + static_cast<int64_t>(row) * rb, rb,
                                 &full[s]);
                } else {
                    atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_ROW);
                    for (uint32_t o = 0; o < rb; o += 16) *reinterpret_cast<uint4 *>(slot + o) = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                    mbar_arrive(&full[s]);
                }
                issued = k + 1;
            }
        }
        const int j = k - L;
        if (lane == 0 && j >= 0 && j < count && !s_abort) {
            const int s = j % S;
            if (mbar_wait(&full[s], (j / S) & 1, &s_abort)) {
                bulk_store_1d(m + (c0 + j) * rb, g_smem + static_cast<int64_t>(s) * rb, rb);
                bulk_commit_group();
            }
        }
    }
    if (lane == 0) {
        if (s_abort) {   // every issued load lands before the shared memory is released
            volatile int never = 0;
            for (int k = issued > S ? issued - S : 0; k < issued; ++k)
                if (!mbar_wait(&full[k % S], (k / S) & 1, &never)) break;
        }
        bulk_wait_group_all();
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
    pdl_launch_dependents();   // the projection may start streaming its weights now
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
    typename RowChunk<FP8>::type val[kLookupChunksPerWarp / 32];
#pragma unroll
    for (int k = 0; k < kLookupChunksPerWarp / 32; ++k) {
        const int c = part * kLookupChunksPerWarp + k * 32 + lane;
        if (c < c_end) val[k] = load_row_chunk<FP8>(p.table[h], row, p.chunks_per_row, c);
    }
    const float scale = p.scale[h];
#pragma unroll
    for (int k = 0; k < kLookupChunksPerWarp / 32; ++k) {
        const int c = part * kLookupChunksPerWarp + k * 32 + lane;
        if (c < c_end) dst[c] = chunk_to_m(val[k], scale);
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

// Small batches (at most kStageSmallRows (token, table) rows): remap + hash, in-batch dedup
// and the copy of the distinct rows in ONE kernel, so that a decode step's prefetch from host
// memory pays one launch and one dependent chain instead of three.  Every CTA hashes the whole
// batch and dedups it in shared memory itself (a few hundred rows: cheaper than a second
// launch), then copies its share of the distinct rows' 16-byte chunks; CTA 0 alone writes the
// row ids, the slots and the distinct-row lists.  Results are those of hash_kernel,
// stage_dedup_kernel and stage_copy_kernel: the same slots (distinct rows numbered in
// increasing order per table) and the same staged bytes.
constexpr int kStageSmallRows = 256;
constexpr int kStageSmallThreads = 512;   // 16 warps: with 8 CTAs, one warp per distinct row of a 64 x 2 step
constexpr int kStageChunksPerLane = 16;   // loads in flight per lane and row (rows of up to 8 KB in one pass)

__global__ void __launch_bounds__(kStageSmallThreads) stage_small_kernel(
    const int32_t *__restrict__ ids, const int32_t *__restrict__ remap, const int32_t *__restrict__ history,
    uint32_t *__restrict__ idx_out, int32_t *__restrict__ xr_out, uint32_t *__restrict__ staged_idx,
    uint32_t *__restrict__ unique_rows, int32_t *__restrict__ n_unique, const __grid_constant__ HashParams hp,
    const __grid_constant__ StageParams sp) {
    __shared__ uint32_t s_row[kStageSmallRows];    // [n_tok, H] row ids
    __shared__ uint32_t s_slot[kStageSmallRows];   // slot of each (token, table)
    __shared__ uint32_t s_uniq[kStageSmallRows];   // [H][n_tok] distinct rows, increasing
    __shared__ int32_t s_nu[ENGRAM_MAX_TABLES];
    const int H = hp.H;
    const int n_tok = hp.B * hp.T;
    const int rows = n_tok * H;
    const bool writer = blockIdx.x == 0;
    if (threadIdx.x < H) s_nu[threadIdx.x] = 0;
    for (int n = threadIdx.x; n < n_tok; n += blockDim.x)
        hash_token(ids, remap, history, s_row + n * H, writer ? xr_out : nullptr, hp, n);
    __syncthreads();
    // a (token, table) row is a head if no earlier token of the table has the same row id
    // (s_slot holds the flag for now) ...
    for (int e = threadIdx.x; e < rows; e += blockDim.x) {
        const int h = e % H;
        const uint32_t r = s_row[e];
        uint32_t head = 1;
        for (int m = 0; m < e / H; ++m) head &= s_row[m * H + h] != r;
        s_slot[e] = head;
    }
    __syncthreads();
    // ... and its slot is the number of heads of the table with a smaller row id
    uint32_t slot[(kStageSmallRows + kStageSmallThreads - 1) / kStageSmallThreads];
    for (int e = threadIdx.x, k = 0; e < rows; e += blockDim.x, ++k) {
        const int h = e % H;
        const uint32_t r = s_row[e];
        uint32_t below = 0;
        for (int m = 0; m < n_tok; ++m) below += s_slot[m * H + h] & static_cast<uint32_t>(s_row[m * H + h] < r);
        slot[k] = below;
        if (s_slot[e]) {
            s_uniq[h * n_tok + below] = r;
            atomicAdd(&s_nu[h], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x, k = 0; e < rows; e += blockDim.x, ++k) s_slot[e] = slot[k];
    __syncthreads();
    if (writer) {
        for (int e = threadIdx.x; e < rows; e += blockDim.x) {
            idx_out[e] = s_row[e];
            staged_idx[e] = s_slot[e];
        }
        for (int h = 0; h < H; ++h)
            for (int i = threadIdx.x; i < s_nu[h]; i += blockDim.x)
                unique_rows[static_cast<int64_t>(h) * sp.capacity + i] = s_uniq[h * n_tok + i];
        if (threadIdx.x < H) n_unique[threadIdx.x] = s_nu[threadIdx.x];
    }
    // copy the distinct rows (table by table, slot order), one warp per row: lane l takes
    // chunks l, l + 32, ... of its row, all of them in flight at once, so that a row costs one
    // round trip over the host link; 32-bit index arithmetic only
    const int lane = threadIdx.x & 31;
    const int gw = static_cast<int>(blockIdx.x) * (kStageSmallThreads / 32) + static_cast<int>(threadIdx.x >> 5);
    const int nw = static_cast<int>(gridDim.x) * (kStageSmallThreads / 32);
    int n_rows = 0;
    for (int h = 0; h < H; ++h) n_rows += s_nu[h];
    const int cpr = sp.chunks_per_row;
    for (int q = gw; q < n_rows; q += nw) {
        int h = 0, sl = q;
        while (sl >= s_nu[h]) {
            sl -= s_nu[h];
            ++h;
        }
        const uint32_t row = s_uniq[h * n_tok + sl];
        const bool ok = row < sp.rows[h];
        if (!ok && lane == 0) atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_ROW);
        const uint4 *src = reinterpret_cast<const uint4 *>(sp.table[h]) + static_cast<int64_t>(ok ? row : 0u) * cpr;
        uint4 *dst = reinterpret_cast<uint4 *>(sp.staging[h]) + static_cast<int64_t>(sl) * cpr;
        for (int c0 = 0; c0 < cpr; c0 += 32 * kStageChunksPerLane) {
            uint4 val[kStageChunksPerLane];
#pragma unroll
            for (int u = 0; u < kStageChunksPerLane; ++u) {
                const int c = c0 + u * 32 + lane;
                val[u] = (ok && c < cpr) ? src[c] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kStageChunksPerLane; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < cpr) dst[c] = val[u];
            }
        }
    }
}

}  // namespace engram

namespace engram {

// ---------------------------------------------------------------- HBM cache of host-table rows
// A direct-mapped cache per table in device memory sits in front of the host-resident
// tables: slot(row) = row mod slots (row ids are already hash outputs, uniform mod P).
// tags[slot] = row + 1 of the cached row (0 = empty); claim[slot] is per-call scratch that is
// 0xFFFFFFFF between calls.  Per call, over the batch's distinct rows (from stage_dedup_kernel):
//   probe:  hit = (tags[slot] == row + 1).  A hit pins its slot for this call
//           (claim := 0); a miss bids for its slot (claim := min(claim, row + 1)).
//   decide: a miss wins its slot iff claim[slot] == row + 1 (so no slot that is read this call
//           is written this call, and at most one row is written into each slot).
//   copy:   staging <- cache slot (hit) or host row (miss); a winner also writes the cache slot.
//   commit: winners set tags[slot] = row + 1 (after their data is in place); every touched
//           slot's claim goes back to 0xFFFFFFFF.
// Staging always receives the exact row; the cache only decides where the bytes come from.
struct CacheParams {
    void *data[ENGRAM_MAX_TABLES];        // [slots, row bytes]
    uint32_t *tags[ENGRAM_MAX_TABLES];    // [slots]
    uint32_t *claim[ENGRAM_MAX_TABLES];   // [slots]
    uint64_t slot_mask;                   // slots - 1 (slots a power of two)
    uint64_t rows[ENGRAM_MAX_TABLES];     // table sizes: an out-of-range row never enters the cache
    const uint32_t *unique_rows;          // [H, capacity]
    const int32_t *n_unique;              // [H]
    uint32_t *flags;                      // [H, capacity]: 1 = hit, 2 = miss that fills its slot, 0 = other miss
    int32_t *n_hits;                      // [H]
    int32_t H, capacity;
};

__global__ void cache_probe_kernel(const __grid_constant__ CacheParams p) {
    const int h = blockIdx.y;
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= __ldg(p.n_unique + h)) return;
    const uint32_t row = __ldg(p.unique_rows + static_cast<int64_t>(h) * p.capacity + s);
    const uint64_t slot = row & p.slot_mask;
    const bool hit = p.tags[h][slot] == row + 1u;   // only rows inside the table are ever tagged
    if (hit) {
        atomicMin(p.claim[h] + slot, 0u);
        atomicAdd(p.n_hits + h, 1);
    } else if (row < p.rows[h]) {
        atomicMin(p.claim[h] + slot, row + 1u);
    }
    p.flags[static_cast<int64_t>(h) * p.capacity + s] = hit ? 1u : 0u;
}

__global__ void cache_decide_kernel(const __grid_constant__ CacheParams p) {
    const int h = blockIdx.y;
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= __ldg(p.n_unique + h)) return;
    const int64_t i = static_cast<int64_t>(h) * p.capacity + s;
    if (p.flags[i] == 1u) return;
    const uint32_t row = __ldg(p.unique_rows + i);
    if (p.claim[h][row & p.slot_mask] == row + 1u) p.flags[i] = 2u;
}

__global__ void cache_commit_kernel(const __grid_constant__ CacheParams p) {
    const int h = blockIdx.y;
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= __ldg(p.n_unique + h)) return;
    const int64_t i = static_cast<int64_t>(h) * p.capacity + s;
    const uint32_t row = __ldg(p.unique_rows + i);
    const uint64_t slot = row & p.slot_mask;
    if (p.flags[i] == 2u) p.tags[h][slot] = row + 1u;
    p.claim[h][slot] = 0xFFFFFFFFu;
}

// Copy of the distinct rows into staging, from the cache (hits) or the host tables (misses);
// a miss that won its slot also writes the cache.  16-byte chunks, many CTAs wide.
template <int UNROLL>
__global__ void __launch_bounds__(256) cache_copy_kernel(const __grid_constant__ StageParams sp,
                                                         const __grid_constant__ CacheParams p) {
    const int64_t per_table = static_cast<int64_t>(sp.capacity) * sp.chunks_per_row;
    const int64_t total = per_table * sp.H;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < total;
         base += stride * UNROLL) {
        uint4 val[UNROLL];
        int64_t dst[UNROLL], cdst[UNROLL];
        int hh[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t i = base + u * stride;
            dst[u] = -1;
            cdst[u] = -1;
            hh[u] = 0;
            if (i < total) {
                const int h = static_cast<int>(i / per_table);
                const int64_t r = i - h * per_table;
                const int32_t s = static_cast<int32_t>(r / sp.chunks_per_row);
                const int32_t c = static_cast<int32_t>(r - static_cast<int64_t>(s) * sp.chunks_per_row);
                if (s < __ldg(sp.n_unique + h)) {
                    const int64_t k = static_cast<int64_t>(h) * sp.capacity + s;
                    const uint32_t row = __ldg(sp.unique_rows + k);
                    const uint32_t flag = p.flags[k];
                    const uint64_t slot = row & p.slot_mask;
                    hh[u] = h;
                    dst[u] = r;
                    if (flag == 1u) {
                        val[u] = reinterpret_cast<const uint4 *>(p.data[h])[slot * sp.chunks_per_row + c];
                    } else if (row < sp.rows[h]) {
                        val[u] = reinterpret_cast<const uint4 *>(sp.table[h])[static_cast<int64_t>(row) * sp.chunks_per_row + c];
                        if (flag == 2u) cdst[u] = static_cast<int64_t>(slot) * sp.chunks_per_row + c;
                    } else {
                        val[u] = make_uint4(0, 0, 0, 0);
                        atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_ROW);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            if (dst[u] >= 0) reinterpret_cast<uint4 *>(sp.staging[hh[u]])[dst[u]] = val[u];
            if (cdst[u] >= 0) reinterpret_cast<uint4 *>(p.data[hh[u]])[cdst[u]] = val[u];
        }
    }
}

__global__ void cache_reset_kernel(uint32_t *tags, uint32_t *claim, int64_t slots) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < slots;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        tags[i] = 0u;
        claim[i] = 0xFFFFFFFFu;
    }
}

}  // namespace engram
