// Step 3 (the row gather) in row order, for large batches on HBM-resident tables.
//
// A batch reads many rows more than once: frequent n-grams repeat within and across
// sequences (the conditional-memory lookup is a deterministic, O(1) addressing of 2-/3-gram
// keys, so a repeated gram reads the same row).  In token order the repeats of a row are far
// apart in time, and L2 has long evicted the row when it is read again.  Here the batch's
// (token, table) items are first grouped by row: items whose rows fall in the same bucket
// (table h, row >> shift_h, 4096 buckets per table) are listed together, and the gather walks
// the list bucket by bucket.  Every repeat of a row then follows its first read within a few
// dozen items, while the row is still in L2, so DRAM sees each distinct row about once; and
// the table is walked in increasing address order, which keeps the translation of the
// 10^7-row tables' pages local.  The list order within a bucket depends on atomics, but each
// item writes its own token's slice of m, so m is bit-identical to the token-order gather.
//
// Three small kernels build the list (count per bucket, exclusive scan, scatter; the atomics
// are aggregated per warp over the lanes that share a bucket, __match_any_sync), then
// gather_ordered_kernel copies the rows.
#pragma once
#include "kernels_lookup.cuh"

namespace engram {

constexpr int kOrderBucketsLog2 = 12;
constexpr int kOrderBuckets = 1 << kOrderBucketsLog2;   // per table
constexpr int kOrderThreads = 256;
constexpr int kOrderScanThreads = 1024;

struct OrderParams {
    int32_t H;
    int32_t shift[ENGRAM_MAX_TABLES];   // bucket of a row of table h: row >> shift[h]
    int64_t n_items;                    // n_tok * H (< 2^32)
};

// bucket of item i = (token n, table h), i = n * H + h; rows beyond the table (only possible
// for caller-supplied ids) go to the table's last bucket, and the gather flags them
__device__ __forceinline__ uint32_t order_bucket(const OrderParams &p, uint32_t i, uint32_t row) {
    const uint32_t h = i % static_cast<uint32_t>(p.H);
    const uint32_t b = min(row >> p.shift[h], static_cast<uint32_t>(kOrderBuckets - 1));
    return h * kOrderBuckets + b;
}

__global__ void __launch_bounds__(kOrderThreads) order_count_kernel(const uint32_t *__restrict__ idx,
                                                                   uint32_t *__restrict__ counts,
                                                                   const __grid_constant__ OrderParams p) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const bool in = i < p.n_items;
    // every lane takes part in the match; lanes past the end carry a key no bucket has
    const uint32_t key = in ? order_bucket(p, static_cast<uint32_t>(i), __ldg(idx + i)) : 0xFFFFFFFFu;
    const uint32_t same = __match_any_sync(0xFFFFFFFFu, key);
    const int lane = threadIdx.x & 31;
    if (in && lane == __ffs(same) - 1) atomicAdd(counts + key, static_cast<uint32_t>(__popc(same)));
}

// cursor = exclusive scan of n counts (the first list slot of each bucket), in one CTA: each
// thread sums a contiguous run, the run totals are scanned across the block, then each run
// is written out.
__global__ void __launch_bounds__(kOrderScanThreads) order_scan_kernel(const uint32_t *__restrict__ counts,
                                                                      uint32_t *__restrict__ cursor, int32_t n) {
    __shared__ uint32_t s_warp[kOrderScanThreads / 32];
    const int per = (n + kOrderScanThreads - 1) / kOrderScanThreads;
    const int b0 = min(n, static_cast<int>(threadIdx.x) * per);
    const int b1 = min(n, b0 + per);
    uint32_t run = 0;
    for (int j = b0; j < b1; ++j) run += counts[j];
    // inclusive scan of the run totals: within the warp, then across warps
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    uint32_t base = x - run + (warp > 0 ? s_warp[warp - 1] : 0u);
    for (int j = b0; j < b1; ++j) {
        cursor[j] = base;
        base += counts[j];
    }
}

// order[slot] = (item, row), slots of one bucket contiguous, buckets in (table, row) order
__global__ void __launch_bounds__(kOrderThreads) order_scatter_kernel(const uint32_t *__restrict__ idx,
                                                                     uint32_t *__restrict__ cursor,
                                                                     uint2 *__restrict__ order,
                                                                     const __grid_constant__ OrderParams p) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const bool in = i < p.n_items;
    const uint32_t row = in ? __ldg(idx + i) : 0u;
    const uint32_t key = in ? order_bucket(p, static_cast<uint32_t>(i), row) : 0xFFFFFFFFu;
    const uint32_t same = __match_any_sync(0xFFFFFFFFu, key);
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(same) - 1;
    uint32_t base = 0;
    if (in && lane == leader) base = atomicAdd(cursor + key, static_cast<uint32_t>(__popc(same)));
    base = __shfl_sync(0xFFFFFFFFu, base, leader);   // every lane reads its group's leader
    if (in) {
        const uint32_t rank = __popc(same & ((1u << lane) - 1u));
        order[base + rank] = make_uint2(static_cast<uint32_t>(i), row);
    }
}

// m[n, h*d_e + c] = table_h[row, c] for every listed item (n * H + h, row), as 16-byte chunks:
// chunk j of the launch is column chunk j % chunks_per_row of list slot j / chunks_per_row.
// Consecutive threads take consecutive chunks, so each row is read and each slice of m
// written as contiguous pieces; UNROLL independent chunks in flight per thread.
template <int UNROLL, bool FP8>
__global__ void __launch_bounds__(256) gather_ordered_kernel(const uint2 *__restrict__ order, uint4 *__restrict__ m,
                                                             const __grid_constant__ GatherParams p) {
    pdl_launch_dependents();   // the projection may prefetch its weight tiles while this drains
    // 32-bit chunk indices: the host takes this path only when the last index plus one grid
    // stride per unrolled chunk fits
    const uint32_t total = static_cast<uint32_t>(p.n_tok * p.chunks_per_tok);
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t base = blockIdx.x * blockDim.x + threadIdx.x; base < total; base += stride * UNROLL) {
        uint2 ent[UNROLL];
        int32_t cc[UNROLL], hh[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const uint32_t j = base + u * stride;
            ent[u] = make_uint2(0u, 0xFFFFFFFFu);
            cc[u] = 0;
            hh[u] = 0;
            if (j < total) {
                const uint32_t s = fastdiv(j, p.div_row);
                cc[u] = static_cast<int32_t>(j - s * p.div_row.d);
                ent[u] = __ldg(order + s);
                hh[u] = static_cast<int32_t>(ent[u].x - fastdiv(ent[u].x, p.div_h) * p.div_h.d);
            }
        }
        typename RowChunk<FP8>::type val[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const uint32_t j = base + u * stride;
            val[u] = zero_chunk<FP8>();
            if (j < total) {
                if (ent[u].y < p.rows[hh[u]])
                    val[u] = load_row_chunk<FP8>(p.table[hh[u]], ent[u].y, p.chunks_per_row, cc[u]);
                else
                    atomicOr(&g_engram_status, ENGRAM_STATUS_BAD_ROW);
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const uint32_t j = base + u * stride;
            if (j < total)
                m[static_cast<uint64_t>(ent[u].x) * p.chunks_per_row + cc[u]] = chunk_to_m(val[u], p.scale[hh[u]]);
        }
    }
}

}  // namespace engram
