// Host side of the C ABI declared in include/engram.h: validation, derived constants,
// workspace layout, TMA descriptor encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "engram.h"
#include "kernels_gate.cuh"
#include "kernels_lookup.cuh"
#include "kernels_order.cuh"
#include "kernels_proj_pair.cuh"
#include "ptx.cuh"

namespace {

constexpr uint32_t kPlanMagic = 0xE9A7B200u;
thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(ENGRAM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define ENGRAM_CUDA_TRY(expr, what)              \
    do {                                         \
        cudaError_t e_ = (expr);                 \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

// Kernels launched by this library in this process (engram_kernel_launches).
std::atomic<uint64_t> g_kernel_launches{0};

// After a <<<...>>> launch: count it, then check that it was accepted.
#define ENGRAM_LAUNCHED(what)                                                 \
    do {                                                                      \
        g_kernel_launches.fetch_add(1, std::memory_order_relaxed);            \
        ENGRAM_CUDA_TRY(cudaGetLastError(), what);                            \
    } while (0)

// ---------------------------------------------------------------- host-side integer helpers
uint64_t splitmix64_first(uint64_t state) {
    uint64_t z = state + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t mulmod(uint64_t a, uint64_t b, uint64_t m) {
    return static_cast<uint64_t>((static_cast<unsigned __int128>(a) * b) % m);
}

uint64_t powmod(uint64_t a, uint64_t e, uint64_t m) {
    uint64_t r = 1 % m;
    a %= m;
    while (e) {
        if (e & 1) r = mulmod(r, a, m);
        a = mulmod(a, a, m);
        e >>= 1;
    }
    return r;
}

// Deterministic Miller-Rabin for n < 2^32 (witnesses 2, 7, 61).
bool is_prime_u32(uint64_t n) {
    if (n < 2) return false;
    for (uint64_t p : {2ull, 3ull, 5ull, 7ull, 11ull, 13ull, 61ull}) {
        if (n % p == 0) return n == p;
    }
    uint64_t d = n - 1;
    int r = 0;
    while ((d & 1) == 0) {
        d >>= 1;
        ++r;
    }
    for (uint64_t a : {2ull, 7ull, 61ull}) {
        uint64_t x = powmod(a, d, n);
        if (x == 1 || x == n - 1) continue;
        bool comp = true;
        for (int i = 1; i < r; ++i) {
            x = mulmod(x, x, n);
            if (x == n - 1) {
                comp = false;
                break;
            }
        }
        if (comp) return false;
    }
    return true;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_plan(const engram_plan *plan) {
    if (plan == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "plan is NULL");
    if (plan->magic != kPlanMagic) return fail(ENGRAM_ERR_INVALID_ARG, "plan was not initialised by engram_init");
    return ENGRAM_OK;
}

// ---------------------------------------------------------------- workspace layout
constexpr int64_t kFusedLookupMaxRows = 16384;   // (token, table) rows handled by lookup_kernel
constexpr int64_t kRowOrderMinRows = 65536;      // (token, table) rows from which the gather runs in row order
struct Workspace {
    size_t xr, idx, m, v, part, acc, scal;
    size_t staged_idx, unique, n_unique, staging;  // host-resident tables only
    size_t order_count, order_cursor, order;       // row-ordered gather only
    bool staged;                                   // rows go through device staging
    size_t total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Launch with programmatic stream serialization (pdl = true): the kernel may start while the
// previous kernel on the stream finishes (see pdl_wait / pdl_launch_dependents).  Only a
// kernel whose predecessor belongs to the same entry-point call is launched that way: the
// kernels before pdl_wait read inputs (weights, conv state, h) that an earlier call's kernels
// may still be writing if they were let run alongside, so the first kernel of each call
// waits for everything before it.
template <typename... Params, typename... Args>
cudaError_t launch_ex(bool pdl, void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e == cudaSuccess) g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
    return e;
}

template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
    return launch_ex(true, kernel, grid, block, smem, stream, std::forward<Args>(args)...);
}

bool fp8_tables(const engram_plan *plan) { return plan->cfg.table_dtype == ENGRAM_TABLE_FP8_E4M3; }
int table_elem_bytes(const engram_plan *plan) { return fp8_tables(plan) ? 1 : 2; }

// The gather as bulk copies staged in shared memory (ENGRAM_FLAG_BULK_GATHER): bf16 rows of at
// most 8 KB (a ring of 8, or 32 rows under 2 KB, per one-warp CTA: at most 64 KB), list items
// below 2^31.
bool bulk_gather(const engram_plan *plan, int64_t n_tok) {
    const int64_t row_bytes = static_cast<int64_t>(plan->cfg.row_dim) * 2;
    return (plan->cfg.flags & ENGRAM_FLAG_BULK_GATHER) && !fp8_tables(plan) &&
           n_tok * plan->num_tables < (int64_t(1) << 31) && row_bytes * (row_bytes >= 2048 ? 8 : 32) <= 64 * 1024;
}

// Width of the projection's N tile: the widest of 256/128/64 that divides d_h and still
// gives at least two waves of CTAs on the GPU.  ENGRAM_PROJ_TILE_N (64, 128 or 256) forces a
// width (for tuning and tests); it is read once per process.
int choose_bn(int d_h, int64_t n_tok, int M) {
    static const int forced = [] {
        const char *e = std::getenv("ENGRAM_PROJ_TILE_N");
        const int v = e ? std::atoi(e) : 0;
        return (v == 64 || v == 128 || v == 256) ? v : 0;
    }();
    if (forced && d_h % forced == 0) return forced;
    const int64_t m_tiles = (n_tok + engram::kBM - 1) / engram::kBM;
    const int cands[3] = {256, 128, 64};
    for (int bn : cands) {
        if (d_h % bn != 0) continue;
        if (bn == 64 || m_tiles * ((M + 1) * d_h / bn) >= 2 * 148) return bn;
    }
    return 64;
}

// Work decomposition of the projection for n_tok tokens.  When even the widest tile leaves
// most SMs idle (decode-sized batches), K is split so that every SM streams its own slice of
// the weights; the split-K partial accumulators are finished by splitk_reduce_kernel.
struct ProjShape {
    int bn, n_tiles, k_blocks, k_splits, kb_per_split;
    bool pair;   // CTA pairs (proj_pair_kernel): 256-token x 256-channel units
};

ProjShape proj_shape(const engram_plan *plan, int64_t n_tok, bool allow_split) {
    ProjShape ps{};
    const int d_h = plan->cfg.hidden_dim;
    ps.k_blocks = (plan->mem_dim + engram::kBK - 1) / engram::kBK;
    ps.k_splits = 1;
    ps.kb_per_split = ps.k_blocks;
    const int64_t m_tiles = (n_tok + engram::kBM - 1) / engram::kBM;
    const int sms = 148;
    int wide = 64;
    for (int bn : {256, 128}) {
        if (d_h % bn == 0) {
            wide = bn;
            break;
        }
    }
    const int M = plan->num_branches;
    const int64_t mn = m_tiles * ((M + 1) * d_h / wide);
    // ENGRAM_PROJ_SPLITS (>= 1) forces the split count of decode-sized batches (tuning);
    // read once per process.
    static const int forced_splits = [] {
        const char *e = std::getenv("ENGRAM_PROJ_SPLITS");
        const int v = e ? std::atoi(e) : 0;
        return v > 0 ? v : 0;
    }();
    int splits = 1;
    if (allow_split && mn > 0 && mn < sms) {
        splits = forced_splits ? forced_splits : static_cast<int>(sms / mn);
        if (splits > ps.k_blocks / 4) splits = ps.k_blocks / 4;
        if (splits < 1) splits = 1;
    }
    if (splits > 1) {
        ps.bn = wide;
        ps.kb_per_split = (ps.k_blocks + splits - 1) / splits;
        ps.k_splits = (ps.k_blocks + ps.kb_per_split - 1) / ps.kb_per_split;
    } else {
        ps.bn = choose_bn(d_h, n_tok, M);
    }
    // CTA pairs for d_h % 256 == 0: whole-K units when there are at least two waves of them;
    // K split across pairs when even one wave of units would leave pairs idle (decode-sized
    // batches), like the single-CTA split above but with each weight tile read by one pair
    if (d_h % engram::kPairBN == 0 && !(plan->cfg.flags & ENGRAM_FLAG_SINGLE_CTA_MMA)) {
        const int64_t mn2 = (n_tok + engram::kPairRows - 1) / engram::kPairRows * ((M + 1) * d_h / engram::kPairBN);
        int sp = 0;
        if (mn2 >= sms) {
            sp = 1;
        } else if (allow_split && mn2 > 0 && mn2 < sms / 2) {
            sp = forced_splits ? forced_splits : static_cast<int>((sms / 2) / mn2);
            if (sp > ps.k_blocks / 4) sp = ps.k_blocks / 4;
            if (sp < 2) sp = 0;
        }
        if (sp > 0) {
            ps.pair = true;
            ps.bn = engram::kPairBN;
            ps.kb_per_split = (ps.k_blocks + sp - 1) / sp;
            ps.k_splits = (ps.k_blocks + ps.kb_per_split - 1) / ps.kb_per_split;
        }
    }
    ps.n_tiles = (M + 1) * d_h / ps.bn;
    return ps;
}

// Which kernels engram_forward runs for a batch of n_tok tokens (engram_forward_path).
struct ForwardPath {
    bool fused_lookup;    // remap + hash + gather in one kernel (decode-sized, HBM tables)
    bool staged;          // host-mapped tables: the batch's distinct rows are staged into HBM
    bool pair;            // the projection's MMAs span CTA pairs
    bool row_order;       // the gather walks the rows grouped by row id (kernels_order.cuh)
    ProjShape ps;
};

ForwardPath forward_path(const engram_plan *plan, int64_t n_tok) {
    ForwardPath f{};
    f.ps = proj_shape(plan, n_tok, true);
    f.staged = plan->cfg.table_location == ENGRAM_TABLES_HOST_MAPPED && n_tok <= engram::kStageMaxTok;
    f.fused_lookup = !f.staged && plan->cfg.table_location == ENGRAM_TABLES_DEVICE &&
                     n_tok * plan->num_tables <= kFusedLookupMaxRows;
    f.pair = f.ps.pair;
    // row order (opt-in): HBM tables through the hash + gather path, enough rows for the list to pay,
    // and 32-bit list items and chunk indices (with slack for the grid stride)
    const int64_t rows = n_tok * plan->num_tables;
    f.row_order = !f.staged && !f.fused_lookup && plan->cfg.table_location == ENGRAM_TABLES_DEVICE &&
                  (plan->cfg.flags & ENGRAM_FLAG_ROW_ORDER_GATHER) && rows >= kRowOrderMinRows &&
                  rows * (plan->cfg.row_dim / 8) < (int64_t(1) << 31);
    return f;
}

Workspace layout(const engram_plan *plan, int64_t n_tok) {
    Workspace w{};
    const int H = plan->num_tables;
    const int d_h = plan->cfg.hidden_dim;
    const ProjShape ps = proj_shape(plan, n_tok, true);
    const int n_tiles = ps.n_tiles;
    size_t off = 0;
    w.xr = off;   off = align256(off + sizeof(int32_t) * n_tok);
    w.idx = off;  off = align256(off + sizeof(uint32_t) * n_tok * H);
    w.m = off;    off = align256(off + sizeof(uint16_t) * n_tok * plan->mem_dim);
    const size_t v_bytes = sizeof(uint16_t) * n_tok * d_h;
    w.v = off;    off = align256(off + v_bytes);
    w.part = off; off = align256(off + sizeof(float4) * n_tok * n_tiles);
    w.acc = off;
    if (ps.k_splits > 1) off = align256(off + sizeof(float) * ps.k_splits * n_tok * ps.n_tiles * ps.bn);
    w.scal = off; off = align256(off + sizeof(float2) * n_tok * plan->num_branches);
    const ForwardPath fp = forward_path(plan, n_tok);
    w.staged = fp.staged;
    if (fp.row_order) {
        w.order_count = off;  off = align256(off + sizeof(uint32_t) * H * engram::kOrderBuckets);
        w.order_cursor = off; off = align256(off + sizeof(uint32_t) * H * engram::kOrderBuckets);
        w.order = off;        off = align256(off + sizeof(uint2) * n_tok * H);
    }
    if (w.staged) {
        w.staged_idx = off; off = align256(off + sizeof(uint32_t) * n_tok * H);
        w.unique = off;     off = align256(off + sizeof(uint32_t) * n_tok * H);
        w.n_unique = off;   off = align256(off + sizeof(int32_t) * H);
        w.staging = off;    off = align256(off + static_cast<size_t>(table_elem_bytes(plan)) * n_tok * H * plan->cfg.row_dim);
    }
    w.total = off;
    return w;
}

// ---------------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Row-major bf16 [rows, cols] -> tensor map with a box of box_rows x 64 columns (128 B),
// 128-byte swizzle, zero fill outside the tensor.
int make_map_bf16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto enc = get_encode_fn();
    if (enc == nullptr) return fail(ENGRAM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(engram::kBK), box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ENGRAM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return ENGRAM_OK;
}

int sm_count() {
    static int count[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 64 && count[dev]) return count[dev];
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (dev < 64) count[dev] = n;
    return n;
}

template <int BN, bool SPLIT>
int set_proj_smem_attr() {
    // Per device: the attribute is a property of the function on the current device.
    static bool done[64] = {};
    int dev = 0;
    ENGRAM_CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 64 && done[dev]) return ENGRAM_OK;
    ENGRAM_CUDA_TRY(cudaFuncSetAttribute(engram::proj_kernel<BN, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         engram::ProjCfg<BN>::kSmemBytes),
                    "cudaFuncSetAttribute(proj_kernel)");
    if (dev < 64) done[dev] = true;
    return ENGRAM_OK;
}

// Test hooks of the projection: a shorter bound on every pipeline wait, and a stalled
// pipeline (no loads issued) that makes the first wait run out.
struct ProjTest {
    uint64_t wait_limit_ns = 0;
    int stall = 0;
};

template <int BN>
int launch_proj(const engram_plan *plan, const engram_weights *w, const uint16_t *h, const uint16_t *m,
                int64_t n_tok, uint16_t *v, float4 *part, cudaStream_t stream, float *acc = nullptr,
                int k_splits = 1, int kb_per_split = 0, bool run_reduce = true,
                engram::ProjParams *params_out = nullptr, const ProjTest &test = ProjTest(), bool pdl = true) {
    const int d_m = plan->mem_dim, d_h = plan->cfg.hidden_dim;
    CUtensorMap map_m, map_wk, map_wv;
    int rc;
    const int M = plan->num_branches;
    if ((rc = make_map_bf16(&map_wk, w->w_k, static_cast<uint64_t>(M) * d_h, d_m, BN)) != ENGRAM_OK) return rc;
    if ((rc = make_map_bf16(&map_wv, w->w_v, d_h, d_m, BN)) != ENGRAM_OK) return rc;
    if ((rc = make_map_bf16(&map_m, m, static_cast<uint64_t>(n_tok), d_m, engram::kBM)) != ENGRAM_OK) return rc;
    const bool split = acc != nullptr && k_splits > 1;
    if ((rc = split ? set_proj_smem_attr<BN, true>() : set_proj_smem_attr<BN, false>()) != ENGRAM_OK) return rc;
    engram::ProjParams p{};
    p.h = h;
    p.gamma_q = w->gamma_q;
    p.gamma_k = w->gamma_k;
    p.v = v;
    p.part = part;
    p.n_tok = n_tok;
    p.d_m = d_m;
    p.d_h = d_h;
    p.n_tiles = (M + 1) * d_h / BN;
    p.M = M;
    p.k_blocks = (d_m + engram::kBK - 1) / engram::kBK;
    p.m_tiles = static_cast<int32_t>((n_tok + engram::kBM - 1) / engram::kBM);
    p.k_splits = (acc != nullptr && k_splits > 1) ? k_splits : 1;
    p.kb_per_split = p.k_splits > 1 ? kb_per_split : p.k_blocks;
    p.acc_out = p.k_splits > 1 ? acc : nullptr;
    p.w_packed = BN == 256 ? static_cast<const uint8_t *>(w->w_packed) : nullptr;
    p.wait_limit_ns = test.wait_limit_ns;
    p.stall = test.stall;
    const int64_t total = static_cast<int64_t>(p.m_tiles) * p.n_tiles * p.k_splits;
    if (total > 0x7FFFFFFF) return fail(ENGRAM_ERR_UNSUPPORTED, "too many projection tiles");
    const int64_t sms = sm_count();
    dim3 grid(static_cast<unsigned>(total < sms ? total : sms));
    ENGRAM_CUDA_TRY(launch_ex(pdl, split ? engram::proj_kernel<BN, true> : engram::proj_kernel<BN, false>, grid,
                               dim3(engram::kProjThreads), engram::ProjCfg<BN>::kSmemBytes, stream, map_m, map_wk,
                               map_wv, p),
                    "proj_kernel launch");
    if (params_out) *params_out = p;
    if (p.k_splits > 1 && run_reduce) {
        engram::splitk_reduce_kernel<<<dim3(p.n_tiles, static_cast<unsigned>(n_tok)), engram::kReduceThreads, 0,
                                       stream>>>(p, BN);
        ENGRAM_LAUNCHED("splitk_reduce_kernel launch");
    }
    return ENGRAM_OK;
}

template <bool SPLIT>
int set_pair_smem_attr() {
    static bool done[64] = {};
    int dev = 0;
    ENGRAM_CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 64 && done[dev]) return ENGRAM_OK;
    ENGRAM_CUDA_TRY(cudaFuncSetAttribute(engram::proj_pair_kernel<SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         engram::PairCfg::kSmemBytes),
                    "cudaFuncSetAttribute(proj_pair_kernel)");
    if (dev < 64) done[dev] = true;
    return ENGRAM_OK;
}

// CTA pairs that can be resident at once (one CTA per SM; a pair needs two SMs of one GPC).
template <bool SPLIT>
int max_pairs(int *out) {
    static int cached[64] = {};
    int dev = 0;
    ENGRAM_CUDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 64 && cached[dev]) {
        *out = cached[dev];
        return ENGRAM_OK;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(engram::kProjThreads);
    cfg.dynamicSmemBytes = engram::PairCfg::kSmemBytes;
    int n = 0;
    ENGRAM_CUDA_TRY(cudaOccupancyMaxActiveClusters(&n, engram::proj_pair_kernel<SPLIT>, &cfg),
                    "cudaOccupancyMaxActiveClusters(proj_pair_kernel)");
    if (n < 1) return fail(ENGRAM_ERR_CUDA, "no CTA pair of the projection fits on this device");
    if (dev < 64) cached[dev] = n;
    *out = n;
    return ENGRAM_OK;
}

// Projection on CTA pairs: 256-token x 256-channel units (see kernels_proj_pair.cuh); with
// k_splits > 1, K-split units writing raw partial accumulators to acc (finished like the
// single-CTA split).
int launch_proj_pair(const engram_plan *plan, const engram_weights *w, const uint16_t *h, const uint16_t *m,
                     int64_t n_tok, uint16_t *v, float4 *part, cudaStream_t stream, float *acc, int k_splits,
                     int kb_per_split, bool run_reduce, engram::ProjParams *params_out, bool pdl) {
    const int d_m = plan->mem_dim, d_h = plan->cfg.hidden_dim, M = plan->num_branches;
    constexpr int BN = engram::kPairBN;
    CUtensorMap map_m, map_wk, map_wv;
    int rc;
    if (w->w_packed != nullptr) {
        // the packed tiles as rows of 64 columns, already in the tensor cores' layout: boxes of
        // 128 rows copied as they are (no swizzle)
        auto enc = get_encode_fn();
        if (enc == nullptr) return fail(ENGRAM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
        const uint64_t k_blocks = (d_m + engram::kBK - 1) / engram::kBK;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(engram::kBK),
                              static_cast<cuuint64_t>((M + 1) * d_h / BN) * k_blocks * BN};
        cuuint64_t strides[1] = {engram::kBK * 2};
        cuuint32_t box[2] = {static_cast<cuuint32_t>(engram::kBK), BN / 2};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = enc(&map_wk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(w->w_packed), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(ENGRAM_ERR_CUDA, "cuTensorMapEncodeTiled(packed weights) failed (%d)", static_cast<int>(r));
        map_wv = map_wk;
    } else {
        if ((rc = make_map_bf16(&map_wk, w->w_k, static_cast<uint64_t>(M) * d_h, d_m, BN / 2)) != ENGRAM_OK) return rc;
        if ((rc = make_map_bf16(&map_wv, w->w_v, d_h, d_m, BN / 2)) != ENGRAM_OK) return rc;
    }
    if ((rc = make_map_bf16(&map_m, m, static_cast<uint64_t>(n_tok), d_m, engram::kBM)) != ENGRAM_OK) return rc;
    const bool split = acc != nullptr && k_splits > 1;
    if ((rc = split ? set_pair_smem_attr<true>() : set_pair_smem_attr<false>()) != ENGRAM_OK) return rc;
    int pairs = 0;
    if ((rc = split ? max_pairs<true>(&pairs) : max_pairs<false>(&pairs)) != ENGRAM_OK) return rc;
    engram::ProjParams p{};
    p.h = h;
    p.gamma_q = w->gamma_q;
    p.gamma_k = w->gamma_k;
    p.v = v;
    p.part = part;
    p.n_tok = n_tok;
    p.d_m = d_m;
    p.d_h = d_h;
    p.n_tiles = (M + 1) * d_h / BN;
    p.M = M;
    p.k_blocks = (d_m + engram::kBK - 1) / engram::kBK;
    p.m_tiles = static_cast<int32_t>((n_tok + engram::kPairRows - 1) / engram::kPairRows);
    p.k_splits = split ? k_splits : 1;
    p.kb_per_split = split ? kb_per_split : p.k_blocks;
    p.acc_out = split ? acc : nullptr;
    p.w_packed = static_cast<const uint8_t *>(w->w_packed);
    const int64_t total = static_cast<int64_t>(p.m_tiles) * p.n_tiles * p.k_splits;
    if (total > 0x7FFFFFFF) return fail(ENGRAM_ERR_UNSUPPORTED, "too many projection tiles");
    // ENGRAM_PROJ_PAIRS (>= 1) caps the number of CTA pairs (tuning); read once per process.
    static const int forced_pairs = [] {
        const char *e = std::getenv("ENGRAM_PROJ_PAIRS");
        const int v = e ? std::atoi(e) : 0;
        return v > 0 ? v : 0;
    }();
    if (forced_pairs && forced_pairs < pairs) pairs = forced_pairs;
    const int64_t npairs = total < pairs ? total : pairs;
    ENGRAM_CUDA_TRY(launch_ex(pdl, split ? engram::proj_pair_kernel<true> : engram::proj_pair_kernel<false>,
                               dim3(static_cast<unsigned>(2 * npairs)), dim3(engram::kProjThreads),
                               engram::PairCfg::kSmemBytes, stream, map_m, map_wk, map_wv, p),
                    "proj_pair_kernel launch");
    if (params_out) *params_out = p;
    if (split && run_reduce) {
        engram::splitk_reduce_kernel<<<dim3(p.n_tiles, static_cast<unsigned>(n_tok)), engram::kReduceThreads, 0,
                                       stream>>>(p, BN);
        ENGRAM_LAUNCHED("splitk_reduce_kernel launch");
    }
    return ENGRAM_OK;
}

int validate_weights(const engram_plan *plan, const engram_weights *w) {
    if (w == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "weights is NULL");
    const void *ptrs[6] = {w->w_k, w->w_v, w->gamma_q, w->gamma_k, w->gamma_c, w->conv_w};
    const char *names[6] = {"w_k", "w_v", "gamma_q", "gamma_k", "gamma_c", "conv_w"};
    for (int i = 0; i < 6; ++i) {
        if (ptrs[i] == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "weights.%s is NULL", names[i]);
        if (!aligned16(ptrs[i])) return fail(ENGRAM_ERR_INVALID_ARG, "weights.%s is not 16-byte aligned", names[i]);
    }
    if (w->w_packed != nullptr) {
        if (plan->cfg.hidden_dim % 256 != 0)
            return fail(ENGRAM_ERR_INVALID_ARG, "weights.w_packed given but hidden_dim %% 256 != 0 (no packed form)");
        if (!aligned16(w->w_packed)) return fail(ENGRAM_ERR_INVALID_ARG, "weights.w_packed is not 16-byte aligned");
    }
    return ENGRAM_OK;
}

size_t packed_weights_bytes(const engram_plan *plan) {
    const int d_h = plan->cfg.hidden_dim;
    if (d_h % 256 != 0) return 0;
    const int64_t k_blocks = (plan->mem_dim + engram::kBK - 1) / engram::kBK;
    const int64_t rows = static_cast<int64_t>(plan->num_branches + 1) * d_h;
    return static_cast<size_t>(rows / 256 * k_blocks) * 32768u;
}

engram::HashParams make_hash_params(const engram_plan *plan, int32_t B, int32_t T) {
    engram::HashParams p{};
    const engram_config &c = plan->cfg;
    const int K = c.heads_per_order;
    for (int oi = 0; oi < c.num_orders; ++oi)
        for (int j = 0; j < K; ++j) {
            const int h = oi * K + j;
            p.order[h] = c.orders[oi];
            p.prime[h] = static_cast<uint64_t>(c.table_rows[h]);
            p.barrett[h] = static_cast<uint64_t>((static_cast<unsigned __int128>(1) << 64) / p.prime[h]);
            for (int i = 0; i < ENGRAM_MAX_ORDERS; ++i) p.mult[h][i] = plan->mult[h][i];
        }
    p.H = plan->num_tables;
    p.max_order = c.orders[c.num_orders - 1];
    p.hist_len = plan->hist_len;
    p.pad_id = c.pad_id;
    p.vocab_in = c.vocab_in;
    p.B = B;
    p.T = T;
    return p;
}

// Fused remap + hash + gather, one warp per (token, table) row.
int launch_lookup(const engram_plan *plan, const int32_t *ids, const int32_t *remap, const int32_t *history,
                  int32_t B, int32_t T, const void *const *tables, int32_t *xr_out, uint16_t *m,
                  cudaStream_t stream) {
    engram::LookupParams p{};
    p.hash = make_hash_params(plan, B, T);
    for (int h = 0; h < plan->num_tables; ++h) {
        p.table[h] = tables[h];
        p.scale[h] = plan->cfg.table_scale[h];
    }
    p.chunks_per_row = plan->cfg.row_dim / 8;
    p.warps_per_row = (p.chunks_per_row + engram::kLookupChunksPerWarp - 1) / engram::kLookupChunksPerWarp;
    const int64_t warps = static_cast<int64_t>(B) * T * plan->num_tables * p.warps_per_row;
    const int threads = 256;
    const int64_t blocks = (warps * 32 + threads - 1) / threads;
    auto kern = fp8_tables(plan) ? engram::lookup_kernel<true> : engram::lookup_kernel<false>;
    kern<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(ids, remap, history, xr_out,
                                                                reinterpret_cast<uint4 *>(m), p);
    ENGRAM_LAUNCHED("lookup_kernel launch");
    return ENGRAM_OK;
}

int launch_hash(const engram_plan *plan, const int32_t *ids, const int32_t *remap, const int32_t *history,
                int32_t B, int32_t T, uint32_t *idx, int32_t *xr_out, cudaStream_t stream) {
    const engram::HashParams p = make_hash_params(plan, B, T);
    const int64_t n_tok = static_cast<int64_t>(B) * T;
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((n_tok + threads - 1) / threads);
    engram::hash_kernel<<<blocks, threads, 0, stream>>>(ids, remap, history, idx, xr_out, p);
    ENGRAM_LAUNCHED("hash_kernel launch");
    return ENGRAM_OK;
}


// rows_override > 0 bounds every table at that many rows (device staging buffers).
int launch_gather(const engram_plan *plan, const uint32_t *idx, const void *const *tables, int64_t n_tok,
                  uint16_t *m, cudaStream_t stream, int64_t rows_override = 0) {
    engram::GatherParams p{};
    const int H = plan->num_tables;
    for (int h = 0; h < H; ++h) {
        p.table[h] = tables[h];
        p.scale[h] = plan->cfg.table_scale[h];
        p.rows[h] = static_cast<uint64_t>(rows_override > 0 ? rows_override : plan->cfg.table_rows[h]);
    }
    p.H = H;
    p.chunks_per_row = plan->cfg.row_dim / 8;
    p.chunks_per_tok = H * p.chunks_per_row;
    p.n_tok = n_tok;
    const int64_t total = n_tok * p.chunks_per_tok;
    p.div_h = engram::make_fastdiv(static_cast<uint32_t>(H));
    // ENGRAM_FLAG_BULK_GATHER (bf16 rows): bulk copies staged in shared memory
    // (gather_bulk_kernel); otherwise, and for FP8 rows (dequantised on the way), the register
    // gather below
    if (bulk_gather(plan, n_tok)) {
        const int64_t row_bytes = static_cast<int64_t>(p.chunks_per_row) * 16;
        const int64_t items = n_tok * H;
        const bool wide = row_bytes >= 2048;
        using BK = void (*)(const uint32_t *, uint8_t *, const engram::GatherParams, int64_t);
        const BK kern = wide ? engram::gather_bulk_kernel<8, 4> : engram::gather_bulk_kernel<32, 16>;
        const int slots = wide ? 8 : 32;
        const size_t smem = static_cast<size_t>(slots) * row_bytes;
        ENGRAM_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)),
                        "cudaFuncSetAttribute(gather_bulk_kernel)");
        int per_sm = 0;
        ENGRAM_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32, smem),
                        "cudaOccupancyMaxActiveBlocksPerMultiprocessor(gather_bulk_kernel)");
        if (per_sm < 1) per_sm = 1;
        int64_t grid = static_cast<int64_t>(sm_count()) * per_sm;
        if (grid > items) grid = items;
        const int64_t per_cta = (items + grid - 1) / grid;
        grid = (items + per_cta - 1) / per_cta;
        kern<<<static_cast<unsigned>(grid), 32, smem, stream>>>(idx, reinterpret_cast<uint8_t *>(m), p, per_cta);
        ENGRAM_LAUNCHED("gather_bulk_kernel launch");
        return ENGRAM_OK;
    }
    // independent chunks per thread: ENGRAM_GATHER_UNROLL (4 or 8) overrides, for tuning
    static const int forced_unroll = [] {
        const char *e = std::getenv("ENGRAM_GATHER_UNROLL");
        const int v = e ? std::atoi(e) : 0;
        return (v == 4 || v == 8) ? v : 0;
    }();
    const int unroll = forced_unroll ? forced_unroll : 4;
    const int threads = 256;
    int64_t blocks = (total + threads * unroll - 1) / (threads * unroll);
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;  // 8 x 256 threads resident per SM
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    p.div_row = engram::make_fastdiv(static_cast<uint32_t>(p.chunks_per_row));
    p.div_tok = engram::make_fastdiv(static_cast<uint32_t>(p.chunks_per_tok));
    const bool f8 = fp8_tables(plan);
    // 32-bit chunk indices when the last index plus one grid stride per unrolled chunk fits
    const bool idx32 = total + blocks * threads * (unroll + 1) < (int64_t(1) << 32);
    using K = void (*)(const uint32_t *, uint4 *, const engram::GatherParams);
    K kern;
    if (idx32)
        kern = unroll == 8 ? (f8 ? engram::gather_kernel<8, true, uint32_t> : engram::gather_kernel<8, false, uint32_t>)
                           : (f8 ? engram::gather_kernel<4, true, uint32_t> : engram::gather_kernel<4, false, uint32_t>);
    else
        kern = unroll == 8 ? (f8 ? engram::gather_kernel<8, true, int64_t> : engram::gather_kernel<8, false, int64_t>)
                           : (f8 ? engram::gather_kernel<4, true, int64_t> : engram::gather_kernel<4, false, int64_t>);
    kern<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(idx, reinterpret_cast<uint4 *>(m), p);
    ENGRAM_LAUNCHED("gather_kernel launch");
    return ENGRAM_OK;
}

// The gather in row order (kernels_order.cuh): count the batch's (token, table) rows per
// bucket, scan the counts, list the rows bucket by bucket, then copy them.  count / cursor:
// H * kOrderBuckets words each; order: n_tok * H entries.  HBM-resident tables only.
int launch_gather_ordered(const engram_plan *plan, const uint32_t *idx, const void *const *tables, int64_t n_tok,
                          uint16_t *m, uint32_t *count, uint32_t *cursor, uint2 *order, cudaStream_t stream) {
    const int H = plan->num_tables;
    const int64_t items = n_tok * H;
    engram::OrderParams op{};
    op.H = H;
    op.n_items = items;
    for (int h = 0; h < H; ++h) {
        // bucket = row >> shift: the table's rows spread over at most kOrderBuckets buckets
        int bits = 0;
        while (bits < 32 && (uint64_t(1) << bits) < static_cast<uint64_t>(plan->cfg.table_rows[h])) ++bits;
        op.shift[h] = bits > engram::kOrderBucketsLog2 ? bits - engram::kOrderBucketsLog2 : 0;
    }
    const int nb = H * engram::kOrderBuckets;
    ENGRAM_CUDA_TRY(cudaMemsetAsync(count, 0, sizeof(uint32_t) * nb, stream), "cudaMemsetAsync(order counts)");
    const unsigned blocks = static_cast<unsigned>((items + engram::kOrderThreads - 1) / engram::kOrderThreads);
    engram::order_count_kernel<<<blocks, engram::kOrderThreads, 0, stream>>>(idx, count, op);
    ENGRAM_LAUNCHED("order_count_kernel launch");
    engram::order_scan_kernel<<<1, engram::kOrderScanThreads, 0, stream>>>(count, cursor, nb);
    ENGRAM_LAUNCHED("order_scan_kernel launch");
    engram::order_scatter_kernel<<<blocks, engram::kOrderThreads, 0, stream>>>(idx, cursor, order, op);
    ENGRAM_LAUNCHED("order_scatter_kernel launch");

    engram::GatherParams p{};
    for (int h = 0; h < H; ++h) {
        p.table[h] = tables[h];
        p.scale[h] = plan->cfg.table_scale[h];
        p.rows[h] = static_cast<uint64_t>(plan->cfg.table_rows[h]);
    }
    p.H = H;
    p.chunks_per_row = plan->cfg.row_dim / 8;
    p.chunks_per_tok = H * p.chunks_per_row;
    p.n_tok = n_tok;
    p.div_row = engram::make_fastdiv(static_cast<uint32_t>(p.chunks_per_row));
    p.div_h = engram::make_fastdiv(static_cast<uint32_t>(H));
    const int64_t total = n_tok * p.chunks_per_tok;   // < 2^31 (forward_path)
    constexpr int unroll = 4;
    const int threads = 256;
    int64_t gblocks = (total + threads * unroll - 1) / (threads * unroll);
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;  // 8 x 256 threads resident per SM
    if (gblocks > cap) gblocks = cap;
    if (gblocks < 1) gblocks = 1;
    auto kern = fp8_tables(plan) ? engram::gather_ordered_kernel<unroll, true> : engram::gather_ordered_kernel<unroll, false>;
    kern<<<static_cast<unsigned>(gblocks), threads, 0, stream>>>(order, reinterpret_cast<uint4 *>(m), p);
    ENGRAM_LAUNCHED("gather_ordered_kernel launch");
    return ENGRAM_OK;
}

engram::GateParams make_gate_params(const engram_plan *plan, const engram_weights *w, const uint16_t *h,
                                    const uint16_t *v, const float4 *part, int n_tiles, int32_t B, int32_t T,
                                    uint16_t *conv_state, uint16_t *out, float *delta) {
    engram::GateParams p{};
    const int d_h = plan->cfg.hidden_dim;
    p.h = h;
    p.v = v;
    p.part = part;
    p.gamma_c = w->gamma_c;
    p.conv_w = w->conv_w;
    p.conv_state = conv_state;
    p.out = out;
    p.delta = delta;
    p.B = B;
    p.T = T;
    p.d_h = d_h;
    p.n_tiles = n_tiles;
    p.M = plan->num_branches;
    p.n_key_tiles = n_tiles / (p.M + 1);
    p.ksize = plan->cfg.conv_kernel;
    p.dil = plan->cfg.conv_dilation;
    p.state_len = plan->state_len;
    p.tok_chunk = 1;
    p.eps = plan->cfg.eps;
    p.inv_sqrt_d = 1.0f / std::sqrt(static_cast<float>(d_h));
    return p;
}

int launch_gate_conv(const engram_plan *plan, const engram_weights *w, const uint16_t *h, const uint16_t *v,
                     const float4 *part, int n_tiles, int32_t B, int32_t T, uint16_t *conv_state, uint16_t *out,
                     float *delta, cudaStream_t stream, float2 *scal = nullptr) {
    engram::GateParams p{};
    const int d_h = plan->cfg.hidden_dim;
    p.h = h;
    p.v = v;
    p.part = part;
    p.gamma_c = w->gamma_c;
    p.conv_w = w->conv_w;
    p.conv_state = conv_state;
    p.out = out;
    p.delta = delta;
    p.B = B;
    p.T = T;
    p.d_h = d_h;
    p.n_tiles = n_tiles;
    p.M = plan->num_branches;
    p.n_key_tiles = n_tiles / (p.M + 1);
    p.ksize = plan->cfg.conv_kernel;
    p.dil = plan->cfg.conv_dilation;
    p.state_len = plan->state_len;
    constexpr int kChain = 12;   // outputs per residue chain in the k=4, dilation-3 fast path
    const bool k4d3 = p.ksize == 4 && p.dil == 3;
    // the single-branch kernels (decode, short stateful chains) serve M = 1; the generic
    // kernel and the 4-channel prefill kernel serve every M
    const bool fast = k4d3 && p.M == 1 && (conv_state == nullptr || T <= 3 * kChain);
    p.tok_chunk = fast ? 3 * kChain : (conv_state != nullptr ? T : 32);
    p.eps = plan->cfg.eps;
    p.inv_sqrt_d = 1.0f / std::sqrt(static_cast<float>(d_h));
    const int threads = fast ? engram::kGateFastThreads : engram::kGateThreads;
    const int per_thread = fast ? 2 : 4;   // channels per thread
    const unsigned slices = static_cast<unsigned>((d_h / per_thread + threads - 1) / threads) * p.M;
    const size_t smem = sizeof(float) * 2 * static_cast<size_t>(p.tok_chunk + p.state_len);
    if (smem > 48 * 1024) {
        ENGRAM_CUDA_TRY(cudaFuncSetAttribute(engram::gate_conv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem)),
                        "cudaFuncSetAttribute(gate_conv_kernel)");
    }
    if (fast && conv_state != nullptr && T == 1) {
        const unsigned dslices = static_cast<unsigned>((d_h / 2 + engram::kDecodeThreads - 1) / engram::kDecodeThreads);
        ENGRAM_CUDA_TRY(launch_pdl(engram::gate_conv_decode_kernel, dim3(dslices, static_cast<unsigned>(B)),
                                   dim3(engram::kDecodeThreads), 0, stream, p),
                        "gate_conv_decode_kernel launch");
        return ENGRAM_OK;
    }
    dim3 grid(static_cast<unsigned>((T + p.tok_chunk - 1) / p.tok_chunk), static_cast<unsigned>(B), slices);
    if (k4d3 && scal != nullptr && conv_state == nullptr) {
        // scalars once per (token, branch) instead of once per (CTA, halo-extended chunk)
        const int64_t items = static_cast<int64_t>(B) * T * p.M;
        engram::gate_scalars_kernel<<<static_cast<unsigned>((items * 8 + 255) / 256), 256, 0, stream>>>(
            part, static_cast<int64_t>(B) * T, n_tiles, p.n_key_tiles, p.M, d_h, p.eps, p.inv_sqrt_d, scal);
        ENGRAM_LAUNCHED("gate_scalars_kernel launch");
        p.scal = scal;
    }
    if (p.scal != nullptr) {
        // streaming kernel: 9*G tokens per CTA, each thread walking 9*(G+1) positions (the
        // first 9 are the conv halo).  G minimises waves x (positions walked per CTA + a
        // fixed per-CTA cost worth 36 positions): long sequences take the longest walk that
        // fills the waves, short batches (few CTAs in all) a short one.
        const int slices = (d_h / 4 + engram::kStreamThreads - 1) / engram::kStreamThreads;
        const int64_t per_wave = static_cast<int64_t>(sm_count()) * engram::kStreamMinBlocks;
        int best_g = 16;
        int64_t best_cost = -1;
        for (int g : {16, 8, 4, 1}) {
            const int64_t ctas = static_cast<int64_t>((T + 9 * g - 1) / (9 * g)) * p.M * B * slices;
            const int64_t cost = ((ctas + per_wave - 1) / per_wave) * (9 * (g + 1) + 36);
            if (best_cost < 0 || cost < best_cost) {
                best_cost = cost;
                best_g = g;
            }
        }
        const dim3 grid(static_cast<unsigned>((T + 9 * best_g - 1) / (9 * best_g)) * p.M * slices,
                        static_cast<unsigned>(B));
        using SK = void (*)(const engram::GateParams);
        const bool dl = delta != nullptr;
        const SK k = best_g == 16 ? (dl ? engram::gate_stream_kernel<16, true> : engram::gate_stream_kernel<16, false>)
                   : best_g == 8  ? (dl ? engram::gate_stream_kernel<8, true> : engram::gate_stream_kernel<8, false>)
                   : best_g == 4  ? (dl ? engram::gate_stream_kernel<4, true> : engram::gate_stream_kernel<4, false>)
                                  : (dl ? engram::gate_stream_kernel<1, true> : engram::gate_stream_kernel<1, false>);
        k<<<grid, engram::kStreamThreads, 0, stream>>>(p);
        ENGRAM_LAUNCHED("gate_stream_kernel launch");
        return ENGRAM_OK;
    }
    if (fast) engram::gate_conv_k4d3_kernel<kChain><<<grid, threads, 0, stream>>>(p);
    else engram::gate_conv_kernel<<<grid, threads, smem, stream>>>(p);
    ENGRAM_LAUNCHED("gate_conv_kernel launch");
    return ENGRAM_OK;
}

int launch_stage(const engram_plan *plan, const uint32_t *idx, int64_t n_tok, const void *const *tables,
                 void *const *staging, int32_t capacity, uint32_t *staged_idx, uint32_t *unique_rows,
                 int32_t *n_unique, cudaStream_t stream, const engram_row_cache *cache = nullptr,
                 uint32_t *row_flags = nullptr, int32_t *n_hits = nullptr) {
    const int H = plan->num_tables;
    int N = 1;
    while (N < n_tok) N <<= 1;
    const size_t smem = sizeof(uint32_t) * 2 * static_cast<size_t>(N);
    if (smem > 48 * 1024)
        ENGRAM_CUDA_TRY(cudaFuncSetAttribute(engram::stage_dedup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem)),
                        "cudaFuncSetAttribute(stage_dedup_kernel)");
    engram::stage_dedup_kernel<<<H, engram::kDedupThreads, smem, stream>>>(
        idx, static_cast<int32_t>(n_tok), H, capacity, staged_idx, unique_rows, n_unique);
    ENGRAM_LAUNCHED("stage_dedup_kernel launch");
    engram::StageParams p{};
    for (int h = 0; h < H; ++h) {
        p.table[h] = tables[h];
        p.staging[h] = staging[h];
        p.rows[h] = static_cast<uint64_t>(plan->cfg.table_rows[h]);
    }
    p.unique_rows = unique_rows;
    p.n_unique = n_unique;
    p.H = H;
    p.capacity = capacity;
    p.chunks_per_row = plan->cfg.row_dim * table_elem_bytes(plan) / 16;   // rows copied as stored
    const int64_t total = static_cast<int64_t>(H) * n_tok * p.chunks_per_row;
    constexpr int kUnroll = 4;
    int64_t blocks = (total + 256 * kUnroll - 1) / (256 * kUnroll);
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (cache == nullptr) {
        engram::stage_copy_kernel<kUnroll><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
        ENGRAM_LAUNCHED("stage_copy_kernel launch");
        return ENGRAM_OK;
    }
    engram::CacheParams cp{};
    for (int h = 0; h < H; ++h) {
        cp.data[h] = cache->data[h];
        cp.tags[h] = cache->tags[h];
        cp.claim[h] = cache->claim[h];
        cp.rows[h] = static_cast<uint64_t>(plan->cfg.table_rows[h]);
    }
    cp.slot_mask = static_cast<uint64_t>(cache->slots) - 1;
    cp.unique_rows = unique_rows;
    cp.n_unique = n_unique;
    cp.flags = row_flags;
    cp.n_hits = n_hits;
    cp.H = H;
    cp.capacity = capacity;
    const dim3 rgrid(static_cast<unsigned>((n_tok + 255) / 256), static_cast<unsigned>(H));
    engram::cache_probe_kernel<<<rgrid, 256, 0, stream>>>(cp);
    ENGRAM_LAUNCHED("cache_probe_kernel launch");
    engram::cache_decide_kernel<<<rgrid, 256, 0, stream>>>(cp);
    ENGRAM_LAUNCHED("cache_decide_kernel launch");
    engram::cache_copy_kernel<kUnroll><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p, cp);
    ENGRAM_LAUNCHED("cache_copy_kernel launch");
    engram::cache_commit_kernel<<<rgrid, 256, 0, stream>>>(cp);
    ENGRAM_LAUNCHED("cache_commit_kernel launch");
    return ENGRAM_OK;
}

// Remap + hash + dedup + copy of host-table rows in one kernel (batches of at most
// kStageSmallRows (token, table) rows); xr: remapped ids out, or NULL.
int launch_stage_small(const engram_plan *plan, const int32_t *ids, const int32_t *remap, const int32_t *history,
                       int32_t B, int32_t T, const void *const *tables, void *const *staging, int32_t capacity,
                       uint32_t *idx, int32_t *xr, uint32_t *staged_idx, uint32_t *unique_rows, int32_t *n_unique,
                       cudaStream_t stream) {
    const int H = plan->num_tables;
    const engram::HashParams hp = make_hash_params(plan, B, T);
    engram::StageParams sp{};
    for (int h = 0; h < H; ++h) {
        sp.table[h] = tables[h];
        sp.staging[h] = staging[h];
        sp.rows[h] = static_cast<uint64_t>(plan->cfg.table_rows[h]);
    }
    sp.H = H;
    sp.capacity = capacity;
    sp.chunks_per_row = plan->cfg.row_dim * table_elem_bytes(plan) / 16;
    // few CTAs, one warp per distinct row (a row's reads all in flight at once): enough to
    // cover the host link's latency, while leaving the SMs to whatever the prefetch overlaps
    // with (measured on a 64-token step over a 2560^3 GEMM: 8 CTAs hide the most; more
    // shorten the prefetch a little but slow what it overlaps).  ENGRAM_STAGE_CTAS (>= 1)
    // overrides the CTA count (tuning); read once per process.
    static const int forced_ctas = [] {
        const char *e = std::getenv("ENGRAM_STAGE_CTAS");
        const int v = e ? std::atoi(e) : 0;
        return v > 0 ? v : 0;
    }();
    const int64_t rows = static_cast<int64_t>(H) * B * T;   // distinct rows at most
    constexpr int warps = engram::kStageSmallThreads / 32;
    int64_t blocks = (rows + warps - 1) / warps;
    const int64_t cap = forced_ctas ? forced_ctas : 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    engram::stage_small_kernel<<<static_cast<unsigned>(blocks), engram::kStageSmallThreads, 0, stream>>>(
        ids, remap, history, idx, xr, staged_idx, unique_rows, n_unique, hp, sp);
    ENGRAM_LAUNCHED("stage_small_kernel launch");
    return ENGRAM_OK;
}

int check_row_cache(const engram_plan *plan, const engram_row_cache *cache) {
    if (cache == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "cache is NULL");
    if (cache->slots < 1 || cache->slots > (int64_t(1) << 32) || (cache->slots & (cache->slots - 1)))
        return fail(ENGRAM_ERR_INVALID_ARG, "cache slots must be a power of two in [1, 2^32]");
    for (int h = 0; h < plan->num_tables; ++h) {
        if (!cache->data[h] || !cache->tags[h] || !cache->claim[h])
            return fail(ENGRAM_ERR_INVALID_ARG, "cache buffers of table %d are NULL", h);
        if (!aligned16(cache->data[h])) return fail(ENGRAM_ERR_INVALID_ARG, "cache data of table %d not 16-byte aligned", h);
    }
    return ENGRAM_OK;
}

// Stage events are profiling hooks.  Under stream capture they must become event-record
// nodes of the graph (cudaEventRecordExternal) so that they can be timed after a replay.
cudaError_t record_stage_event(void *ev, cudaStream_t stream) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &st);
    if (e != cudaSuccess) return e;
    if (st == cudaStreamCaptureStatusActive)
        return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev), stream, cudaEventRecordExternal);
    return cudaEventRecord(static_cast<cudaEvent_t>(ev), stream);
}

// history / xr (engram_forward's decode steps): when the step ends in decode_fused_kernel, that
// kernel also advances the hash history and *history_done is set; otherwise the caller does.
// in_call: the kernel before the projection belongs to the same entry-point call (engram_forward),
// so the projection may overlap it (launch_ex).
int gate_conv_impl(const engram_plan *plan, const engram_weights *w, const uint16_t *h, const uint16_t *m,
                   int32_t B, int32_t T, uint16_t *conv_state, uint16_t *out, float *delta, uint8_t *ws,
                   cudaStream_t stream, void *const *events, bool in_call, int32_t *history = nullptr,
                   const int32_t *xr = nullptr, bool *history_done = nullptr) {
    if (history_done) *history_done = false;
    const int64_t n_tok = static_cast<int64_t>(B) * T;
    const Workspace L = layout(plan, n_tok);
    const ProjShape ps = proj_shape(plan, n_tok, true);
    uint16_t *v = reinterpret_cast<uint16_t *>(ws + L.v);
    float4 *part = reinterpret_cast<float4 *>(ws + L.part);
    float *acc = ps.k_splits > 1 ? reinterpret_cast<float *>(ws + L.acc) : nullptr;
    const int d_h = plan->cfg.hidden_dim;
    // one-token decode steps after a split-K projection: reduce + gate + conv in one kernel
    const bool fused_decode = ps.k_splits > 1 && T == 1 && plan->num_branches == 1 && plan->cfg.conv_kernel == 4 &&
                              plan->cfg.conv_dilation == 3 && d_h <= 8 * engram::kFusedDecodeMaxThreads &&
                              d_h % 256 == 0;   // d_h / 8 threads: whole warps
    engram::ProjParams pp{};
    int rc;
    if (events) ENGRAM_CUDA_TRY(record_stage_event(events[0], stream), "cudaEventRecord");
    const int n_tiles = ps.n_tiles;
    if (ps.pair)
        rc = launch_proj_pair(plan, w, h, m, n_tok, v, part, stream, acc, ps.k_splits, ps.kb_per_split, !fused_decode,
                              &pp, in_call);
    else if (ps.bn == 256)
        rc = launch_proj<256>(plan, w, h, m, n_tok, v, part, stream, acc, ps.k_splits, ps.kb_per_split, !fused_decode, &pp,
                              ProjTest(), in_call);
    else if (ps.bn == 128)
        rc = launch_proj<128>(plan, w, h, m, n_tok, v, part, stream, acc, ps.k_splits, ps.kb_per_split, !fused_decode, &pp,
                              ProjTest(), in_call);
    else
        rc = launch_proj<64>(plan, w, h, m, n_tok, v, part, stream, acc, ps.k_splits, ps.kb_per_split, !fused_decode, &pp,
                              ProjTest(), in_call);
    if (rc != ENGRAM_OK) return rc;
    if (events) ENGRAM_CUDA_TRY(record_stage_event(events[1], stream), "cudaEventRecord");
    if (fused_decode) {
        engram::GateParams gp = make_gate_params(plan, w, h, v, part, ps.n_tiles, B, T, conv_state, out, delta);
        if (history != nullptr && xr != nullptr && plan->hist_len > 0) {
            gp.history = history;
            gp.xr = xr;
            gp.hist_len = plan->hist_len;
        }
        ENGRAM_CUDA_TRY(launch_pdl(d_h <= 8 * 320 ? engram::decode_fused_kernel<320>
                                                  : engram::decode_fused_kernel<engram::kFusedDecodeMaxThreads>,
                                   dim3(static_cast<unsigned>(B)), dim3(d_h / 8), 0, stream, pp, gp),
                        "decode_fused_kernel launch");
        ENGRAM_CUDA_TRY(cudaGetLastError(), "decode_fused_kernel launch");
        if (history_done) *history_done = gp.history != nullptr;
        return ENGRAM_OK;
    }
    return launch_gate_conv(plan, w, h, v, part, n_tiles, B, T, conv_state, out, delta, stream,
                            reinterpret_cast<float2 *>(ws + L.scal));
}

int check_bt(int32_t B, int32_t T) {
    if (B < 0 || T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B and T must be >= 0 (got %d, %d)", B, T);
    if (static_cast<int64_t>(B) * T > (int64_t(1) << 31))
        return fail(ENGRAM_ERR_UNSUPPORTED, "B*T above 2^31 tokens per call");
    if (B > 65535) return fail(ENGRAM_ERR_UNSUPPORTED, "B above 65535 sequences per call");
    return ENGRAM_OK;
}

// ---------------------------------------------------------------- no-allocation variant
// Scratch for engram_gate_conv_noalloc: one array per device in the library's static device
// data.  Host code may not pass the symbol itself to a kernel (on the host it only names a
// shadow variable); its device address is looked up below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[ENGRAM_NOALLOC_SCRATCH_BYTES];

// Looked up on every call, with the caller's device current: a host-side lookup that
// allocates nothing, and stays right if the context (and the module with it) is recreated.
int noalloc_scratch(uint8_t **out) {
    void *p = nullptr;
    ENGRAM_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(no-alloc scratch)");
    *out = static_cast<uint8_t *>(p);
    return ENGRAM_OK;
}

}  // namespace

// =====================================================================================
extern "C" {

const char *engram_last_error(void) { return g_last_error.c_str(); }

const char *engram_version(void) { return "0.1.0"; }

size_t engram_sizeof(const char *type_name) {
    if (type_name == nullptr) return 0;
    if (std::strcmp(type_name, "engram_config") == 0) return sizeof(engram_config);
    if (std::strcmp(type_name, "engram_plan") == 0) return sizeof(engram_plan);
    if (std::strcmp(type_name, "engram_weights") == 0) return sizeof(engram_weights);
    if (std::strcmp(type_name, "engram_row_cache") == 0) return sizeof(engram_row_cache);
    return 0;
}

int engram_init(const engram_config *cfg, engram_plan *plan) {
    g_last_error.clear();
    if (cfg == nullptr || plan == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "cfg and plan must be non-NULL");
    const engram_config &c = *cfg;
    if (c.num_orders < 1 || c.num_orders > ENGRAM_MAX_ORDERS)
        return fail(ENGRAM_ERR_UNSUPPORTED, "num_orders must be in 1..%d", ENGRAM_MAX_ORDERS);
    for (int i = 0; i < c.num_orders; ++i) {
        if (c.orders[i] < 1 || c.orders[i] > ENGRAM_MAX_ORDERS)
            return fail(ENGRAM_ERR_UNSUPPORTED, "order %d outside 1..%d", c.orders[i], ENGRAM_MAX_ORDERS);
        if (i > 0 && c.orders[i] <= c.orders[i - 1])
            return fail(ENGRAM_ERR_INVALID_ARG, "orders must be strictly increasing");
    }
    if (c.heads_per_order < 1) return fail(ENGRAM_ERR_INVALID_ARG, "heads_per_order must be >= 1");
    const int H = c.num_orders * c.heads_per_order;
    if (H > ENGRAM_MAX_TABLES) return fail(ENGRAM_ERR_UNSUPPORTED, "num_orders * heads_per_order > %d", ENGRAM_MAX_TABLES);
    for (int h = 0; h < H; ++h) {
        const int64_t P = c.table_rows[h];
        if (P < 2 || P > 0xFFFFFFFFll) return fail(ENGRAM_ERR_INVALID_ARG, "table_rows[%d] = %lld outside [2, 2^32)", h, (long long)P);
        if (!is_prime_u32(static_cast<uint64_t>(P)))
            return fail(ENGRAM_ERR_INVALID_ARG, "table_rows[%d] = %lld is not prime", h, (long long)P);
    }
    for (int h = H; h < ENGRAM_MAX_TABLES; ++h)
        if (c.table_rows[h] != 0) return fail(ENGRAM_ERR_INVALID_ARG, "table_rows[%d] set beyond the %d tables", h, H);
    if (c.row_dim <= 0 || c.row_dim % 8 != 0) return fail(ENGRAM_ERR_UNSUPPORTED, "row_dim must be a positive multiple of 8");
    if (c.hidden_dim <= 0 || c.hidden_dim % 64 != 0)
        return fail(ENGRAM_ERR_UNSUPPORTED, "hidden_dim must be a positive multiple of 64");
    if (static_cast<int64_t>(H) * c.row_dim > (1 << 20)) return fail(ENGRAM_ERR_UNSUPPORTED, "memory dim above 2^20");
    if (c.vocab_in <= 0 || c.vocab_out <= 0) return fail(ENGRAM_ERR_INVALID_ARG, "vocab sizes must be positive");
    if (c.vocab_out == 0x7FFFFFFF) return fail(ENGRAM_ERR_INVALID_ARG, "vocab_out too large (pad id must fit)");
    if (c.pad_id != c.vocab_out) return fail(ENGRAM_ERR_INVALID_ARG, "pad_id must equal vocab_out");
    if (c.conv_kernel < 1 || c.conv_kernel > 8) return fail(ENGRAM_ERR_UNSUPPORTED, "conv_kernel must be in 1..8");
    if (c.conv_dilation != c.orders[c.num_orders - 1])
        return fail(ENGRAM_ERR_INVALID_ARG, "conv_dilation must equal the largest order");
    if (!(c.eps > 0.f) || !std::isfinite(c.eps)) return fail(ENGRAM_ERR_INVALID_ARG, "eps must be a positive finite number");
    if (c.table_location != ENGRAM_TABLES_DEVICE && c.table_location != ENGRAM_TABLES_HOST_MAPPED)
        return fail(ENGRAM_ERR_INVALID_ARG, "unknown table_location");
    for (int i = 0; i < 4; ++i)
        if (c.reserved[i] != 0) return fail(ENGRAM_ERR_INVALID_ARG, "reserved fields must be zero");
    const int M = c.num_branches == 0 ? 1 : c.num_branches;
    if (M < 1 || M > ENGRAM_MAX_BRANCHES)
        return fail(ENGRAM_ERR_UNSUPPORTED, "num_branches must be in 0..%d", ENGRAM_MAX_BRANCHES);
    if (c.table_dtype != ENGRAM_TABLE_BF16 && c.table_dtype != ENGRAM_TABLE_FP8_E4M3)
        return fail(ENGRAM_ERR_INVALID_ARG, "unknown table_dtype %d", c.table_dtype);
    for (int h = 0; h < ENGRAM_MAX_TABLES; ++h) {
        const float sc = c.table_scale[h];
        if (c.table_dtype == ENGRAM_TABLE_FP8_E4M3 && h < H) {
            // products of codes (2^-9 .. 448) and scales in this range stay normal fp32 values
            if (!(sc >= 0x1p-100f && sc <= 0x1p100f))
                return fail(ENGRAM_ERR_INVALID_ARG, "table_scale[%d] must lie in [2^-100, 2^100]", h);
        } else if (sc != 0.f) {
            return fail(ENGRAM_ERR_INVALID_ARG, "table_scale[%d] must be 0 (bf16 tables or beyond the %d tables)", h, H);
        }
    }
    if (c.table_dtype == ENGRAM_TABLE_FP8_E4M3 && c.row_dim % 16 != 0)
        return fail(ENGRAM_ERR_UNSUPPORTED, "FP8 tables need row_dim % 16 == 0");
    if (c.flags & ~(ENGRAM_FLAG_SINGLE_CTA_MMA | ENGRAM_FLAG_ROW_ORDER_GATHER | ENGRAM_FLAG_BULK_GATHER))
        return fail(ENGRAM_ERR_INVALID_ARG, "unknown flags 0x%x", c.flags);

    std::memset(plan, 0, sizeof *plan);
    plan->cfg = c;
    for (int oi = 0; oi < c.num_orders; ++oi)
        for (int j = 0; j < c.heads_per_order; ++j)
            for (int i = 0; i < c.orders[oi]; ++i) {
                const uint64_t key = c.hash_seed ^ ((static_cast<uint64_t>(c.orders[oi]) << 16) ^
                                                    (static_cast<uint64_t>(j) << 8) ^ static_cast<uint64_t>(i));
                plan->mult[oi * c.heads_per_order + j][i] = splitmix64_first(key) | 1ull;
            }
    plan->num_tables = H;
    plan->num_branches = M;
    plan->mem_dim = H * c.row_dim;
    plan->hist_len = c.orders[c.num_orders - 1] - 1;
    plan->state_len = (c.conv_kernel - 1) * c.conv_dilation;
    plan->magic = kPlanMagic;
    return ENGRAM_OK;
}

size_t engram_workspace_size(const engram_plan *plan, int64_t n_tok) {
    if (plan == nullptr || plan->magic != kPlanMagic || n_tok < 0) return 0;
    return layout(plan, n_tok).total;
}

int engram_remap(const engram_plan *plan, const int32_t *ids, int64_t n, const int32_t *remap, int32_t *out,
                 engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if (n < 0) return fail(ENGRAM_ERR_INVALID_ARG, "n must be >= 0");
    if (n == 0) return ENGRAM_OK;
    if (!ids || !remap || !out) return fail(ENGRAM_ERR_INVALID_ARG, "ids, remap and out must be non-NULL");
    const int threads = 256;
    int64_t blocks = (n + threads - 1) / threads;
    if (blocks > 65535LL * 16) blocks = 65535LL * 16;
    engram::remap_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
        ids, n, remap, plan->cfg.vocab_in, plan->cfg.pad_id, out);
    ENGRAM_LAUNCHED("remap_kernel launch");
    return ENGRAM_OK;
}

int engram_hash(const engram_plan *plan, const int32_t *ids_remapped, int32_t B, int32_t T,
                const int32_t *history, uint32_t *idx, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = check_bt(B, T)) != ENGRAM_OK) return rc;
    if (static_cast<int64_t>(B) * T == 0) return ENGRAM_OK;
    if (!ids_remapped || !idx) return fail(ENGRAM_ERR_INVALID_ARG, "ids_remapped and idx must be non-NULL");
    return launch_hash(plan, ids_remapped, nullptr, history, B, T, idx, nullptr, static_cast<cudaStream_t>(stream));
}

int engram_advance_history(const engram_plan *plan, const int32_t *ids_remapped, int32_t B, int32_t T,
                           int32_t *history, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = check_bt(B, T)) != ENGRAM_OK) return rc;
    if (B == 0 || plan->hist_len == 0) return ENGRAM_OK;
    if (!history || (T > 0 && !ids_remapped)) return fail(ENGRAM_ERR_INVALID_ARG, "history and ids must be non-NULL");
    engram::advance_history_kernel<<<(B + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(
        ids_remapped, B, T, history, plan->hist_len);
    ENGRAM_LAUNCHED("advance_history_kernel launch");
    return ENGRAM_OK;
}

int engram_gather(const engram_plan *plan, const uint32_t *idx, const void *const *tables, int64_t n_tok,
                  uint16_t *m, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if (n_tok < 0) return fail(ENGRAM_ERR_INVALID_ARG, "n_tok must be >= 0");
    if (n_tok == 0) return ENGRAM_OK;
    if (!idx || !tables || !m) return fail(ENGRAM_ERR_INVALID_ARG, "idx, tables and m must be non-NULL");
    if (!aligned16(m)) return fail(ENGRAM_ERR_INVALID_ARG, "m is not 16-byte aligned");
    for (int h = 0; h < plan->num_tables; ++h) {
        if (!tables[h]) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] is NULL", h);
        if (!aligned16(tables[h])) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] is not 16-byte aligned", h);
    }
    return launch_gather(plan, idx, tables, n_tok, m, static_cast<cudaStream_t>(stream));
}

int engram_gather_bounded(const engram_plan *plan, const uint32_t *idx, const void *const *tables,
                          int64_t n_tok, int64_t rows, uint16_t *m, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if (n_tok < 0 || rows < 1) return fail(ENGRAM_ERR_INVALID_ARG, "n_tok must be >= 0 and rows >= 1");
    if (n_tok == 0) return ENGRAM_OK;
    if (!idx || !tables || !m) return fail(ENGRAM_ERR_INVALID_ARG, "idx, tables and m must be non-NULL");
    if (!aligned16(m)) return fail(ENGRAM_ERR_INVALID_ARG, "m is not 16-byte aligned");
    for (int h = 0; h < plan->num_tables; ++h) {
        if (!tables[h]) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] is NULL", h);
        if (!aligned16(tables[h])) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] is not 16-byte aligned", h);
    }
    return launch_gather(plan, idx, tables, n_tok, m, static_cast<cudaStream_t>(stream), rows);
}

int engram_stage_rows(const engram_plan *plan, const uint32_t *idx, int64_t n_tok, const void *const *tables,
                      void *const *staging, int32_t capacity, uint32_t *staged_idx, uint32_t *unique_rows,
                      int32_t *n_unique, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if (n_tok < 0) return fail(ENGRAM_ERR_INVALID_ARG, "n_tok must be >= 0");
    if (n_tok == 0) return ENGRAM_OK;
    if (n_tok > engram::kStageMaxTok)
        return fail(ENGRAM_ERR_UNSUPPORTED, "engram_stage_rows handles at most %d tokens per call", engram::kStageMaxTok);
    if (capacity < n_tok) return fail(ENGRAM_ERR_INVALID_ARG, "capacity %d < n_tok %lld", capacity, (long long)n_tok);
    if (!idx || !tables || !staging || !staged_idx || !unique_rows || !n_unique)
        return fail(ENGRAM_ERR_INVALID_ARG, "NULL argument");
    for (int h = 0; h < plan->num_tables; ++h) {
        if (!tables[h] || !staging[h]) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] or staging[%d] is NULL", h, h);
        if (!aligned16(tables[h]) || !aligned16(staging[h]))
            return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] / staging[%d] not 16-byte aligned", h, h);
    }
    return launch_stage(plan, idx, n_tok, tables, staging, capacity, staged_idx, unique_rows, n_unique,
                        static_cast<cudaStream_t>(stream));
}

int engram_stage_rows_from_ids(const engram_plan *plan, const int32_t *ids, const int32_t *remap, int32_t B,
                               int32_t T, const int32_t *history, const void *const *tables, void *const *staging,
                               int32_t capacity, uint32_t *idx, uint32_t *staged_idx, uint32_t *unique_rows,
                               int32_t *n_unique, engram_stream_t stream_) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = check_bt(B, T)) != ENGRAM_OK) return rc;
    const int64_t n_tok = static_cast<int64_t>(B) * T;
    if (n_tok == 0) return ENGRAM_OK;
    if (n_tok > engram::kStageMaxTok)
        return fail(ENGRAM_ERR_UNSUPPORTED, "engram_stage_rows_from_ids handles at most %d tokens per call",
                    engram::kStageMaxTok);
    if (capacity < n_tok) return fail(ENGRAM_ERR_INVALID_ARG, "capacity %d < n_tok %lld", capacity, (long long)n_tok);
    if (!ids || !idx || !tables || !staging || !staged_idx || !unique_rows || !n_unique)
        return fail(ENGRAM_ERR_INVALID_ARG, "NULL argument");
    for (int h = 0; h < plan->num_tables; ++h) {
        if (!tables[h] || !staging[h]) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] or staging[%d] is NULL", h, h);
        if (!aligned16(tables[h]) || !aligned16(staging[h]))
            return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] / staging[%d] not 16-byte aligned", h, h);
    }
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (n_tok * plan->num_tables <= engram::kStageSmallRows)
        return launch_stage_small(plan, ids, remap, history, B, T, tables, staging, capacity, idx, nullptr,
                                  staged_idx, unique_rows, n_unique, stream);
    if ((rc = launch_hash(plan, ids, remap, history, B, T, idx, nullptr, stream)) != ENGRAM_OK) return rc;
    return launch_stage(plan, idx, n_tok, tables, staging, capacity, staged_idx, unique_rows, n_unique, stream);
}

size_t engram_packed_weights_size(const engram_plan *plan) {
    if (plan == nullptr || plan->magic != kPlanMagic) return 0;
    return packed_weights_bytes(plan);
}

int engram_pack_weights(const engram_plan *plan, const uint16_t *w_k, const uint16_t *w_v, void *packed,
                        size_t packed_bytes, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    const size_t need = packed_weights_bytes(plan);
    if (need == 0) return fail(ENGRAM_ERR_UNSUPPORTED, "no packed form for hidden_dim %% 256 != 0");
    if (!w_k || !w_v || !packed) return fail(ENGRAM_ERR_INVALID_ARG, "w_k, w_v and packed must be non-NULL");
    if (!aligned16(w_k) || !aligned16(w_v) || !aligned16(packed))
        return fail(ENGRAM_ERR_INVALID_ARG, "w_k, w_v and packed must be 16-byte aligned");
    if (packed_bytes < need) return fail(ENGRAM_ERR_INVALID_ARG, "packed buffer too small: need %zu bytes", need);
    const int64_t n_chunks = static_cast<int64_t>(need / 16);
    int64_t blocks = (n_chunks + 255) / 256;
    if (blocks > static_cast<int64_t>(sm_count()) * 16) blocks = static_cast<int64_t>(sm_count()) * 16;
    engram::pack_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        w_k, w_v, static_cast<int64_t>(plan->num_branches) * plan->cfg.hidden_dim, plan->mem_dim,
        (plan->mem_dim + engram::kBK - 1) / engram::kBK, n_chunks, static_cast<uint4 *>(packed));
    ENGRAM_LAUNCHED("pack_weights_kernel launch");
    return ENGRAM_OK;
}

int engram_row_cache_reset(const engram_plan *plan, const engram_row_cache *cache, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = check_row_cache(plan, cache)) != ENGRAM_OK) return rc;
    for (int h = 0; h < plan->num_tables; ++h) {
        int64_t blocks = (cache->slots + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;
        engram::cache_reset_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
            cache->tags[h], cache->claim[h], cache->slots);
        ENGRAM_LAUNCHED("cache_reset_kernel launch");
    }
    return ENGRAM_OK;
}

int engram_stage_rows_cached(const engram_plan *plan, const uint32_t *idx, int64_t n_tok, const void *const *tables,
                             const engram_row_cache *cache, void *const *staging, int32_t capacity,
                             uint32_t *staged_idx, uint32_t *unique_rows, int32_t *n_unique, uint32_t *row_flags,
                             int32_t *n_hits, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if (n_tok < 0) return fail(ENGRAM_ERR_INVALID_ARG, "n_tok must be >= 0");
    if (n_tok == 0) return ENGRAM_OK;
    if ((rc = check_row_cache(plan, cache)) != ENGRAM_OK) return rc;
    if (n_tok > engram::kStageMaxTok)
        return fail(ENGRAM_ERR_UNSUPPORTED, "engram_stage_rows_cached handles at most %d tokens per call", engram::kStageMaxTok);
    if (capacity < n_tok) return fail(ENGRAM_ERR_INVALID_ARG, "capacity %d < n_tok %lld", capacity, (long long)n_tok);
    if (!idx || !tables || !staging || !staged_idx || !unique_rows || !n_unique || !row_flags || !n_hits)
        return fail(ENGRAM_ERR_INVALID_ARG, "NULL argument");
    for (int h = 0; h < plan->num_tables; ++h) {
        if (!tables[h] || !staging[h]) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] or staging[%d] is NULL", h, h);
        if (!aligned16(tables[h]) || !aligned16(staging[h]))
            return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] / staging[%d] not 16-byte aligned", h, h);
    }
    return launch_stage(plan, idx, n_tok, tables, staging, capacity, staged_idx, unique_rows, n_unique,
                        static_cast<cudaStream_t>(stream), cache, row_flags, n_hits);
}

int engram_gate_conv(const engram_plan *plan, const engram_weights *w, const uint16_t *h, const uint16_t *m,
                     int32_t B, int32_t T, uint16_t *conv_state, uint16_t *out, float *delta_dbg, void *workspace,
                     size_t workspace_bytes, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = check_bt(B, T)) != ENGRAM_OK) return rc;
    if ((rc = validate_weights(plan, w)) != ENGRAM_OK) return rc;
    const int64_t n_tok = static_cast<int64_t>(B) * T;
    if (n_tok == 0) return ENGRAM_OK;
    if (!h || !m || !out) return fail(ENGRAM_ERR_INVALID_ARG, "h, m and out must be non-NULL");
    if (!aligned16(h) || !aligned16(m) || !aligned16(out) || (delta_dbg && !aligned16(delta_dbg)) ||
        (conv_state && !aligned16(conv_state)))
        return fail(ENGRAM_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (conv_state && T > 16384) return fail(ENGRAM_ERR_UNSUPPORTED, "T above 16384 with a conv state");
    const size_t need = layout(plan, n_tok).total;
    if (!workspace || workspace_bytes < need)
        return fail(ENGRAM_ERR_INVALID_ARG, "workspace too small: need %zu bytes", need);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(ENGRAM_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    return gate_conv_impl(plan, w, h, m, B, T, conv_state, out, delta_dbg, static_cast<uint8_t *>(workspace),
                          static_cast<cudaStream_t>(stream), nullptr, false);
}

int engram_forward(const engram_plan *plan, const engram_weights *w, const void *const *tables,
                   const int32_t *ids, const int32_t *remap, int32_t B, int32_t T, int32_t *history,
                   uint16_t *conv_state, const uint16_t *h, uint16_t *out, float *delta_dbg, void *workspace,
                   size_t workspace_bytes, engram_stream_t stream_, void *const *stage_events) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = check_bt(B, T)) != ENGRAM_OK) return rc;
    if ((rc = validate_weights(plan, w)) != ENGRAM_OK) return rc;
    const int64_t n_tok = static_cast<int64_t>(B) * T;
    if (n_tok == 0) return ENGRAM_OK;
    if (!ids || !h || !out || !tables) return fail(ENGRAM_ERR_INVALID_ARG, "ids, tables, h and out must be non-NULL");
    if (!aligned16(h) || !aligned16(out) || (delta_dbg && !aligned16(delta_dbg)) || (conv_state && !aligned16(conv_state)))
        return fail(ENGRAM_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    for (int t = 0; t < plan->num_tables; ++t) {
        if (!tables[t]) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] is NULL", t);
        if (!aligned16(tables[t])) return fail(ENGRAM_ERR_INVALID_ARG, "tables[%d] is not 16-byte aligned", t);
    }
    if (conv_state && T > 16384) return fail(ENGRAM_ERR_UNSUPPORTED, "T above 16384 with a conv state");
    const Workspace L = layout(plan, n_tok);
    if (!workspace || workspace_bytes < L.total)
        return fail(ENGRAM_ERR_INVALID_ARG, "workspace too small: need %zu bytes", L.total);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return fail(ENGRAM_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int32_t *xr = reinterpret_cast<int32_t *>(ws + L.xr);
    uint32_t *idx = reinterpret_cast<uint32_t *>(ws + L.idx);
    uint16_t *m = reinterpret_cast<uint16_t *>(ws + L.m);
    auto rec = [&](int i) -> int {
        if (stage_events) ENGRAM_CUDA_TRY(record_stage_event(stage_events[i], stream), "cudaEventRecord");
        return ENGRAM_OK;
    };
    // Decode-sized batches on HBM-resident tables: remap + hash + gather in one kernel (the
    // row ids stay in registers).  Larger batches: the hash kernel, then the wide gather.
    const ForwardPath fp = forward_path(plan, n_tok);
    const bool fused_lookup = fp.fused_lookup;
    if ((rc = rec(0)) != ENGRAM_OK) return rc;
    const bool stage_small = L.staged && n_tok * plan->num_tables <= engram::kStageSmallRows;
    if (fused_lookup) {
        if ((rc = rec(1)) != ENGRAM_OK) return rc;
        if ((rc = launch_lookup(plan, ids, remap, history, B, T, tables, xr, m, stream)) != ENGRAM_OK) return rc;
    } else if (stage_small) {
        // host-resident tables, decode-sized batch: hash + dedup + staging copy in one kernel
        const int64_t stage_bytes = n_tok * plan->cfg.row_dim * table_elem_bytes(plan);   // per table
        void *stage_ptr[ENGRAM_MAX_TABLES];
        for (int hh = 0; hh < plan->num_tables; ++hh) stage_ptr[hh] = ws + L.staging + static_cast<int64_t>(hh) * stage_bytes;
        if ((rc = launch_stage_small(plan, ids, remap, history, B, T, tables, stage_ptr, static_cast<int32_t>(n_tok),
                                     idx, xr, reinterpret_cast<uint32_t *>(ws + L.staged_idx),
                                     reinterpret_cast<uint32_t *>(ws + L.unique),
                                     reinterpret_cast<int32_t *>(ws + L.n_unique), stream)) != ENGRAM_OK)
            return rc;
        if ((rc = rec(1)) != ENGRAM_OK) return rc;
    } else {
        if ((rc = launch_hash(plan, ids, remap, history, B, T, idx, xr, stream)) != ENGRAM_OK) return rc;
        if ((rc = rec(1)) != ENGRAM_OK) return rc;
    }
    if (fused_lookup) {
        // rows already in m
    } else if (L.staged) {
        // host-resident tables: fetch each distinct row of the batch once into HBM staging,
        // then gather from there (results are bit-identical to the HBM-resident path)
        const int H = plan->num_tables;
        void *stage_ptr[ENGRAM_MAX_TABLES];
        const int64_t stage_bytes = n_tok * plan->cfg.row_dim * table_elem_bytes(plan);   // per table
        for (int h = 0; h < H; ++h) stage_ptr[h] = ws + L.staging + static_cast<int64_t>(h) * stage_bytes;
        uint32_t *sidx = reinterpret_cast<uint32_t *>(ws + L.staged_idx);
        if (!stage_small &&
            (rc = launch_stage(plan, idx, n_tok, tables, stage_ptr, static_cast<int32_t>(n_tok), sidx,
                               reinterpret_cast<uint32_t *>(ws + L.unique), reinterpret_cast<int32_t *>(ws + L.n_unique),
                               stream)) != ENGRAM_OK)
            return rc;
        if ((rc = launch_gather(plan, sidx, stage_ptr, n_tok, m, stream, n_tok)) != ENGRAM_OK) return rc;
    } else if (fp.row_order) {
        if ((rc = launch_gather_ordered(plan, idx, tables, n_tok, m, reinterpret_cast<uint32_t *>(ws + L.order_count),
                                        reinterpret_cast<uint32_t *>(ws + L.order_cursor),
                                        reinterpret_cast<uint2 *>(ws + L.order), stream)) != ENGRAM_OK)
            return rc;
    } else if ((rc = launch_gather(plan, idx, tables, n_tok, m, stream)) != ENGRAM_OK) {
        return rc;
    }
    bool history_done = false;
    if ((rc = gate_conv_impl(plan, w, h, m, B, T, conv_state, out, delta_dbg, ws, stream,
                             stage_events ? stage_events + 2 : nullptr, true, history, xr, &history_done)) != ENGRAM_OK)
        return rc;
    if ((rc = rec(4)) != ENGRAM_OK) return rc;
    if (history != nullptr && plan->hist_len > 0 && !history_done) {
        ENGRAM_CUDA_TRY(launch_pdl(engram::advance_history_kernel, dim3((B + 127) / 128), dim3(128), 0, stream,
                                   static_cast<const int32_t *>(xr), B, T, history, static_cast<int32_t>(plan->hist_len)),
                        "advance_history_kernel launch");
    }
    return ENGRAM_OK;
}

int engram_gate_conv_noalloc(const engram_plan *plan, const engram_weights *w, const uint16_t *h,
                             const uint16_t *m, int32_t B, int32_t T, uint16_t *conv_state, uint16_t *out,
                             float *delta_dbg, engram_stream_t stream_) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = check_bt(B, T)) != ENGRAM_OK) return rc;
    if ((rc = validate_weights(plan, w)) != ENGRAM_OK) return rc;
    const int64_t n_tok = static_cast<int64_t>(B) * T;
    if (n_tok == 0) return ENGRAM_OK;
    if (!h || !m || !out) return fail(ENGRAM_ERR_INVALID_ARG, "h, m and out must be non-NULL");
    if (!aligned16(h) || !aligned16(m) || !aligned16(out) || (delta_dbg && !aligned16(delta_dbg)) ||
        (conv_state && !aligned16(conv_state)))
        return fail(ENGRAM_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (conv_state && T > 16384) return fail(ENGRAM_ERR_UNSUPPORTED, "T above 16384 with a conv state");
    const int d_h = plan->cfg.hidden_dim;
    const int bn = choose_bn(d_h, n_tok, plan->num_branches);
    const int n_tiles = (plan->num_branches + 1) * d_h / bn;
    const size_t v_bytes = align256(sizeof(uint16_t) * static_cast<size_t>(n_tok) * d_h);
    const size_t part_bytes = align256(sizeof(float4) * static_cast<size_t>(n_tok) * n_tiles);
    if (v_bytes + part_bytes > ENGRAM_NOALLOC_SCRATCH_BYTES)
        return fail(ENGRAM_ERR_UNSUPPORTED,
                    "%lld tokens need %zu bytes of scratch; the static scratch holds %u bytes",
                    static_cast<long long>(n_tok), v_bytes + part_bytes, ENGRAM_NOALLOC_SCRATCH_BYTES);
    uint8_t *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != ENGRAM_OK) return rc;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    uint16_t *v = reinterpret_cast<uint16_t *>(scratch);
    float4 *part = reinterpret_cast<float4 *>(scratch + v_bytes);
    // the first kernel of the call: no overlap with the caller's earlier kernels (launch_ex)
    if (bn == 256) rc = launch_proj<256>(plan, w, h, m, n_tok, v, part, stream, nullptr, 1, 0, true, nullptr, ProjTest(), false);
    else if (bn == 128) rc = launch_proj<128>(plan, w, h, m, n_tok, v, part, stream, nullptr, 1, 0, true, nullptr, ProjTest(), false);
    else rc = launch_proj<64>(plan, w, h, m, n_tok, v, part, stream, nullptr, 1, 0, true, nullptr, ProjTest(), false);
    if (rc != ENGRAM_OK) return rc;
    return launch_gate_conv(plan, w, h, v, part, n_tiles, B, T, conv_state, out, delta_dbg, stream);
}

int engram_forward_path(const engram_plan *plan, int32_t B, int32_t T, uint32_t *path) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = check_bt(B, T)) != ENGRAM_OK) return rc;
    if (path == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "path is NULL");
    const int64_t n_tok = static_cast<int64_t>(B) * T;
    const ForwardPath fp = forward_path(plan, n_tok);
    uint32_t bits = 0;
    if (fp.fused_lookup) bits |= ENGRAM_PATH_FUSED_LOOKUP;
    if (fp.staged) bits |= ENGRAM_PATH_STAGED_ROWS;
    if (fp.ps.k_splits > 1) bits |= ENGRAM_PATH_SPLIT_K;
    if (fp.pair) bits |= ENGRAM_PATH_PAIR_MMA;
    if (fp.row_order) bits |= ENGRAM_PATH_ROW_ORDER;
    if (!fp.fused_lookup && !fp.row_order && bulk_gather(plan, n_tok)) bits |= ENGRAM_PATH_BULK_GATHER;
    *path = bits;
    return ENGRAM_OK;
}

int engram_synchronize(engram_stream_t stream) {
    ENGRAM_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize");
    uint32_t s = 0;
    ENGRAM_CUDA_TRY(cudaMemcpyFromSymbol(&s, g_engram_status, sizeof s), "cudaMemcpyFromSymbol");
    if (s & ENGRAM_STATUS_WAIT_TIMEOUT)
        return fail(ENGRAM_ERR_TIMEOUT, "a pipeline wait inside a kernel gave up (device status 0x%x)", s);
    return ENGRAM_OK;
}

int engram_selftest_wait_timeout(const engram_plan *plan, const engram_weights *w, const uint16_t *h,
                                 const uint16_t *m, int64_t n_tok, void *workspace, size_t workspace_bytes,
                                 uint64_t wait_limit_ns, engram_stream_t stream) {
    int rc;
    if ((rc = check_plan(plan)) != ENGRAM_OK) return rc;
    if ((rc = validate_weights(plan, w)) != ENGRAM_OK) return rc;
    if (n_tok < 1 || n_tok > (int64_t(1) << 31)) return fail(ENGRAM_ERR_INVALID_ARG, "n_tok must be in 1..2^31");
    if (wait_limit_ns < 1000 || wait_limit_ns > 1000000000ull)
        return fail(ENGRAM_ERR_INVALID_ARG, "wait_limit_ns must be in [1 us, 1 s]");
    if (!h || !m || !aligned16(h) || !aligned16(m))
        return fail(ENGRAM_ERR_INVALID_ARG, "h and m must be non-NULL and 16-byte aligned");
    const Workspace L = layout(plan, n_tok);
    if (!workspace || workspace_bytes < L.total)
        return fail(ENGRAM_ERR_INVALID_ARG, "workspace too small: need %zu bytes", L.total);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint16_t *v = reinterpret_cast<uint16_t *>(ws + L.v);
    float4 *part = reinterpret_cast<float4 *>(ws + L.part);
    ProjTest test;
    test.wait_limit_ns = wait_limit_ns;
    test.stall = 1;
    return launch_proj<64>(plan, w, h, m, n_tok, v, part, static_cast<cudaStream_t>(stream), nullptr, 1, 0, false,
                           nullptr, test, false);
}

uint64_t engram_kernel_launches(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

int engram_device_status(uint32_t *status, int clear) {
    if (!status) return fail(ENGRAM_ERR_INVALID_ARG, "status is NULL");
    ENGRAM_CUDA_TRY(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
    uint32_t s = 0;
    ENGRAM_CUDA_TRY(cudaMemcpyFromSymbol(&s, g_engram_status, sizeof s), "cudaMemcpyFromSymbol");
    if (clear) {
        const uint32_t zero = 0;
        ENGRAM_CUDA_TRY(cudaMemcpyToSymbol(g_engram_status, &zero, sizeof zero), "cudaMemcpyToSymbol");
    }
    *status = s;
    return ENGRAM_OK;
}

}  // extern "C"
