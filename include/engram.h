/*
 * engram.h -- C ABI of the B200 (sm_100a) hashed n-gram embedding lookup.
 *
 * The lookup ("Engram" conditional memory / N-gram Embedding) runs six steps per token:
 *   1. remap the token id through a many-to-one vocabulary-compression table
 *      [yktysq.com "Qwen 4用上DeepSeek的Engram", 四个关键组件 #1 Tokenizer Compression];
 *   2. form the 2-gram (x_{t-1}, x_t) and 3-gram (x_{t-2}, x_{t-1}, x_t) keys and hash each with
 *      K independent heads into prime-sized tables [same page, #2 Multi-Head Hashing;
 *      zhichai.net "Qwen3.8-Flash-Next 把容量从「计算」搬到「存储」", §2.3 N-gram Embedding];
 *   3. gather one row per head and concatenate the rows into the memory vector m
 *      [yktysq #2; zhichai §2.3: 16 rows x 160 values = E_t in R^2560];
 *   4. gate: q = RMSNorm(h), k = RMSNorm(W_k m), v = W_v m, g = sigmoid(q.k / sqrt(d_h)),
 *      U = g v [yktysq #3 Context-aware Gating; zhichai §2.3 g_t, U_t];
 *   5. depthwise causal conv, kernel 4, dilation = largest order, on RMSNorm(U), then SiLU
 *      [yktysq #4; zhichai §2.3 Delta_t = U_t + SiLU(DWConv(RMSNorm(U_t)))];
 *   6. residual: out = h + Delta [zhichai §2.3 R~_t = R_t + Delta_t].
 *
 * Conventions (every entry point):
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major, dense, unless
 *     stated otherwise.  bf16 tensors are passed as their raw 16-bit patterns (uint16_t).
 *   - Pointers to bf16 / fp32 tensors must be 16-byte aligned.
 *   - The library allocates no device memory.  Scratch comes from the caller's workspace,
 *     sized by engram_workspace_size().
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and returns an int status: ENGRAM_OK or a negative ENGRAM_ERR_* code.  Arguments are
 *     validated on the host before anything is launched; on error nothing is launched and
 *     engram_last_error() describes the problem (thread-local string).
 *   - Data-dependent errors found on the device (a token id outside [0, vocab_in), a row id
 *     outside its table) never fault: the offending element reads the pad id / a zero row
 *     and a bit is set in the per-device status word, read by engram_device_status().
 *   - Calls on one stream are ordered; calls that share output or workspace buffers on
 *     different streams race.
 */
#ifndef ENGRAM_H
#define ENGRAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status codes */
#define ENGRAM_OK 0
#define ENGRAM_ERR_INVALID_ARG (-1) /* null / misaligned pointer, bad size, dim mismatch */
#define ENGRAM_ERR_UNSUPPORTED (-2) /* valid but not handled: d_e % 8, order outside 1..4, ... */
#define ENGRAM_ERR_CUDA (-3)        /* a CUDA runtime call failed; see engram_last_error() */
#define ENGRAM_ERR_TIMEOUT (-5)     /* a bounded device-side wait gave up (engram_synchronize);
                                       -4 is not used */

/* bits of the per-device status word (engram_device_status) */
#define ENGRAM_STATUS_BAD_TOKEN 0x1u    /* a token id was outside [0, vocab_in) */
#define ENGRAM_STATUS_BAD_ROW 0x2u      /* a row id was outside [0, table_rows[h]) */
#define ENGRAM_STATUS_WAIT_TIMEOUT 0x4u /* a pipeline wait inside a kernel gave up */

/* ---------------------------------------------------------------- limits */
#define ENGRAM_MAX_ORDERS 4
#define ENGRAM_MAX_TABLES 32
#define ENGRAM_MAX_HIST 3 /* largest order - 1 */
#define ENGRAM_MAX_BRANCHES 8

typedef void *engram_stream_t; /* cudaStream_t */

enum engram_table_location {
    ENGRAM_TABLES_DEVICE = 0,     /* tables resident in HBM */
    ENGRAM_TABLES_HOST_MAPPED = 1 /* tables in pinned, mapped host memory */
};

/* Element type of the n-gram tables.  The pages store bf16 rows; e4m3 rows with one
 * dequantisation scale per table halve the table bytes (and the bytes a lookup reads).  An
 * e4m3 value is dequantised into m as the bf16 nearest to decode(code) * table_scale[h]
 * (ties to even, one rounding of the exact product); decode() is the OCP FP8 E4M3 format
 * (bias 7, no infinities, codes 0x7F / 0xFF are NaN). */
enum engram_table_dtype {
    ENGRAM_TABLE_BF16 = 0,
    ENGRAM_TABLE_FP8_E4M3 = 1
};

/* Static description of one lookup layer.  Filled by the caller, checked by engram_init. */
typedef struct engram_config {
    int32_t num_orders;                   /* |O|, 1..ENGRAM_MAX_ORDERS */
    int32_t orders[ENGRAM_MAX_ORDERS];    /* n-gram orders, strictly increasing, each 1..4;
                                             the pages use {2, 3} */
    int32_t heads_per_order;              /* K >= 1; tables H = num_orders * K <= 32 */
    int64_t table_rows[ENGRAM_MAX_TABLES]; /* P_h, each a prime < 2^32, for h = oi*K + j */
    int32_t row_dim;                      /* d_e, multiple of 8 */
    int32_t hidden_dim;                   /* d_h, multiple of 64 */
    int32_t vocab_in;                     /* V: ids are in [0, V) */
    int32_t vocab_out;                    /* V': remapped ids are in [0, V') */
    int32_t pad_id;                       /* id used before a sequence start; must be V' */
    int32_t conv_kernel;                  /* depthwise conv taps, 1..8 (pages: 4) */
    int32_t conv_dilation;                /* must equal the largest order (pages) */
    int32_t table_location;               /* enum engram_table_location */
    uint64_t hash_seed;                   /* seeds the per-head hash multipliers */
    float eps;                            /* RMSNorm epsilon (> 0) */
    int32_t flags;                        /* ENGRAM_FLAG_* bits */
    int32_t table_dtype;                  /* enum engram_table_dtype */
    float table_scale[ENGRAM_MAX_TABLES]; /* FP8 tables: dequantisation scale of table h,
                                             in [2^-100, 2^100]; must be 0 for bf16 tables
                                             and beyond the H tables */
    int32_t num_branches;                 /* M, 1..ENGRAM_MAX_BRANCHES (0 reads as 1): the
                                             multi-branch form, see "Branches" below */
    int32_t reserved[4];                  /* must be zero */
} engram_config;

/* Branches [yktysq #4: with a multi-branch residual stream the branches share one embedding
 * table and one value projection, and each has its own key projection, so that every branch
 * gates the memory differently; zhichai §2.2: the residual stream is widened to 4 branches].
 * With M = num_branches > 1, for every branch b of token n:
 *   k~_b = W_k^b m, v = W_v m (shared), g_b = sigmoid(RMSNorm(h_b).RMSNorm(k~_b) / sqrt(d_h)),
 *   U_b = g_b v, Delta_b = U_b + SiLU(DWConv(RMSNorm(U_b))), out_b = h_b + Delta_b,
 * with the gains and conv weights shared by the branches.  Layouts:
 *   h, out, delta_dbg: [B*T, M, d_h] (branch b of token n is row n*M + b);
 *   w_k: [M*d_h, d_m] (branch b's key projection is rows b*d_h .. b*d_h + d_h - 1);
 *   conv_state: [B, M, state_len, d_h].
 * M = 1 is the single-branch layer, with the layouts stated at each entry point. */

/* engram_config.flags */
#define ENGRAM_FLAG_SINGLE_CTA_MMA 0x4 /* never pair CTAs for the projection's MMAs (see
                                          ENGRAM_PATH_PAIR_MMA); results are bit-identical either
                                          way.  Bits 0x1 and 0x2 are retired and rejected. */
#define ENGRAM_FLAG_ROW_ORDER_GATHER 0x8 /* gather large batches grouped by row id: in-batch
                                            dedup of the HBM reads (see ENGRAM_PATH_ROW_ORDER);
                                            results are bit-identical either way */
#define ENGRAM_FLAG_BULK_GATHER 0x10 /* gather bf16 rows (at most 8 KB) with bulk copies staged
                                        in shared memory (see ENGRAM_PATH_BULK_GATHER), in
                                        engram_gather and engram_forward; bit-identical */

/* Validated config plus derived constants.  Caller-owned, plain data: engram_init fills
 * it, every other call reads it.  Do not modify its fields. */
typedef struct engram_plan {
    engram_config cfg;
    uint64_t mult[ENGRAM_MAX_TABLES][ENGRAM_MAX_ORDERS]; /* hash multipliers a_{o,j,i} */
    int32_t num_tables;  /* H */
    int32_t mem_dim;     /* d_m = H * d_e */
    int32_t hist_len;    /* largest order - 1 */
    int32_t state_len;   /* (conv_kernel - 1) * conv_dilation */
    uint32_t magic;
    int32_t num_branches; /* M >= 1 */
    int32_t reserved[2];
} engram_plan;

/* Weights of the gate and conv (device pointers, bf16 patterns). */
typedef struct engram_weights {
    const uint16_t *w_k;     /* [M*d_h, d_m], row r = output channel r (M = 1: [d_h, d_m]) */
    const uint16_t *w_v;     /* [d_h, d_m] */
    const uint16_t *gamma_q; /* [d_h] RMSNorm gain of the query (hidden state) */
    const uint16_t *gamma_k; /* [d_h] RMSNorm gain of the key */
    const uint16_t *gamma_c; /* [d_h] RMSNorm gain of the conv input */
    const uint16_t *conv_w;  /* [d_h, conv_kernel]; tap i reads position t - i*dilation */
    const void *w_packed;    /* NULL, or [W_k ; W_v] re-laid by engram_pack_weights from these same
                                w_k / w_v; the projections then stream it instead (same results) */
} engram_weights;

/* Projection weights re-laid for streaming.  The projections read [W_k ; W_v] ((M+1)*d_h rows
 * of d_m values) in tiles of 256 rows x 64 columns; in the row-major matrices each such tile
 * is 256 separate 128-byte pieces 2*d_m bytes apart, which DRAM serves poorly when the
 * weights do not stay in L2 (decode-sized batches stream all of them every step).  The packed
 * copy stores every tile as one contiguous 32 KB block, already in the 128-byte-swizzled
 * K-major shared-memory layout the tensor cores read, so each tile is fetched by one linear
 * bulk copy.  Layout: tile (t, b) -- rows 256t..256t+255 of [W_k ; W_v], columns 64b..64b+63
 * (zero beyond d_m) -- at byte (t * k_blocks + b) * 32768, k_blocks = ceil(d_m / 64); row r of
 * the tile at r * 128; its 16-byte chunk j (columns 8j..8j+7) at chunk position j XOR (r mod 8).
 * Only for d_h % 256 == 0 (otherwise the size is 0 and the row-major weights are used). */
size_t engram_packed_weights_size(const engram_plan *plan);
int engram_pack_weights(const engram_plan *plan, const uint16_t *w_k, const uint16_t *w_v, void *packed,
                        size_t packed_bytes, engram_stream_t stream);

/* Validate `cfg` and fill `plan` (host only, no CUDA call).  Checks: orders, K, H <= 32,
 * primality of every table_rows[h] (deterministic Miller-Rabin), d_e % 8 == 0 (d_e % 16 == 0
 * for FP8 tables), d_h % 64 == 0, pad_id == vocab_out, dilation == largest order, eps > 0,
 * table scales, reserved == 0.
 * Derives the hash multipliers: a_{o,j,i} = SplitMix64(seed ^ (o<<16 ^ j<<8 ^ i)) | 1. */
int engram_init(const engram_config *cfg, engram_plan *plan);

/* Bytes of device workspace engram_forward / engram_gate_conv need for n_tok = B*T tokens
 * (remapped ids, row ids, memory vectors, fp16 value projections, per-tile partial sums;
 * each region 256-byte aligned).  0 on an invalid plan. */
size_t engram_workspace_size(const engram_plan *plan, int64_t n_tok);

/* Step 1 [yktysq #1]: out[i] = remap[ids[i]] for i < n.
 * ids, out: int32 [n] (may alias).  remap: int32 [vocab_in], values in [0, vocab_out).
 * An id outside [0, vocab_in) yields pad_id and sets ENGRAM_STATUS_BAD_TOKEN. */
int engram_remap(const engram_plan *plan, const int32_t *ids, int64_t n, const int32_t *remap,
                 int32_t *out, engram_stream_t stream);

/* Step 2 [yktysq #2; zhichai §2.3]: row ids of every n-gram head.
 * ids_remapped: int32 [B, T] in [0, vocab_out].
 * history: NULL, or int32 [B, hist_len] remapped ids preceding position 0 (oldest first);
 *          positions before both the sequence and the history use pad_id.
 * idx: uint32 [B*T, H], column h = oi*K + j (order-major, head-minor).
 * Hash: s = XOR_i (x'_{t-i} + 1) * a_{o,j,i} mod 2^64; idx = fmix64(s) mod P_h, where fmix64
 * is the MurmurHash3 64-bit finaliser. */
int engram_hash(const engram_plan *plan, const int32_t *ids_remapped, int32_t B, int32_t T,
                const int32_t *history, uint32_t *idx, engram_stream_t stream);

/* Decode bookkeeping: history <- last hist_len ids of (history ++ ids_remapped[b, :]), in
 * place.  history: int32 [B, hist_len]. */
int engram_advance_history(const engram_plan *plan, const int32_t *ids_remapped, int32_t B,
                           int32_t T, int32_t *history, engram_stream_t stream);

/* Step 3 [yktysq #2; zhichai §2.3]: m[n, h*d_e:(h+1)*d_e] = tables[h][idx[n, h], :].
 * tables: HOST array of H pointers, each to [table_rows[h], d_e] elements of
 * cfg.table_dtype (bf16 patterns, or e4m3 codes), in device memory, or in pinned mapped
 * host memory when cfg.table_location == ENGRAM_TABLES_HOST_MAPPED.
 * idx: uint32 [n_tok, H].  m: bf16 [n_tok, d_m].  bf16 bit patterns are copied unchanged;
 * e4m3 codes are dequantised (see engram_table_dtype).
 * A row id >= table_rows[h] yields a zero row and sets ENGRAM_STATUS_BAD_ROW. */
int engram_gather(const engram_plan *plan, const uint32_t *idx, const void *const *tables,
                  int64_t n_tok, uint16_t *m, engram_stream_t stream);

/* Step 3 with host-resident tables (a7) [zhichai §2.3: the row ids are known as soon as the
 * token enters the network, so the table can live in host memory and be prefetched;
 * communeify "Engram 到底是什麼": asynchronous prefetch from system RAM overlapped with
 * compute; xiaodao: host memory and the host link become the bottleneck].
 * Copies each DISTINCT row the batch needs, once, from the tables into device staging:
 *   staging[h][staged_idx[n, h], :] == tables[h][idx[n, h], :]   for every token n.
 * idx: uint32 [n_tok, H] (device).  tables: HOST array of H pointers to pinned, mapped
 * host memory (or device memory) [table_rows[h], d_e].  staging: HOST array of H device
 * pointers, each [capacity, d_e] of the tables' element type (rows are copied as stored:
 * e4m3 codes stay e4m3 and are dequantised by the gather that reads the staging).
 * staged_idx: uint32 [n_tok, H] (device, out).
 * unique_rows: uint32 [H, capacity] (device, out): the distinct row ids in increasing order.
 * n_unique: int32 [H] (device, out).  n_tok <= capacity, n_tok <= 8192.
 * The copy is done by a kernel reading the mapped host memory directly (zero-copy), many
 * CTAs wide; call it on a side stream to overlap the host-link transfer with other work.
 * engram_forward takes this path itself when cfg.table_location is
 * ENGRAM_TABLES_HOST_MAPPED and B*T <= 8192 (above that it gathers straight from the mapped
 * tables); results are bit-identical to HBM-resident tables. */
int engram_stage_rows(const engram_plan *plan, const uint32_t *idx, int64_t n_tok,
                      const void *const *tables, void *const *staging, int32_t capacity,
                      uint32_t *staged_idx, uint32_t *unique_rows, int32_t *n_unique,
                      engram_stream_t stream);

/* Steps 1-2 and the staging of engram_stage_rows in one call: idx = engram_hash of the
 * (remapped) ids -- ids, remap, B, T and history as in engram_forward and engram_hash --
 * then the batch's distinct rows staged exactly as engram_stage_rows stages them (same
 * staged_idx, unique_rows, n_unique and staging contents).  idx: uint32 [B*T, H] (device,
 * out).  Batches of at most 256 (token, table) rows (a decode step) run as ONE kernel that
 * hashes, dedups in shared memory and copies from the host tables, so the prefetch of a step
 * pays one launch; larger batches run the hash kernel, then engram_stage_rows' kernels.
 * B*T <= 8192, capacity >= B*T.  engram_forward takes the one-kernel path itself for
 * decode-sized batches on ENGRAM_TABLES_HOST_MAPPED tables. */
int engram_stage_rows_from_ids(const engram_plan *plan, const int32_t *ids, const int32_t *remap, int32_t B,
                               int32_t T, const int32_t *history, const void *const *tables, void *const *staging,
                               int32_t capacity, uint32_t *idx, uint32_t *staged_idx, uint32_t *unique_rows,
                               int32_t *n_unique, engram_stream_t stream);

/* An HBM cache of host-table rows, in front of ENGRAM_TABLES_HOST_MAPPED tables [zhichai
 * §2.3: n-gram frequencies are Zipf-like, so a few rows are read most of the time and can
 * live in fast memory while the rest stays in host memory; the pages also report that real
 * traffic shows little reuse across tokens, so the benefit depends on the stream].
 * Direct-mapped, one per table: row r lives in slot r mod slots.  All buffers are DEVICE
 * memory owned by the caller:
 *   data[h]:  [slots, d_e] elements of the table type (bf16 patterns or e4m3 codes);
 *   tags[h]:  uint32 [slots], row id + 1 of the row held in the slot, 0 = empty;
 *   claim[h]: uint32 [slots], scratch that holds 0xFFFFFFFF between calls.
 * engram_row_cache_reset() establishes that state (empty cache).  Contents are only ever
 * changed by engram_stage_rows_cached on the caller's stream; calls that share a cache must
 * be ordered on one stream. */
typedef struct engram_row_cache {
    void *data[ENGRAM_MAX_TABLES];
    uint32_t *tags[ENGRAM_MAX_TABLES];
    uint32_t *claim[ENGRAM_MAX_TABLES];
    int64_t slots; /* power of two, 1 .. 2^32 */
} engram_row_cache;

/* Empty every table's cache (tags 0, claims 0xFFFFFFFF).  Asynchronous on `stream`. */
int engram_row_cache_reset(const engram_plan *plan, const engram_row_cache *cache, engram_stream_t stream);

/* engram_stage_rows with the row cache in front of the tables: the batch's distinct rows are
 * copied into staging from the cache where it holds them and from the host tables otherwise;
 * of the rows fetched from the host, each one that maps to a slot that no other distinct row
 * of this call reads or bids for (ties: the smallest row id) is also written into the cache.
 * staging, staged_idx, unique_rows and n_unique are exactly those of engram_stage_rows (the
 * staged rows are bit-identical whatever the cache holds).
 * row_flags: uint32 [H, capacity] device scratch.  n_hits: int32 [H] device, ACCUMULATES the
 * number of distinct rows served from the cache (zero it to count one call). */
int engram_stage_rows_cached(const engram_plan *plan, const uint32_t *idx, int64_t n_tok,
                             const void *const *tables, const engram_row_cache *cache,
                             void *const *staging, int32_t capacity, uint32_t *staged_idx,
                             uint32_t *unique_rows, int32_t *n_unique, uint32_t *row_flags,
                             int32_t *n_hits, engram_stream_t stream);

/* engram_gather over tables that all hold `rows` rows (e.g. the staging buffers filled by
 * engram_stage_rows, with staged_idx as idx).  Same layout and error behaviour as
 * engram_gather, with `rows` as every table's bound. */
int engram_gather_bounded(const engram_plan *plan, const uint32_t *idx, const void *const *tables,
                          int64_t n_tok, int64_t rows, uint16_t *m, engram_stream_t stream);

/* Steps 4-6 [yktysq #3, #4; zhichai §2.3]: gate, conv, residual for B sequences of T tokens.
 * h: bf16 [B*T, d_h] hidden states.  m: bf16 [B*T, d_m] memory vectors.
 * conv_state: NULL for prefill (zero left padding), or bf16 [B, state_len, d_h] conv inputs
 *             of the state_len positions before this call, oldest first; updated in place.
 *             With a state, T <= 16384.
 * out: bf16 [B*T, d_h] = bf16_rne(h + Delta).  May not alias h.
 * delta_dbg: NULL, or fp32 [B*T, d_h] receiving Delta before the residual add.
 * The projections k~ = W_k m and v = W_v m run on the tcgen05 tensor cores (bf16 inputs,
 * fp32 accumulation; v is kept in fp16 between the projection and the gate, its norm is
 * taken in fp32); norms, gate and conv run in fp32.
 * workspace: >= engram_workspace_size(plan, B*T) bytes, 256-byte aligned. */
int engram_gate_conv(const engram_plan *plan, const engram_weights *w, const uint16_t *h,
                     const uint16_t *m, int32_t B, int32_t T, uint16_t *conv_state,
                     uint16_t *out, float *delta_dbg, void *workspace, size_t workspace_bytes,
                     engram_stream_t stream);

/* Steps 1-6 chained: remap + hash (one kernel), gather, projections with the gate's partial
 * reductions fused in their epilogue, then gate + conv + residual, then the history update
 * when `history` is given.  Kernels per call (engram_forward_path tells which apply): prefill
 * batches launch remap + hash, gather, projection, gate scalars and the streaming gate + conv
 * kernel (5), and with ENGRAM_PATH_ROW_ORDER three more ahead of the gather (count rows per
 * bucket, scan, list; 8); batches of at most 16,384 (token, table) rows on HBM-resident tables fuse
 * remap + hash + gather into one kernel; decode-sized batches on host-mapped tables fuse
 * remap + hash + dedup + staging into one; one-token decode steps whose projection splits K
 * finish the split sums, gate, conv and the history update in one kernel (lookup,
 * projection, that kernel: 3).
 * engram_kernel_launches() counts them.
 * ids: int32 [B, T] raw token ids.  remap: int32 [vocab_in], or NULL when ids are already
 * in the compressed vocabulary.  history / conv_state: NULL for prefill, or the decode state
 * (read, then updated in place).  Other arguments as in the steps above.
 * stage_events: NULL, or an array of ENGRAM_FORWARD_STAGES + 1 cudaEvent_t recorded on
 * `stream` before each stage and after the last (a profiling hook; no effect on results).
 * Under stream capture they are recorded as external event nodes, so a replayed graph can
 * be timed per stage.
 * CUDA graphs: after one eager call on a device (which resolves the tensor-map encoder and
 * sets kernel attributes), engram_forward / engram_gate_conv may be captured and replayed. */
#define ENGRAM_FORWARD_STAGES 4 /* hash, gather, projections, gate+conv */
int engram_forward(const engram_plan *plan, const engram_weights *w,
                   const void *const *tables, const int32_t *ids, const int32_t *remap,
                   int32_t B, int32_t T, int32_t *history, uint16_t *conv_state,
                   const uint16_t *h, uint16_t *out, float *delta_dbg, void *workspace,
                   size_t workspace_bytes, engram_stream_t stream, void *const *stage_events);

/* Steps 4-6 like engram_gate_conv, for callers that cannot allocate device memory: no
 * workspace argument.  This entry point has no counterpart in the pages; it exists for
 * hosts that hand an operator only its inputs and outputs and own every device allocation
 * themselves (plugin and custom-op interfaces of inference servers, runtimes with a fixed
 * memory budget, code paths where the device-wide synchronisation of cudaMalloc/cudaFree is
 * not acceptable).  Its scratch (fp16 value projections and per-tile partial sums) lives in
 * a statically sized array in the library's device data, ENGRAM_NOALLOC_SCRATCH_BYTES per
 * GPU, which every GPU that loads the library holds until the process exits.
 *  - Sizes: the call needs 2*B*T*d_h bytes for v (fp16) plus 16*B*T*(2*d_h/BN) bytes of
 *    partial sums (BN = 64, 128 or 256, the projection tile width), each rounded up to 256; a
 *    request that does not fit returns ENGRAM_ERR_UNSUPPORTED and launches nothing.  At
 *    d_h = 2560 that is about 5,000 tokens per call.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress, a host-side
 *    lookup) with the caller's device current; the first call on a device may load the
 *    library's device code there, so make it before any stream capture.  No call allocates
 *    or frees memory.
 *  - Every call on a device shares the one array and leaves its contents behind.  No part of
 *    it needs clearing: each element a call reads is written earlier in the same call.
 *    Calls that overlap on the GPU (other streams, other host threads) race on the array
 *    and must be serialised by the caller.
 * Other arguments, layouts and results are those of engram_gate_conv. */
#define ENGRAM_NOALLOC_SCRATCH_BYTES (32u << 20)
int engram_gate_conv_noalloc(const engram_plan *plan, const engram_weights *w, const uint16_t *h,
                             const uint16_t *m, int32_t B, int32_t T, uint16_t *conv_state,
                             uint16_t *out, float *delta_dbg, engram_stream_t stream);

/* The kernels engram_forward runs for a batch of B sequences of T tokens, as ENGRAM_PATH_*
 * bits in *path (host only, no CUDA call).  A diagnostic for tests and benchmarks:
 *   FUSED_LOOKUP   remap + hash + gather in one kernel (at most 16,384 (token, table) rows,
 *                  HBM-resident tables); m is written by it;
 *   STAGED_ROWS    host-mapped tables: the batch's distinct rows are staged into HBM first;
 *   SPLIT_K        the projection splits K across CTAs (decode-sized batches);
 *   PAIR_MMA       the projection runs on pairs of CTAs (a thread-block cluster of two), each
 *                  tensor-core MMA spanning both: 256-token x 256-channel tiles, each CTA
 *                  holding half of every operand tile (d_h % 256 == 0 and
 *                  ENGRAM_FLAG_SINGLE_CTA_MMA not set; whole-K tiles when there are at least
 *                  148 of them, K split across pairs when fewer than 74 would leave pairs
 *                  idle); the workspace's partial sums then have (M+1)*d_h/256 columns per
 *                  token;
 *   ROW_ORDER      the gather walks the batch's (token, table) rows grouped by row id (buckets
 *                  of neighbouring rows, table by table) instead of in token order, so that
 *                  every repeat of a row in the batch follows its first read while the row is
 *                  still in L2: DRAM reads each distinct row about once (in-batch dedup of the
 *                  HBM reads; m is bit-identical).  ENGRAM_FLAG_ROW_ORDER_GATHER set,
 *                  HBM-resident tables, the hash + gather path, at least 65,536 rows per
 *                  call.  Opt-in: m is then written in row order, as scattered slices, and on
 *                  B200 that costs more write bandwidth than the saved reads;
 *   BULK_GATHER    the gather (in token order) moves each row global -> shared -> global with
 *                  one bulk copy each way (TMA engine; a ring of rows per one-warp CTA, each
 *                  CTA filling one contiguous stretch of m) instead of 16-byte register copies.
 *                  ENGRAM_FLAG_BULK_GATHER set, bf16 rows of at most 8 KB, the hash + gather
 *                  path.  Opt-in: on B200 the register gather keeps more bytes in flight per
 *                  SM and is faster.
 * Otherwise the hash kernel writes the row ids and the gather kernel writes m in token order. */
#define ENGRAM_PATH_FUSED_LOOKUP 0x1u
#define ENGRAM_PATH_STAGED_ROWS 0x2u
#define ENGRAM_PATH_SPLIT_K 0x8u
#define ENGRAM_PATH_PAIR_MMA 0x10u
#define ENGRAM_PATH_ROW_ORDER 0x20u
#define ENGRAM_PATH_BULK_GATHER 0x40u
int engram_forward_path(const engram_plan *plan, int32_t B, int32_t T, uint32_t *path);

/* Wait for `stream` and report what the device found: ENGRAM_ERR_TIMEOUT if a pipeline wait
 * inside one of this library's kernels on the current device gave up since the status word
 * was last cleared (the kernel then abandoned its work and returned, so its outputs are
 * undefined, but the device stays usable); ENGRAM_ERR_CUDA if the stream reports a CUDA
 * error; ENGRAM_OK otherwise.  Does not clear the status word (engram_device_status does). */
int engram_synchronize(engram_stream_t stream);

/* Self-test of the bounded waits (no counterpart in the pages: it checks this library's
 * failure handling).  Runs the projection kernel of engram_gate_conv over n_tok tokens with
 * its producer stalled -- no tile is ever loaded -- and every pipeline wait bounded by
 * wait_limit_ns (1 us .. 1 s) instead of the built-in 2 s.  Each CTA's first wait for a stage
 * runs out, raises ENGRAM_STATUS_WAIT_TIMEOUT, and the CTA unwinds: its other roles stop
 * waiting, its tensor memory is released and it exits.  engram_synchronize(stream) then
 * returns ENGRAM_ERR_TIMEOUT.  Arguments as engram_gate_conv (h, m: bf16 [n_tok, d_h] and
 * [n_tok, d_m], never read; workspace >= engram_workspace_size(plan, n_tok)).  Clear the
 * status word afterwards with engram_device_status(&s, 1). */
int engram_selftest_wait_timeout(const engram_plan *plan, const engram_weights *w, const uint16_t *h,
                                 const uint16_t *m, int64_t n_tok, void *workspace, size_t workspace_bytes,
                                 uint64_t wait_limit_ns, engram_stream_t stream);

/* Read (and optionally clear) the status word of the current device.  Synchronises the
 * device.  *status receives the OR of ENGRAM_STATUS_* bits since the last clear. */
int engram_device_status(uint32_t *status, int clear);

/* Description of the last error on this thread ("" if none). */
const char *engram_last_error(void);

/* Library version, e.g. "0.1.0". */
const char *engram_version(void);

/* Number of kernels this library has launched in this process so far (all host threads and
 * devices; a launch is counted once the CUDA runtime has accepted it, whether it runs eagerly
 * or is recorded into a CUDA graph being captured).  A diagnostic: read it before and after
 * a call to learn how many kernels that call launches. */
uint64_t engram_kernel_launches(void);

/* sizeof() of a public struct, by name ("engram_config", "engram_plan", "engram_weights",
 * "engram_row_cache"),
 * so that bindings in other languages can check their layout; 0 for an unknown name. */
size_t engram_sizeof(const char *type_name);

#ifdef __cplusplus
}
#endif
#endif /* ENGRAM_H */
