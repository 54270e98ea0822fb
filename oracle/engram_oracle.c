/*
 * CPU oracle for the hashed n-gram embedding lookup ("Engram" / N-gram Embedding).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously-correct statement of
 * what the lookup computes.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline may load it.  It shares no code, header, table or constant generator with the
 * CUDA library; the two are compared, never combined.
 *
 * Arithmetic: integers for remap/hash/gather (bit-exact), IEEE double for everything
 * floating point, one final round-to-nearest-even to bf16 for the layer output.
 * bf16 inputs are passed as their raw 16-bit patterns and widened exactly.
 *
 * Sources (web pages, cited by title and section):
 *   [yktysq]   "Qwen 4用上DeepSeek的Engram！125B MoE一张4090能跑不用量化" (yktysq.com),
 *              section "Engram 的设计有四个关键组件" (components 1-4).
 *   [zhichai]  "Qwen3.8-Flash-Next 把容量从「计算」搬到「存储」" (zhichai.net),
 *              section 2.3 "Embedding：N-gram Embedding".
 *   [zjcp]     "Engram 真能让 1T 参数模型在本地跑？" (zjcp.cc), section 一 "Engram 到底是什么".
 *   [communeify] "Qwen3.8-Flash-Next ... Engram" (communeify.com), "Engram 到底是什麼？".
 * Where the pages leave a step open, the reading taken is stated at the function.
 *
 * Parity pins: every function here is checked by tests that do not re-type its formula
 * (published test vectors, closed forms, brute force, invariants).  No function here is
 * "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>

#define ORACLE_MAX_ORDERS 4
#define ORACLE_MAX_HEADS 64

/* ------------------------------------------------------------------------------------------
 * bf16 <-> double
 * ------------------------------------------------------------------------------------------ */

/* Exact widening: a bf16 pattern is the upper half of an IEEE binary32 pattern. */
double oracle_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a finite double to the nearest bf16 (8 significant bits), ties to even, in ONE
 * rounding step (no detour through binary32, which would round twice).  The result is
 * returned as its 16-bit pattern.  Values below the binary32 normal range are rounded on
 * the subnormal grid 2^-133; values past the largest bf16 saturate to infinity. */
uint16_t oracle_double_to_bf16(double x)
{
    if (x == 0.0) return signbit(x) ? 0x8000u : 0x0000u;
    int sign = x < 0.0;
    double a = fabs(x);
    int e = ilogb(a);              /* a in [2^e, 2^(e+1)) */
    if (e < -126) e = -126;        /* subnormal grid */
    double q = ldexp(1.0, e - 7);  /* spacing of bf16 values in this binade */
    double r = a / q;              /* exact: division by a power of two */
    double fl = floor(r);
    double frac = r - fl;          /* exact */
    double n;
    if (frac > 0.5) n = fl + 1.0;
    else if (frac < 0.5) n = fl;
    else n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double y = n * q;              /* exact, representable in binary32 */
    uint16_t out;
    if (y > 3.3895313892515355e38) {
        out = 0x7f80u;             /* +inf */
    } else {
        float f = (float)y;        /* exact */
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        out = (uint16_t)(u >> 16);
    }
    return (uint16_t)(out | (sign ? 0x8000u : 0u));
}

/* ------------------------------------------------------------------------------------------
 * FP8 (e4m3) tables.  The pages store bf16 rows; the e4m3 variant with one dequantisation
 * scale per table is an extension.  Reading taken: the value gathered into m is the bf16
 * nearest to decode(code) * scale (ties to even), rounded once from the exact product.
 * ------------------------------------------------------------------------------------------ */

/* Value of an e4m3 code from the OCP 8-bit floating point (FP8 E4M3) definition: bit 7 sign,
 * bits 6-3 exponent with bias 7, bits 2-0 mantissa; exponent field 0 encodes the subnormals
 * m * 2^-9; S.1111.111 is NaN and there are no infinities. */
double oracle_e4m3_to_double(uint8_t code)
{
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* One dequantised element: a 4-bit significand times the 24-bit significand of `scale` is
 * exact in double, so oracle_double_to_bf16 rounds the true product once.  NaN codes give the
 * quiet NaN pattern 0x7FC0 (with the code's sign). */
uint16_t oracle_dequant_e4m3(uint8_t code, float scale)
{
    const double v = oracle_e4m3_to_double(code);
    if (isnan(v)) return (uint16_t)(0x7FC0u | ((code & 0x80u) ? 0x8000u : 0u));
    return oracle_double_to_bf16(v * (double)scale);
}

/* A whole e4m3 table (n elements) to bf16 patterns. */
void oracle_dequant_table(const uint8_t *codes, int64_t n, float scale, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_dequant_e4m3(codes[i], scale);
}

/* ------------------------------------------------------------------------------------------
 * Hash primitives (reading of the pages: they fix only "deterministic hash", "K independent
 * heads per order" and "prime-sized tables" [yktysq, component 2; zhichai §2.3].  The hash
 * taken here is: multiply-xor of the gram's ids with per-(order, head, position) odd 64-bit
 * multipliers, then the 64-bit finaliser of MurmurHash3 (Austin Appleby, public domain),
 * then reduction modulo the table's prime.  The multipliers are the first output of a
 * SplitMix64 generator (Sebastiano Vigna, public domain) seeded per (order, head, position).)
 * ------------------------------------------------------------------------------------------ */

/* First output of a SplitMix64 generator whose state is `state`: the state advances by the
 * golden-ratio increment, then the output mix is applied. */
uint64_t oracle_splitmix64(uint64_t state)
{
    uint64_t z = state + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* MurmurHash3 64-bit finaliser ("fmix64"). */
uint64_t oracle_fmix64(uint64_t k)
{
    k ^= k >> 33;
    k *= 0xFF51AFD7ED558CCDull;
    k ^= k >> 33;
    k *= 0xC4CEB9FE1A85EC53ull;
    k ^= k >> 33;
    return k;
}

/* Multiplier for gram position i (0 = current token, 1 = previous, ...) of head j of
 * order o.  Forced odd so that it is invertible modulo 2^64. */
uint64_t oracle_hash_multiplier(uint64_t seed, int order, int head, int pos)
{
    uint64_t key = seed ^ (((uint64_t)order << 16) ^ ((uint64_t)head << 8) ^ (uint64_t)pos);
    return oracle_splitmix64(key) | 1ull;
}

/* Hash of one gram.  gram[0] is the CURRENT token x'_t, gram[i] is x'_{t-i}.
 * s = XOR over i of (x'_{t-i} + 1) * a_{o,j,i}  (mod 2^64);  idx = fmix64(s) mod P. */
uint32_t oracle_hash_gram(const int32_t *gram, int order, int head, uint64_t seed, uint64_t prime)
{
    uint64_t s = 0;
    for (int i = 0; i < order; ++i) {
        uint64_t x = (uint64_t)(int64_t)gram[i] + 1ull;
        s ^= x * oracle_hash_multiplier(seed, order, head, i);
    }
    return (uint32_t)(oracle_fmix64(s) % prime);
}

/* ------------------------------------------------------------------------------------------
 * Step 1: tokenizer-compression remap [yktysq, component 1 "Tokenizer Compression"]:
 * semantically equivalent ids are mapped to one id by a many-to-one table.
 * Returns 0, or -1 if an id lies outside [0, vocab_in).
 * ------------------------------------------------------------------------------------------ */
int oracle_remap(const int32_t *ids, int64_t n, const int32_t *remap, int32_t vocab_in, int32_t *out)
{
    for (int64_t i = 0; i < n; ++i) {
        int32_t x = ids[i];
        if (x < 0 || x >= vocab_in) return -1;
        out[i] = remap[x];
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * Step 2: n-gram keys and multi-head hashing [yktysq, component 2; zhichai §2.3: for token
 * x_t, 2-gram heads use (x_{t-1}, x_t), 3-gram heads use (x_{t-2}, x_{t-1}, x_t); K heads per
 * order; one row id per head].
 *
 * xr       remapped ids, [B, T] row-major.
 * history  NULL, or [B, hist_len] remapped ids that precede position 0 of each sequence,
 *          oldest first (history[b][hist_len-1] is x'_{-1}).  Positions before both the
 *          sequence and the history read pad_id (reading: grams never cross a sequence
 *          start; the pad id V' is reserved for it).
 * idx      output, [B*T, H] with H = num_orders*K, column h = order_index*K + head
 *          (order-major, head-minor: the 2-gram heads come first, as listed on the page).
 * primes   P_h for each of the H tables.
 * ------------------------------------------------------------------------------------------ */
void oracle_hash(const int32_t *xr, int32_t B, int32_t T,
                 const int32_t *history, int32_t hist_len, int32_t pad_id,
                 int32_t num_orders, const int32_t *orders, int32_t K,
                 const uint64_t *primes, uint64_t seed, uint32_t *idx)
{
    int H = num_orders * K;
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t t = 0; t < T; ++t) {
            for (int oi = 0; oi < num_orders; ++oi) {
                int o = orders[oi];
                int32_t gram[ORACLE_MAX_ORDERS + 4];
                for (int i = 0; i < o; ++i) {
                    int32_t p = t - i;
                    int32_t x;
                    if (p >= 0) x = xr[(int64_t)b * T + p];
                    else if (history != NULL && -p <= hist_len) x = history[(int64_t)b * hist_len + hist_len + p];
                    else x = pad_id;
                    gram[i] = x;
                }
                for (int j = 0; j < K; ++j) {
                    int h = oi * K + j;
                    idx[((int64_t)b * T + t) * H + h] = oracle_hash_gram(gram, o, j, seed, primes[h]);
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------------------------
 * Step 3: row gather and concatenation [yktysq, component 2: "all retrieved vectors are
 * concatenated into one memory vector"; zhichai §2.3: 16 rows of 160 values give E_t in
 * R^2560].  m[n, h*d_e + c] = table_h[idx[n, h], c].  Bit patterns are copied unchanged.
 * ------------------------------------------------------------------------------------------ */
void oracle_gather(const uint32_t *idx, int64_t n_tok, int32_t H,
                   const uint16_t *const *tables, int32_t d_e, uint16_t *m)
{
    for (int64_t n = 0; n < n_tok; ++n)
        for (int32_t h = 0; h < H; ++h) {
            const uint16_t *row = tables[h] + (int64_t)idx[n * H + h] * d_e;
            for (int32_t c = 0; c < d_e; ++c)
                m[(n * H + h) * d_e + c] = row[c];
        }
}

/* Step 3 over e4m3 tables: m[n, h*d_e + c] = dequant(table_h[idx[n, h], c], scale[h]). */
void oracle_gather_e4m3(const uint32_t *idx, int64_t n_tok, int32_t H, const uint8_t *const *tables,
                        const float *scale, int32_t d_e, uint16_t *m)
{
    for (int64_t n = 0; n < n_tok; ++n)
        for (int32_t h = 0; h < H; ++h) {
            const uint8_t *row = tables[h] + (int64_t)idx[n * H + h] * d_e;
            for (int32_t c = 0; c < d_e; ++c)
                m[(n * H + h) * d_e + c] = oracle_dequant_e4m3(row[c], scale[h]);
        }
}

/* RMSNorm of a vector: x / sqrt(mean(x^2) + eps) * gamma. */
static void rmsnorm(const double *x, const uint16_t *gamma, int d, double eps, double *y)
{
    double ss = 0.0;
    for (int c = 0; c < d; ++c) ss += x[c] * x[c];
    double inv = 1.0 / sqrt(ss / d + eps);
    for (int c = 0; c < d; ++c) y[c] = x[c] * inv * oracle_bf16_to_double(gamma[c]);
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* ------------------------------------------------------------------------------------------
 * Steps 4-6: context-aware gating, depthwise causal convolution and residual add.
 *
 * Gating [yktysq, component 3: the hidden state is the query, the retrieved memory gives
 * key and value; after RMSNorm a scaled dot product gives one scalar gate that goes to zero
 * when the memory contradicts the context; zhichai §2.3: g_t = Gate(Norm(Q_t), Norm(K_t)),
 * U_t = g_t * V_t]:
 *     k~ = W_k m,  v = W_v m                      (W_* stored [d_h, d_m], row = output)
 *     q  = RMSNorm(h) * gamma_q,  k = RMSNorm(k~) * gamma_k
 *     g  = sigmoid(q . k / sqrt(d_h)),  U = g v
 * Convolution and residual [yktysq, component 4: depthwise causal conv, kernel 4, dilation
 * equal to the largest n-gram order; zhichai §2.3: Delta_t = U_t + SiLU(DWConv(RMSNorm(U_t))),
 * then R~_t = R_t + Delta_t]:
 *     u = RMSNorm(U) * gamma_c
 *     c_t[ch] = sum_{i<ksize} w[ch][i] * u_{t - i*dil}[ch]    (tap 0 = current position,
 *               no bias; positions before the sequence read 0, or conv_state in decode)
 *     Delta = U + c * sigmoid(c),   out = bf16_rne(h + Delta)
 *
 * conv_state  NULL (prefill: zero left padding), or [B, (ksize-1)*dil, d_h] bf16 holding the
 *             conv inputs u of the positions just before this call, oldest first.
 * state_out   NULL, or [B, (ksize-1)*dil, d_h] bf16: the state after this call (the last
 *             (ksize-1)*dil conv inputs of state ++ this call), each rounded to bf16.
 * delta, gate NULL or outputs [B*T, d_h] / [B*T] in double.
 * Returns 0, or -1 on allocation failure.
 * ------------------------------------------------------------------------------------------ */
int oracle_gate_conv(const uint16_t *h, const uint16_t *m, int32_t d_m, int32_t d_h,
                     const uint16_t *Wk, const uint16_t *Wv,
                     const uint16_t *gamma_q, const uint16_t *gamma_k, const uint16_t *gamma_c,
                     const uint16_t *conv_w, int32_t ksize, int32_t dil,
                     int32_t B, int32_t T, double eps,
                     const uint16_t *conv_state, uint16_t *state_out,
                     uint16_t *out, double *delta, double *gate)
{
    int64_t n_tok = (int64_t)B * T;
    int32_t S = (ksize - 1) * dil;
    double *U = (double *)malloc(sizeof(double) * (size_t)n_tok * d_h);
    double *u = (double *)malloc(sizeof(double) * (size_t)n_tok * d_h);
    double *mv = (double *)malloc(sizeof(double) * (size_t)d_m);
    double *hv = (double *)malloc(sizeof(double) * (size_t)d_h);
    double *kt = (double *)malloc(sizeof(double) * (size_t)d_h);
    double *vv = (double *)malloc(sizeof(double) * (size_t)d_h);
    double *q = (double *)malloc(sizeof(double) * (size_t)d_h);
    double *k = (double *)malloc(sizeof(double) * (size_t)d_h);
    if (!U || !u || !mv || !hv || !kt || !vv || !q || !k) {
        free(U); free(u); free(mv); free(hv); free(kt); free(vv); free(q); free(k);
        return -1;
    }
    for (int64_t n = 0; n < n_tok; ++n) {
        for (int32_t c = 0; c < d_m; ++c) mv[c] = oracle_bf16_to_double(m[n * d_m + c]);
        for (int32_t c = 0; c < d_h; ++c) hv[c] = oracle_bf16_to_double(h[n * d_h + c]);
        /* projections */
        for (int32_t r = 0; r < d_h; ++r) {
            double sk = 0.0, sv = 0.0;
            for (int32_t c = 0; c < d_m; ++c) {
                sk += oracle_bf16_to_double(Wk[(int64_t)r * d_m + c]) * mv[c];
                sv += oracle_bf16_to_double(Wv[(int64_t)r * d_m + c]) * mv[c];
            }
            kt[r] = sk;
            vv[r] = sv;
        }
        /* gate */
        rmsnorm(hv, gamma_q, d_h, eps, q);
        rmsnorm(kt, gamma_k, d_h, eps, k);
        double dot = 0.0;
        for (int32_t c = 0; c < d_h; ++c) dot += q[c] * k[c];
        double g = sigmoid(dot / sqrt((double)d_h));
        if (gate) gate[n] = g;
        for (int32_t c = 0; c < d_h; ++c) U[n * d_h + c] = g * vv[c];
        rmsnorm(U + n * d_h, gamma_c, d_h, eps, u + n * d_h);
    }
    /* depthwise causal conv + SiLU + residual */
    for (int32_t b = 0; b < B; ++b)
        for (int32_t t = 0; t < T; ++t) {
            int64_t n = (int64_t)b * T + t;
            for (int32_t c = 0; c < d_h; ++c) {
                double acc = 0.0;
                for (int32_t i = 0; i < ksize; ++i) {
                    int32_t p = t - i * dil;
                    double x;
                    if (p >= 0) x = u[((int64_t)b * T + p) * d_h + c];
                    else if (conv_state != NULL && -p <= S)
                        x = oracle_bf16_to_double(conv_state[((int64_t)b * S + S + p) * d_h + c]);
                    else x = 0.0;
                    acc += oracle_bf16_to_double(conv_w[(int64_t)c * ksize + i]) * x;
                }
                double dlt = U[n * d_h + c] + acc * sigmoid(acc);
                if (delta) delta[n * d_h + c] = dlt;
                out[n * d_h + c] = oracle_double_to_bf16(oracle_bf16_to_double(h[n * d_h + c]) + dlt);
            }
        }
    if (state_out != NULL) {
        for (int32_t b = 0; b < B; ++b)
            for (int32_t s = 0; s < S; ++s) {
                /* state slot s holds the conv input at position T - S + s */
                int32_t p = T - S + s;
                for (int32_t c = 0; c < d_h; ++c) {
                    uint16_t v;
                    if (p >= 0) v = oracle_double_to_bf16(u[((int64_t)b * T + p) * d_h + c]);
                    else if (conv_state != NULL) v = conv_state[((int64_t)b * S + S + p) * d_h + c];
                    else v = 0;
                    state_out[((int64_t)b * S + s) * d_h + c] = v;
                }
            }
    }
    free(U); free(u); free(mv); free(hv); free(kt); free(vv); free(q); free(k);
    return 0;
}

/* Decode bookkeeping: the hash history after this call is the last hist_len remapped ids of
 * (history ++ this call's ids) for each sequence; missing entries are pad_id.  This is what
 * makes the row ids of the next token computable before it is processed [zhichai §2.3,
 * "确定性寻址": the n-gram row ids are known as soon as the token enters the network]. */
void oracle_advance_history(const int32_t *xr, int32_t B, int32_t T,
                            const int32_t *history, int32_t hist_len, int32_t pad_id,
                            int32_t *history_out)
{
    for (int32_t b = 0; b < B; ++b)
        for (int32_t s = 0; s < hist_len; ++s) {
            int32_t p = T - hist_len + s;
            int32_t x;
            if (p >= 0) x = xr[(int64_t)b * T + p];
            else if (history != NULL) x = history[(int64_t)b * hist_len + hist_len + p];
            else x = pad_id;
            history_out[(int64_t)b * hist_len + s] = x;
        }
}

/* The whole lookup, steps 1-6 in order: remap, hash, gather, gate, conv, residual.
 * Returns 0, -1 on a bad id, -2 on allocation failure. */
int oracle_forward(const int32_t *ids, int32_t B, int32_t T,
                   const int32_t *remap, int32_t vocab_in,
                   const int32_t *history, int32_t hist_len, int32_t pad_id,
                   int32_t num_orders, const int32_t *orders, int32_t K,
                   const uint64_t *primes, uint64_t seed,
                   const uint16_t *const *tables, int32_t d_e,
                   const uint16_t *h, int32_t d_h,
                   const uint16_t *Wk, const uint16_t *Wv,
                   const uint16_t *gamma_q, const uint16_t *gamma_k, const uint16_t *gamma_c,
                   const uint16_t *conv_w, int32_t ksize, int32_t dil, double eps,
                   const uint16_t *conv_state, uint16_t *state_out, int32_t *history_out,
                   uint16_t *out, double *delta, double *gate, uint32_t *idx_out)
{
    int64_t n_tok = (int64_t)B * T;
    int32_t H = num_orders * K;
    int32_t d_m = H * d_e;
    int32_t *xr = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_tok > 0 ? n_tok : 1));
    uint32_t *idx = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(n_tok > 0 ? n_tok * H : 1));
    uint16_t *m = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(n_tok > 0 ? n_tok * d_m : 1));
    if (!xr || !idx || !m) { free(xr); free(idx); free(m); return -2; }
    int rc = oracle_remap(ids, n_tok, remap, vocab_in, xr);
    if (rc != 0) { free(xr); free(idx); free(m); return -1; }
    oracle_hash(xr, B, T, history, hist_len, pad_id, num_orders, orders, K, primes, seed, idx);
    oracle_gather(idx, n_tok, H, tables, d_e, m);
    rc = oracle_gate_conv(h, m, d_m, d_h, Wk, Wv, gamma_q, gamma_k, gamma_c, conv_w, ksize, dil,
                          B, T, eps, conv_state, state_out, out, delta, gate);
    if (history_out != NULL)
        oracle_advance_history(xr, B, T, history, hist_len, pad_id, history_out);
    if (idx_out != NULL) memcpy(idx_out, idx, sizeof(uint32_t) * (size_t)(n_tok * H));
    free(xr); free(idx); free(m);
    return rc == 0 ? 0 : -2;
}
