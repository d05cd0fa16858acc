/*
 * oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar C reference of one quantised Mixture-of-Experts
 * decoder layer.  Only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load it; the product path never does.  It shares
 * no code, header, table or helper with the CUDA library.
 *
 * What it follows (pages by title and section):
 *   [HN]  "Show HN: 遅いコンピュータで GLM 5.2 を実行する" (ja.news.hada.io),
 *         section "実装済みの主な機能" (implemented features):
 *           - router bullet: DeepSeek-V3-style sigmoid router, noaux_tc,
 *             routed_scaling_factor, shared expert;
 *           - integer-dot bullet: Q8_0-style int8 activations, integer dot;
 *           - quantisation bullet: int8 / packed int4 / packed int2 weights,
 *             per-row scales, dequantised on use;
 *           - batch-union bullet: each distinct expert of a batch is applied
 *             to every position routed to it (this does not change results:
 *             every (token, expert) pair below is computed the same way).
 *   [DT]  "Comment exécuter un réseau de neurones de 744 milliards de
 *         paramètres sur un ordinateur ordinaire" (devtrends.cc), section
 *         "Comment fonctionne le moteur": an expert is three matrices
 *         (gate, up, down) read together.
 *
 * The pages print no formula.  Where they are silent this file takes the
 * plainest reading and says so at the function.  Numerics:
 *   - Q8_0 and weight quantisation decide codes in fp32 with IEEE division
 *     and round-half-to-even (rintf in the default rounding mode);
 *   - integer block sums are exact int32;
 *   - block partials S_b * d_b are exact in fp64 and summed in fp64;
 *   - router logits, sigmoid, group scores and selection are fp64;
 *   - SwiGLU is evaluated in fp64 from fp32 g, u;
 *   - the combine is accumulated in fp64, shared expert first.
 * Build with -O2 -fno-fast-math -ffp-contract=off (no FMA contraction).
 *
 * Parity pins (tests/test_oracle_pins.py): hand-picked quantiser values,
 * pack/unpack identities, exact rational dots, brute-force routing
 * enumeration, routing invariants, the dense-mixture special case, an exact
 * single-expert case, and SwiGLU values and a whole unsaturated expert
 * derived by exact arithmetic (tests/golden/make_swiglu.py).  Layer-level
 * values are not printed by the pages.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define QBLK 32

/* ------------------------------------------------------------------------ */
/* Q8_0 activation quantisation.  [HN] integer-dot bullet names Q8_0-style
 * int8 activations: blocks of 32 along the row, one scale per block.
 * Reading: d = amax / 127 rounded to fp32 and stored in fp32;
 * q = clamp(round_half_even(x / d), -127, 127); amax == 0 gives d = 0, q = 0. */
void oracle_quant_q8(const float *x, int64_t rows, int64_t len, int8_t *q, float *d)
{
    const int64_t nb = len / QBLK;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float *xb = x + r * len + b * QBLK;
            float amax = 0.0f;
            for (int i = 0; i < QBLK; ++i) {
                float a = fabsf(xb[i]);
                if (a > amax) amax = a;
            }
            float db = amax / 127.0f;
            d[r * nb + b] = db;
            for (int i = 0; i < QBLK; ++i) {
                float v = 0.0f;
                if (db != 0.0f) v = rintf(xb[i] / db);
                if (v > 127.0f) v = 127.0f;
                if (v < -127.0f) v = -127.0f;
                q[r * len + b * QBLK + i] = (int8_t)v;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Per-row weight quantisation.  [HN] quantisation bullet: int8, packed int4,
 * packed int2, one scale per row.  Reading:
 *   int8: scale = amax/127, codes clamp to [-127, 127], one per byte;
 *   int4: scale = amax/7,   codes clamp to [-8, 7],  two per byte,
 *         element 2j in the low nibble of byte j;
 *   int2: scale = amax/2,   codes clamp to [-2, 1],  four per byte,
 *         element 4j+i in bits 2i..2i+1 of byte j (so +amax saturates to +1).
 * Codes are two's complement inside their field. */
static int qmax_of(int bits) { return bits == 8 ? 127 : bits == 4 ? 7 : 2; }
static int qlo_of(int bits) { return bits == 8 ? -127 : bits == 4 ? -8 : -2; }
static int qhi_of(int bits) { return bits == 8 ? 127 : bits == 4 ? 7 : 1; }

int64_t oracle_row_bytes(int64_t K, int bits) { return K * bits / 8; }

int oracle_quant_weights(const float *w, int64_t rows, int64_t K, int bits,
                         uint8_t *codes, float *scales)
{
    if (bits != 8 && bits != 4 && bits != 2) return -1;
    if ((K * bits) % 8 != 0) return -1;
    const int64_t rb = oracle_row_bytes(K, bits);
    const float qmax = (float)qmax_of(bits);
    const float lo = (float)qlo_of(bits), hi = (float)qhi_of(bits);
    const int per = 8 / bits;
    const unsigned mask = (1u << bits) - 1u;
    for (int64_t r = 0; r < rows; ++r) {
        const float *wr = w + r * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(wr[k]);
            if (a > amax) amax = a;
        }
        float s = amax / qmax;
        scales[r] = s;
        uint8_t *cr = codes + r * rb;
        memset(cr, 0, (size_t)rb);
        for (int64_t k = 0; k < K; ++k) {
            float v = 0.0f;
            if (s != 0.0f) v = rintf(wr[k] / s);
            if (v > hi) v = hi;
            if (v < lo) v = lo;
            int c = (int)v;
            unsigned field = (unsigned)c & mask;
            cr[k / per] |= (uint8_t)(field << (bits * (k % per)));
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* FP8 checkpoint weights.  [HN] 実装済みの主な機能, offline-converter bullet:
 * the FP8 shards are dequantised with 128 x 128 block scales and then
 * requantised into the engine's container (the per-row formats above).
 * Reading (the pages name neither the FP8 variant nor the scale's
 * direction): FP8 is e4m3 with no infinities -- 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits; exponent field 0 is subnormal
 * (mantissa * 2^-9); the all-ones code S.1111.111 is NaN (so the largest
 * magnitude is 448) -- and the block scale multiplies:
 *   w[r][k] = (float)( e4m3(code[r][k]) * scale[r / B][k / B] )   (fp32)
 * with the scale grid ceil(rows / B) x ceil(K / B) for block size B.  The
 * requantised row is then oracle_quant_weights of these fp32 values. */
float oracle_fp8_e4m3(uint8_t code)
{
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (float)(sign ? -v : v);
}

void oracle_dequant_fp8(const uint8_t *codes, const float *scale, int64_t rows, int64_t K,
                        int64_t block, float *out)
{
    const int64_t kb = (K + block - 1) / block;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = oracle_fp8_e4m3(codes[r * K + k]) * scale[(r / block) * kb + k / block];
}

/* The whole converter step for one matrix: FP8 + block scales -> per-row
 * int8 / int4 / int2 codes and scales.  Returns oracle_quant_weights's code. */
int oracle_requant_fp8(const uint8_t *codes, const float *scale, int64_t rows, int64_t K,
                       int64_t block, int bits, uint8_t *out_codes, float *out_scales)
{
    float *w = malloc(sizeof(float) * (size_t)(rows * K));
    if (!w) return -2;
    oracle_dequant_fp8(codes, scale, rows, K, block, w);
    int rc = oracle_quant_weights(w, rows, K, bits, out_codes, out_scales);
    free(w);
    return rc;
}

/* Unpack codes back to signed integers (one int8 per element). */
int oracle_unpack_weights(const uint8_t *codes, int64_t rows, int64_t K, int bits, int8_t *out)
{
    if (bits != 8 && bits != 4 && bits != 2) return -1;
    const int64_t rb = oracle_row_bytes(K, bits);
    const int per = 8 / bits;
    const unsigned mask = (1u << bits) - 1u;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            unsigned field = (codes[r * rb + k / per] >> (bits * (k % per))) & mask;
            int v = (int)field;
            if (field & (1u << (bits - 1))) v -= (int)(1u << bits);
            out[r * K + k] = (int8_t)v;
        }
    }
    return 0;
}

static int code_at(const uint8_t *row, int64_t k, int bits)
{
    const int per = 8 / bits;
    const unsigned mask = (1u << bits) - 1u;
    unsigned field = (row[k / per] >> (bits * (k % per))) & mask;
    int v = (int)field;
    if (field & (1u << (bits - 1))) v -= (int)(1u << bits);
    return v;
}

/* ------------------------------------------------------------------------ */
/* Integer block sums.  [HN] integer-dot bullet: int8 activations times
 * int8/int4/int2 weights with an integer dot per 32-block:
 *   S[r][b] = sum over k in block b of w_code[r][k] * x_code[k]  (exact int32). */
void oracle_block_sums(const uint8_t *codes, int bits, int64_t rows, int64_t K,
                       const int8_t *xq, int32_t *S)
{
    const int64_t nb = K / QBLK, rb = oracle_row_bytes(K, bits);
    for (int64_t r = 0; r < rows; ++r) {
        const uint8_t *row = codes + r * rb;
        for (int64_t b = 0; b < nb; ++b) {
            int32_t s = 0;
            for (int i = 0; i < QBLK; ++i) {
                int64_t k = b * QBLK + i;
                s += code_at(row, k, bits) * (int32_t)xq[k];
            }
            S[r * nb + b] = s;
        }
    }
}

/* Dequantised-on-use dot of every row with one Q8_0 vector:
 *   acc_r = sum_b (double)S[r][b] * (double)d_b      (fp64, block order)
 *   out_r = (float)((double)acc_r * (double)scale_r)
 * Each product S*d is exact in fp64 (<= 40 significant bits). */
void oracle_int_dot(const uint8_t *codes, const float *scales, int bits, int64_t rows,
                    int64_t K, const int8_t *xq, const float *xd, float *out)
{
    const int64_t nb = K / QBLK, rb = oracle_row_bytes(K, bits);
    for (int64_t r = 0; r < rows; ++r) {
        const uint8_t *row = codes + r * rb;
        double acc = 0.0;
        for (int64_t b = 0; b < nb; ++b) {
            int32_t s = 0;
            for (int i = 0; i < QBLK; ++i) {
                int64_t k = b * QBLK + i;
                s += code_at(row, k, bits) * (int32_t)xq[k];
            }
            acc += (double)s * (double)xd[b];
        }
        out[r] = (float)(acc * (double)scales[r]);
    }
}

/* ------------------------------------------------------------------------ */
/* Router.  [HN] router bullet: DeepSeek-V3-style sigmoid router with noaux_tc
 * selection, an e_score_correction bias and routed_scaling_factor.  Reading
 * (the pages name the method only):
 *   l_e = x . W_r[e]            fp64 sum of exact fp32*fp32 products
 *   s_e = 1 / (1 + exp(-l_e))   fp64
 *   c_e = s_e + bias_e          choice score; the bias is not in the weights
 *   group score = sum of the two largest c in the group (one if the group
 *                 has a single expert); keep the topk_group best groups;
 *   idx = top_k of c over the kept experts, sorted by descending c;
 *   every tie goes to the lower group / expert index;
 *   w_j = (s_idx_j / sum_i s_idx_i) * routed_scaling_factor, rounded to fp32.
 * Margins reported per token (for the near-tie rule of the parity tests):
 *   kmargin = c(k-th kept) - c((k+1)-th kept)   (+inf if no (k+1)-th),
 *   gmargin = score(gk-th group) - score((gk+1)-th group) (+inf if gk == G). */
typedef struct {
    int hidden, inter, n_routed, n_shared, top_k, n_group, topk_group, bits;
    float routed_scaling_factor;
    float expert_top_p;  /* adaptive expert top-p; 0 or >= 1: off */
} oracle_cfg;

static int route_params_ok(int E, int G, int gk, int k)
{
    if (E <= 0 || G <= 0 || E % G != 0) return 0;
    if (gk <= 0 || gk > G) return 0;
    if (k <= 0 || k > gk * (E / G)) return 0;
    return 1;
}

/* Route one token given its fp64 scores s[E] and choice scores c[E]. */
static void select_token(const double *s, const double *c, int E, int G, int gk, int k,
                         float rsf, int32_t *idx, float *w, double *kmargin, double *gmargin,
                         double *gscore, unsigned char *gkeep, unsigned char *taken)
{
    const int per = E / G;
    for (int g = 0; g < G; ++g) {
        int b1 = -1, b2 = -1;
        for (int i = 0; i < per; ++i) {
            int e = g * per + i;
            if (b1 < 0 || c[e] > c[b1]) b1 = e;
        }
        for (int i = 0; i < per; ++i) {
            int e = g * per + i;
            if (e == b1) continue;
            if (b2 < 0 || c[e] > c[b2]) b2 = e;
        }
        gscore[g] = c[b1] + (b2 >= 0 ? c[b2] : 0.0);
        gkeep[g] = 0;
    }
    /* keep the gk best groups; the first index wins a tie */
    double last_kept = 0.0;
    for (int n = 0; n < gk; ++n) {
        int best = -1;
        for (int g = 0; g < G; ++g)
            if (!gkeep[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
        gkeep[best] = 1;
        last_kept = gscore[best];
    }
    if (gk < G) {
        int nxt = -1;
        for (int g = 0; g < G; ++g)
            if (!gkeep[g] && (nxt < 0 || gscore[g] > gscore[nxt])) nxt = g;
        *gmargin = last_kept - gscore[nxt];
    } else {
        *gmargin = INFINITY;
    }
    for (int e = 0; e < E; ++e) taken[e] = 0;
    double last_c = 0.0;
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e] || !gkeep[e / per]) continue;
            if (best < 0 || c[e] > c[best]) best = e;
        }
        taken[best] = 1;
        idx[j] = best;
        last_c = c[best];
    }
    {
        int nxt = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e] || !gkeep[e / per]) continue;
            if (nxt < 0 || c[e] > c[nxt]) nxt = e;
        }
        *kmargin = (nxt >= 0) ? last_c - c[nxt] : INFINITY;
    }
    double ssum = 0.0;
    for (int j = 0; j < k; ++j) ssum += s[idx[j]];
    for (int j = 0; j < k; ++j) w[j] = (float)((s[idx[j]] / ssum) * (double)rsf);
}

/* Adaptive expert top-p.  [HN] モデルのダウンロードと実行, useful-options
 * bullet: --topp 0.7 "adaptive expert top-p" (30-40 % less disk traffic);
 * the pages give no rule.  Reading: after the group-limited top-k, take the
 * k selected experts by descending sigmoid score s (ties: the earlier slot)
 * and keep each while the scores kept so far sum to less than p times the
 * sum over all k (the first is always kept), so the kept experts carry at
 * least p of the renormalised weight; the others are dropped (idx -1, w 0)
 * and the weights are renormalised over the kept ones:
 *   w_j = (s_j / sum_kept s) * routed_scaling_factor, sums in slot order.
 * pmargin: the smallest |sum_before - p * sum_all| / sum_all over the
 * decisions taken after the first (+inf if k == 1). */
static void apply_top_p(const double *s, int k, double p, float rsf, int32_t *idx, float *w,
                        double *pmargin)
{
    int order[32];
    unsigned char kept[32];
    double total = 0.0;
    for (int j = 0; j < k; ++j) {
        total += s[idx[j]];
        order[j] = j;
        kept[j] = 0;
    }
    /* slots by descending s, the earlier slot first on ties (insertion sort) */
    for (int a = 1; a < k; ++a) {
        int j = order[a], b = a;
        while (b > 0 && s[idx[order[b - 1]]] < s[idx[j]]) {
            order[b] = order[b - 1];
            --b;
        }
        order[b] = j;
    }
    const double cut = p * total;
    double cum = 0.0, margin = INFINITY;
    for (int n = 0; n < k; ++n) {
        const int j = order[n];
        if (n > 0) {
            const double dist = fabs(cum - cut) / total;
            if (dist < margin) margin = dist;
            if (!(cum < cut)) break;
        }
        kept[j] = 1;
        cum += s[idx[j]];
    }
    double ksum = 0.0;
    for (int j = 0; j < k; ++j)
        if (kept[j]) ksum += s[idx[j]];
    for (int j = 0; j < k; ++j) {
        if (kept[j]) {
            w[j] = (float)((s[idx[j]] / ksum) * (double)rsf);
        } else {
            idx[j] = -1;
            w[j] = 0.0f;
        }
    }
    if (pmargin) *pmargin = margin;
}

static int top_p_on(float p) { return p > 0.0f && p < 1.0f; }

static void token_scores(const float *xt, int64_t H, const float *Wr, const float *bias, int E,
                         double *s, double *c)
{
    for (int e = 0; e < E; ++e) {
        const float *we = Wr + (int64_t)e * H;
        double l = 0.0;
        for (int64_t h = 0; h < H; ++h) l += (double)xt[h] * (double)we[h];
        s[e] = 1.0 / (1.0 + exp(-l));
        c[e] = s[e] + (double)bias[e];
    }
}

/* Route T tokens.  Optional outputs (may be NULL): s_out/c_out [T][E],
 * kmargin/gmargin/pmargin [T].  top_p in (0, 1) applies the adaptive expert
 * top-p (dropped slots: idx -1, w 0).  Returns 0, or -1 on invalid parameters. */
int oracle_route(const float *x, int64_t T, int64_t H, const float *Wr, const float *bias,
                 int E, int G, int gk, int k, float rsf, float top_p, int32_t *idx, float *w,
                 double *s_out, double *c_out, double *kmargin, double *gmargin,
                 double *pmargin)
{
    if (!route_params_ok(E, G, gk, k)) return -1;
    double *s = malloc(sizeof(double) * E), *c = malloc(sizeof(double) * E);
    double *gs = malloc(sizeof(double) * G);
    unsigned char *gkeep = malloc(G), *taken = malloc(E);
    for (int64_t t = 0; t < T; ++t) {
        token_scores(x + t * H, H, Wr, bias, E, s, c);
        double km, gm;
        select_token(s, c, E, G, gk, k, rsf, idx + t * k, w + t * k, &km, &gm, gs, gkeep, taken);
        double pm = INFINITY;
        if (top_p_on(top_p)) apply_top_p(s, k, (double)top_p, rsf, idx + t * k, w + t * k, &pm);
        if (pmargin) pmargin[t] = pm;
        if (s_out) memcpy(s_out + t * E, s, sizeof(double) * E);
        if (c_out) memcpy(c_out + t * E, c, sizeof(double) * E);
        if (kmargin) kmargin[t] = km;
        if (gmargin) gmargin[t] = gm;
    }
    free(s); free(c); free(gs); free(gkeep); free(taken);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* One SwiGLU expert on one token.  [DT] an expert is gate, up and down
 * matrices; [HN] integer-dot and quantisation bullets give the int8/int4/int2
 * per-row weights dotted against Q8_0 activations.  Reading (the pages name
 * no activation function; SwiGLU is the GLM/DeepSeek-V3 FFN):
 *   g = int_dot(gate, Q8(x)),  u = int_dot(up, Q8(x))         [I]
 *   h = (float)((g / (1 + exp(-g))) * u)   evaluated in fp64
 *   (hq, hd) = Q8_0(h)                                         [I], [I/32]
 *   e = int_dot(down, hq, hd)                                  [H]
 * If hq_in/hd_in are given they replace Q8_0(h) (re-run with another
 * side's intermediate codes); hq_out/hd_out receive the codes used. */
typedef struct {
    const uint8_t *codes;
    const float *scales;
} oracle_qmat;

/* The SwiGLU activation of one expert's gate and up outputs:
 *   h[i] = (float)( SiLU(g[i]) * u[i] ),  SiLU(g) = g * sigmoid(g) = g / (1 + exp(-g)),
 * evaluated in fp64 from the fp32 g, u and rounded once to fp32.  The sigmoid
 * gates the gate projection g, never the up projection u. */
void oracle_swiglu(const float *g, const float *u, int64_t n, float *h)
{
    for (int64_t i = 0; i < n; ++i) {
        double gd = (double)g[i];
        h[i] = (float)((gd / (1.0 + exp(-gd))) * (double)u[i]);
    }
}

static void expert_token(int64_t H, int64_t I, int bits, const oracle_qmat *gate,
                         const oracle_qmat *up, const oracle_qmat *down, const int8_t *xq,
                         const float *xd, const int8_t *hq_in, const float *hd_in,
                         int8_t *hq_out, float *hd_out, float *e_out, float *scratch)
{
    float *g = scratch, *u = scratch + I, *h = scratch + 2 * I;
    oracle_int_dot(gate->codes, gate->scales, bits, I, H, xq, xd, g);
    oracle_int_dot(up->codes, up->scales, bits, I, H, xq, xd, u);
    oracle_swiglu(g, u, I, h);
    const int8_t *hq;
    const float *hd;
    if (hq_in && hd_in) {
        hq = hq_in;
        hd = hd_in;
        if (hq_out) memcpy(hq_out, hq_in, (size_t)I);
        if (hd_out) memcpy(hd_out, hd_in, sizeof(float) * (size_t)(I / QBLK));
    } else {
        oracle_quant_q8(h, 1, I, hq_out, hd_out);
        hq = hq_out;
        hd = hd_out;
    }
    oracle_int_dot(down->codes, down->scales, bits, H, I, hq, hd, e_out);
}

int oracle_expert(int64_t H, int64_t I, int bits, const oracle_qmat *gate, const oracle_qmat *up,
                  const oracle_qmat *down, const int8_t *xq, const float *xd,
                  const int8_t *hq_in, const float *hd_in, int8_t *hq_out, float *hd_out,
                  float *e_out)
{
    if (H % QBLK || I % QBLK) return -1;
    float *scratch = malloc(sizeof(float) * 3 * (size_t)I);
    if (!scratch) return -2;
    expert_token(H, I, bits, gate, up, down, xq, xd, hq_in, hd_in, hq_out, hd_out, e_out, scratch);
    free(scratch);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The layer.  Steps, in the pages' order: route ([HN] router bullet), Q8_0(x)
 * ([HN] integer-dot bullet), every selected expert plus the shared experts,
 * then the combine.  Reading of the combine (plainest DeepSeek-V3 reading;
 * the pages only name the shared expert):
 *   y_t = (float)( e_shared + sum_{j<k} (double)w_tj * (double)e_{idx_tj} )
 * accumulated in fp64, shared experts first (weight 1, not scaled by
 * routed_scaling_factor), then routed experts in slot order.
 *
 * mats: (E + n_shared) * 3 matrices, expert-major, (gate, up, down); the
 * shared experts come last.  Entries of experts that no token selects may be
 * NULL.  idx_in (optional [T][k]) replaces the routing decision; the weights
 * are then renormalised from this oracle's own s for those experts.
 * hq_in/hd_in (optional [T][k+n_shared][I], [..][I/32]) replace Q8_0(h) per
 * (token, slot); slot j < k is routed slot j, slot k+i is shared expert i.
 * Outputs idx_out/w_out/hq_out/hd_out may be NULL.  nthreads > 1 splits the
 * tokens over OpenMP threads; the arithmetic per token does not change.
 *
 * A dense layer ([HN] router bullet: the first three layers are dense) is
 * n_routed = 0 with top_k = 0: no routing, every token through the shared
 * experts only (weight 1), y_t = (float)(sum of the shared experts' e).
 * Returns 0, -1 on invalid parameters, -3 if a needed expert is NULL. */
int oracle_moe_forward(const oracle_cfg *cfg, const float *Wr, const float *bias,
                       const oracle_qmat *mats, const float *x, int64_t T,
                       const int32_t *idx_in, const int8_t *hq_in, const float *hd_in,
                       int32_t *idx_out, float *w_out, int8_t *hq_out, float *hd_out,
                       float *out, int nthreads)
{
    const int64_t H = cfg->hidden, I = cfg->inter;
    const int E = cfg->n_routed, S = cfg->n_shared, k = cfg->top_k;
    const int G = cfg->n_group, gk = cfg->topk_group, bits = cfg->bits;
    if (H % QBLK || I % QBLK || S < 0) return -1;
    if (bits != 8 && bits != 4 && bits != 2) return -1;
    const int dense = E == 0 && k == 0;
    if (dense ? S < 1 : !route_params_ok(E, G, gk, k)) return -1;
    const int slots = k + S;

    int32_t *idx = malloc(sizeof(int32_t) * (size_t)(T * k));
    float *w = malloc(sizeof(float) * (size_t)(T * k));
    int8_t *xq = malloc((size_t)(T * H));
    float *xd = malloc(sizeof(float) * (size_t)(T * (H / QBLK)));
    if (!idx || !w || !xq || !xd) { free(idx); free(w); free(xq); free(xd); return -2; }

    /* 1. routing (none in a dense layer) */
    if (!dense) {
        double *s = malloc(sizeof(double) * E), *c = malloc(sizeof(double) * E);
        double *gs = malloc(sizeof(double) * G);
        unsigned char *gkeep = malloc(G), *taken = malloc(E);
        for (int64_t t = 0; t < T; ++t) {
            token_scores(x + t * H, H, Wr, bias, E, s, c);
            double km, gm;
            select_token(s, c, E, G, gk, k, cfg->routed_scaling_factor, idx + t * k, w + t * k,
                         &km, &gm, gs, gkeep, taken);
            if (top_p_on(cfg->expert_top_p))
                apply_top_p(s, k, (double)cfg->expert_top_p, cfg->routed_scaling_factor,
                            idx + t * k, w + t * k, NULL);
            if (idx_in) {  /* another side's choice; -1 marks a dropped slot */
                double ssum = 0.0;
                for (int j = 0; j < k; ++j) {
                    idx[t * k + j] = idx_in[t * k + j];
                    if (idx_in[t * k + j] >= 0) ssum += s[idx_in[t * k + j]];
                }
                for (int j = 0; j < k; ++j)
                    w[t * k + j] = idx_in[t * k + j] < 0 ? 0.0f
                                   : (float)((s[idx_in[t * k + j]] / ssum) *
                                             (double)cfg->routed_scaling_factor);
            }
        }
        free(s); free(c); free(gs); free(gkeep); free(taken);
    }
    /* 2. Q8_0(x) */
    oracle_quant_q8(x, T, H, xq, xd);

    /* every needed expert must be present */
    int missing = 0;
    for (int64_t t = 0; t < T && !missing; ++t)
        for (int j = 0; j < slots; ++j) {
            int e = j < k ? idx[t * k + j] : E + (j - k);
            if (j < k && e == -1) continue;  /* a slot top-p dropped */
            if (e < 0 || e >= E + S) { missing = 1; break; }
            for (int m = 0; m < 3; ++m)
                if (!mats[e * 3 + m].codes || !mats[e * 3 + m].scales) missing = 1;
        }
    if (missing) { free(idx); free(w); free(xq); free(xd); return -3; }

    /* 3-4. experts and combine, one token at a time */
    int64_t t;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (t = 0; t < T; ++t) {
        float *scratch = malloc(sizeof(float) * (size_t)(3 * I + H));
        int8_t *hq_tmp = malloc((size_t)I);
        float *hd_tmp = malloc(sizeof(float) * (size_t)(I / QBLK));
        float *e = scratch + 3 * I;
        double *acc = malloc(sizeof(double) * (size_t)H);
        for (int jj = 0; jj < slots; ++jj) {
            /* shared experts first, then routed slots in order */
            int j = jj < S ? k + jj : jj - S;
            int ex = j < k ? idx[t * k + j] : E + (j - k);
            int64_t hs = (t * slots + j);
            if (ex < 0) {  /* a slot top-p dropped: no expert, no contribution */
                if (hq_out) memset(hq_out + hs * I, 0, (size_t)I);
                if (hd_out) memset(hd_out + hs * (I / QBLK), 0, sizeof(float) * (size_t)(I / QBLK));
                if (jj == 0)
                    for (int64_t r = 0; r < H; ++r) acc[r] = 0.0;
                continue;
            }
            const oracle_qmat *m3 = mats + (int64_t)ex * 3;
            const int8_t *hqi = hq_in ? hq_in + hs * I : NULL;
            const float *hdi = hd_in ? hd_in + hs * (I / QBLK) : NULL;
            int8_t *hqo = hq_out ? hq_out + hs * I : hq_tmp;
            float *hdo = hd_out ? hd_out + hs * (I / QBLK) : hd_tmp;
            expert_token(H, I, bits, &m3[0], &m3[1], &m3[2], xq + t * H, xd + t * (H / QBLK),
                         hqi, hdi, hqo, hdo, e, scratch);
            if (jj == 0) {
                for (int64_t r = 0; r < H; ++r)
                    acc[r] = (j < k) ? (double)w[t * k + j] * (double)e[r] : (double)e[r];
            } else {
                for (int64_t r = 0; r < H; ++r)
                    acc[r] += (j < k) ? (double)w[t * k + j] * (double)e[r] : (double)e[r];
            }
        }
        for (int64_t r = 0; r < H; ++r) out[t * H + r] = (float)acc[r];
        free(acc); free(scratch); free(hq_tmp); free(hd_tmp);
    }
    if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * (size_t)(T * k));
    if (w_out) memcpy(w_out, w, sizeof(float) * (size_t)(T * k));
    free(idx); free(w); free(xq); free(xd);
    return 0;
}
