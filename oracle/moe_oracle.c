/*
 * CPU oracle for one MoE FFN layer forward (sigmoid+bias router, top-k,
 * int4 per-row symmetric SwiGLU experts, shared expert, weighted combine).
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  The product path never calls it;
 * it shares no code, header, table or helper with the CUDA library.
 *
 * Plain, slow and single-threaded: every quantity is computed in double
 * precision straight from its definition, in the order the definition states,
 * with no blocking, no bucketing and no fusion.
 *
 * Sources (page titles and sections of the pages describing the method):
 *  - Colibri-Nano model card, "Architecture": 64 experts, top-2, a
 *    2048-wide always-resident shared expert, sigmoid+bias router
 *    (DeepSeek-V3-style aux-loss-free balancing).
 *  - colibri README (project listing, "What's implemented"): DeepSeek-V3-style
 *    sigmoid router (noaux_tc, routed_scaling_factor), shared expert;
 *    packed int4 with per-row scales, dequant-on-use; batch-union MoE.
 *  - nanocolibri-engine README, "Converting a checkpoint yourself":
 *    quantisation is per-row symmetric with f32 scales in a sibling tensor;
 *    router weights and router bias stay f32.
 *  - nanocolibri-engine README, "Knobs" (IDOT=0): the exact f32 dequant path,
 *    which this oracle takes to f64.
 * The pages name the method but do not write its formulas out.  The formulas
 * used (the plainest reading of those passages):
 *   L[t,e]  = sum_h x[t,h] * W[e,h]
 *   s[t,e]  = 1 / (1 + exp(-L[t,e]))                 (sigmoid score)
 *   b[t,e]  = s[t,e] + bias[e]                        (selection key only)
 *   S_t     = the K experts with the largest b (ties: lower expert index;
 *             NaN counts as -infinity)
 *   w[t,k]  = scale * s[t,e_k] / sum_{j in S_t} s[t,j]
 *   FFN(x)  = W2 . (silu(Wg . x) * (Wu . x)),  silu(z) = z * sigmoid(z),
 *             Wg = rows 0..I-1 and Wu = rows I..2I-1 of w13,
 *             every weight dequantised as code * row_scale
 *   out[t]  = sum_k w[t,k] * FFN_{e_k}(x_t) + FFN_shared(x_t) [+ x_t]
 *   (the shared expert has weight 1 and is not multiplied by `scale`).
 * Adaptive expert top-p (opt-in; colibri README, "Quick start" knobs: "--topp
 * 0.7 adaptive expert top-p"), 0 < p < 1: of the K selected experts, taken in
 * decreasing score order (ties: lower expert index), an expert is kept while
 * the scores of the experts kept before it sum to less than p times the
 * scores of all K: the fewest highest-weight experts whose normalised weight
 * reaches p.  Kept experts keep their selection order and are re-weighted
 * over the kept set, w[t,k] = scale * s[t,e_k] / sum_{j kept} s[t,j]; the
 * dropped picks become index -1 with weight 0, after the kept ones.
 * Int4 code layout: byte j of a row holds element 2j in bits 0..3 and element
 * 2j+1 in bits 4..7, each a 4-bit two's-complement value in [-8, 7].
 * Int8 experts (opt-in; nanocolibri-engine README, "Converting a checkpoint
 * yourself": --ebits sets the expert bits, per-row symmetric with f32 scales;
 * colibri README, "What's implemented": int8 / packed int4 quantisation
 * kernels with per-row scales): byte j of a row is element j, an 8-bit
 * two's-complement value in [-128, 127]; every weight is still code *
 * row_scale.  `wbits` (4 or 8) tells which layout the expert weights use.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENOMEM 2

/* bf16 bit pattern -> double (exact: bf16 is the top half of an f32). */
static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* The 4-bit two's-complement code of element j of a packed row. */
static int int4_code(const uint8_t* row, int64_t j) {
    uint8_t byte = row[j >> 1];
    int nib = (j & 1) ? (byte >> 4) : (byte & 0x0F);
    return nib >= 8 ? nib - 16 : nib;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* Decode n codes of a packed row (test hook for the code layout). */
int oracle_unpack_int4(const uint8_t* row, int64_t n, int32_t* codes) {
    if (!row || !codes || n < 0) return ORC_EINVAL;
    for (int64_t j = 0; j < n; ++j) codes[j] = int4_code(row, j);
    return ORC_OK;
}

/* Dot product of a dequantised packed row (code * scale, in double) with a
 * double vector of length n. */
static int int8_code(const uint8_t* row, int64_t j) { return (int)(int8_t)row[j]; }

static double dequant_row_dot(const uint8_t* row, float scale, const double* v, int64_t n, int wbits) {
    double acc = 0.0;
    double s = (double)scale;
    for (int64_t j = 0; j < n; ++j) acc += ((double)(wbits == 8 ? int8_code(row, j) : int4_code(row, j)) * s) * v[j];
    return acc;
}

typedef struct { double key; int32_t e; } sel_item;

static int sel_cmp(const void* a, const void* b) {
    const sel_item* x = (const sel_item*)a;
    const sel_item* y = (const sel_item*)b;
    if (x->key > y->key) return -1;
    if (x->key < y->key) return 1;
    return (x->e < y->e) ? -1 : (x->e > y->e);
}

/* Adaptive top-p over the K picks idx[0..K) with the given scores (see the
 * header): compacts the kept picks to the front, in their order, and writes
 * their re-normalised weights; the rest become -1 / 0.  topp_margin (nullable)
 * receives min over the picks of |cum_before - p * total| / total, how close
 * the decision came to going the other way. */
static void apply_topp(double topp, double scale, const double* scores, int K, int32_t* idx, double* wts,
                       double* topp_margin) {
    int ord[64], keep[64];
    double total = 0.0;
    for (int k = 0; k < K; ++k) {
        ord[k] = k;
        keep[k] = 0;
        total += scores[idx[k]];
    }
    /* insertion sort of the picks by (score desc, expert index asc) */
    for (int i = 1; i < K; ++i) {
        int v = ord[i], j = i - 1;
        while (j >= 0 && (scores[idx[ord[j]]] < scores[idx[v]] ||
                          (scores[idx[ord[j]]] == scores[idx[v]] && idx[ord[j]] > idx[v]))) {
            ord[j + 1] = ord[j];
            --j;
        }
        ord[j + 1] = v;
    }
    double cum = 0.0, mm = INFINITY;
    for (int j = 0; j < K; ++j) {
        double d = fabs(cum - topp * total) / total;
        if (d < mm) mm = d;
        if (cum < topp * total) {
            keep[ord[j]] = 1;
            cum += scores[idx[ord[j]]];
        }
    }
    int32_t kept_idx[64];
    int n = 0;
    for (int k = 0; k < K; ++k)
        if (keep[k]) kept_idx[n++] = idx[k];
    double denom = 0.0;
    for (int k = 0; k < n; ++k) denom += scores[kept_idx[k]];
    for (int k = 0; k < K; ++k) {
        idx[k] = k < n ? kept_idx[k] : -1;
        wts[k] = k < n ? scale * scores[kept_idx[k]] / denom : 0.0;
    }
    if (topp_margin) *topp_margin = mm;
}

/* Router of one token: logits, sigmoid scores, biased keys, top-K by a full
 * sort of (key desc, index asc), margin = key_(K) - key_(K+1), weights; then
 * the adaptive top-p when 0 < topp < 1. */
static int route_one(const double* xt, const float* W, const float* bias, int H, int E, int K,
                     double scale, double topp, const int32_t* forced, double* logits, double* scores,
                     int32_t* idx, double* wts, double* margin, double* topp_margin, sel_item* items) {
    for (int e = 0; e < E; ++e) {
        double L = 0.0;
        const float* We = W + (int64_t)e * H;
        for (int h = 0; h < H; ++h) L += xt[h] * (double)We[h];
        double s = sigmoid(L);
        double key = s + (double)bias[e];
        if (isnan(key)) key = -INFINITY;
        if (logits) logits[e] = L;
        scores[e] = s;
        items[e].key = key;
        items[e].e = e;
    }
    qsort(items, (size_t)E, sizeof(sel_item), sel_cmp);
    if (margin) *margin = (K < E) ? (items[K - 1].key - items[K].key) : INFINITY;
    if (topp_margin) *topp_margin = INFINITY;
    if (forced) {
        /* a forced selection as given (with -1 for picks the top-p dropped) */
        int n = 0;
        for (int k = 0; k < K; ++k) {
            int32_t e = forced[k];
            if (e == -1 && topp > 0.0 && topp < 1.0) {
                idx[k] = -1;
                continue;
            }
            if (e < 0 || e >= E) return ORC_EINVAL;
            idx[k] = e;
            ++n;
        }
        if (n == 0) return ORC_EINVAL;
        double denom = 0.0;
        for (int k = 0; k < K; ++k)
            if (idx[k] >= 0) denom += scores[idx[k]];
        for (int k = 0; k < K; ++k) wts[k] = idx[k] >= 0 ? scale * scores[idx[k]] / denom : 0.0;
        return ORC_OK;
    }
    for (int k = 0; k < K; ++k) idx[k] = items[k].e;
    double denom = 0.0;
    for (int k = 0; k < K; ++k) denom += scores[idx[k]];
    for (int k = 0; k < K; ++k) wts[k] = scale * scores[idx[k]] / denom;
    if (topp > 0.0 && topp < 1.0) apply_topp(topp, scale, scores, K, idx, wts, topp_margin);
    return ORC_OK;
}

/* Selection alone, from given sigmoid scores: top-K of scores + bias per
 * token.  scores: double [T,E]; idx [T,K]; margin [T] (nullable). */
int oracle_select_topk(const double* scores, const float* bias, int32_t T, int32_t E, int32_t K,
                       int32_t* idx, double* margin) {
    if (!scores || !bias || !idx || T < 0 || E <= 0 || K <= 0 || K > E) return ORC_EINVAL;
    sel_item* items = (sel_item*)malloc(sizeof(sel_item) * (size_t)E);
    if (!items) return ORC_ENOMEM;
    for (int32_t t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double key = scores[(int64_t)t * E + e] + (double)bias[e];
            items[e].key = isnan(key) ? -INFINITY : key;
            items[e].e = e;
        }
        qsort(items, (size_t)E, sizeof(sel_item), sel_cmp);
        for (int k = 0; k < K; ++k) idx[(int64_t)t * K + k] = items[k].e;
        if (margin) margin[t] = (K < E) ? (items[K - 1].key - items[K].key) : INFINITY;
    }
    free(items);
    return ORC_OK;
}

/* Router for T tokens.  x: bf16 bits [T,H]; W: f32 [E,H]; bias: f32 [E];
 * topp: 0 = plain top-K, else the adaptive top-p.  Outputs (row-major):
 * logits/scores [T,E] (nullable), idx [T,K], weights [T,K], margin [T] and
 * topp_margin [T] (nullable). */
int oracle_route(const uint16_t* x, const float* W, const float* bias, int32_t T, int32_t H,
                 int32_t E, int32_t K, double scale, double topp, double* logits, double* scores,
                 int32_t* idx, double* weights, double* margin, double* topp_margin) {
    if (!x || !W || !bias || !idx || !weights || T < 0 || H <= 0 || E <= 0 || K <= 0 || K > E)
        return ORC_EINVAL;
    double* xt = (double*)malloc(sizeof(double) * (size_t)H);
    double* sc = (double*)malloc(sizeof(double) * (size_t)E);
    sel_item* items = (sel_item*)malloc(sizeof(sel_item) * (size_t)E);
    int rc = (xt && sc && items) ? ORC_OK : ORC_ENOMEM;
    for (int32_t t = 0; rc == ORC_OK && t < T; ++t) {
        for (int h = 0; h < H; ++h) xt[h] = bf16_bits_to_double(x[(int64_t)t * H + h]);
        rc = route_one(xt, W, bias, H, E, K, scale, topp, NULL, logits ? logits + (int64_t)t * E : NULL,
                       sc, idx + (int64_t)t * K, weights + (int64_t)t * K,
                       margin ? margin + t : NULL, topp_margin ? topp_margin + t : NULL, items);
        if (scores) memcpy(scores + (int64_t)t * E, sc, sizeof(double) * (size_t)E);
    }
    free(xt); free(sc); free(items);
    return rc;
}

/* One SwiGLU expert applied to one token.
 * x: double [H]; w13: [2I, H*wbits/8] (rows 0..I-1 gate, I..2I-1 up);
 * s13: f32 [2I]; w2: [H, I*wbits/8]; s2: f32 [H]; wbits: 4 (packed int4) or 8.
 * h_out: double [I] (nullable), y: double [H]. */
int oracle_expert_ffn(const double* x, int32_t H, int32_t I, const uint8_t* w13, const float* s13,
                      const uint8_t* w2, const float* s2, int32_t wbits, double* h_out, double* y) {
    if (!x || !w13 || !s13 || !w2 || !s2 || !y || H <= 0 || I <= 0 || (H & 1) || (I & 1) ||
        (wbits != 4 && wbits != 8))
        return ORC_EINVAL;
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    if (!h) return ORC_ENOMEM;
    const int64_t row13 = (int64_t)H * wbits / 8, row2 = (int64_t)I * wbits / 8;
    for (int32_t r = 0; r < I; ++r) {
        double g = dequant_row_dot(w13 + (int64_t)r * row13, s13[r], x, H, wbits);
        double u = dequant_row_dot(w13 + (int64_t)(I + r) * row13, s13[I + r], x, H, wbits);
        h[r] = (g * sigmoid(g)) * u;
    }
    for (int32_t j = 0; j < H; ++j) y[j] = dequant_row_dot(w2 + (int64_t)j * row2, s2[j], h, I, wbits);
    if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)I);
    free(h);
    return ORC_OK;
}

/* The layer output for a list of tokens (NULL list = all T tokens, in order).
 *
 * x: bf16 bits [T,H]; router_w f32 [E,H]; router_bias f32 [E];
 * w13 [E,2I,H*wbits/8]; s13 f32 [E,2I]; w2 [E,H,I*wbits/8]; s2 f32 [E,H];
 * sh_* the shared expert with intermediate Is (Is = 0: no shared expert), in
 * the same code layout; wbits: 4 (packed int4) or 8.
 * idx_override [n,K] (nullable): evaluate with these experts instead of the
 * router's choice (weights still come from the router's scores; with top-p,
 * -1 entries are dropped picks).  topp: 0 = plain top-K, else the adaptive
 * top-p.  Outputs: out double [n,H]; idx_out [n,K], w_out [n,K], margin_out
 * [n] (each nullable). */
int oracle_moe_tokens(const uint16_t* x, int32_t T, int32_t H, int32_t E, int32_t K, int32_t I,
                      int32_t Is, double scale, double topp, int32_t residual, const float* router_w,
                      const float* router_bias, const uint8_t* w13, const float* s13,
                      const uint8_t* w2, const float* s2, const uint8_t* sh_w13,
                      const float* sh_s13, const uint8_t* sh_w2, const float* sh_s2, int32_t wbits,
                      const int32_t* tokens, int32_t n_tokens, const int32_t* idx_override,
                      double* out, int32_t* idx_out, double* w_out, double* margin_out) {
    if (!x || !router_w || !router_bias || !w13 || !s13 || !w2 || !s2 || !out) return ORC_EINVAL;
    if (T < 0 || H <= 0 || E <= 0 || K <= 0 || K > E || I <= 0 || Is < 0) return ORC_EINVAL;
    if (Is > 0 && (!sh_w13 || !sh_s13 || !sh_w2 || !sh_s2)) return ORC_EINVAL;
    int32_t n = tokens ? n_tokens : T;
    if (n < 0) return ORC_EINVAL;
    double* xt = (double*)malloc(sizeof(double) * (size_t)H);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    double* sc = (double*)malloc(sizeof(double) * (size_t)E);
    sel_item* items = (sel_item*)malloc(sizeof(sel_item) * (size_t)E);
    int32_t idx[64];
    double wts[64];
    int rc = (xt && y && sc && items) ? ORC_OK : ORC_ENOMEM;
    if (K > 64) rc = ORC_EINVAL;
    if (wbits != 4 && wbits != 8) rc = ORC_EINVAL;
    const int64_t e13 = (int64_t)2 * I * H * wbits / 8, e2 = (int64_t)H * I * wbits / 8;
    for (int32_t i = 0; rc == ORC_OK && i < n; ++i) {
        int32_t t = tokens ? tokens[i] : i;
        if (t < 0 || t >= T) { rc = ORC_EINVAL; break; }
        for (int h = 0; h < H; ++h) xt[h] = bf16_bits_to_double(x[(int64_t)t * H + h]);
        double margin;
        rc = route_one(xt, router_w, router_bias, H, E, K, scale, topp,
                       idx_override ? idx_override + (int64_t)i * K : NULL, NULL, sc, idx, wts,
                       &margin, NULL, items);
        if (rc != ORC_OK) break;
        double* o = out + (int64_t)i * H;
        for (int h = 0; h < H; ++h) o[h] = 0.0;
        for (int k = 0; k < K && rc == ORC_OK; ++k) {
            int32_t e = idx[k];
            if (e < 0) continue; /* dropped by the top-p */
            rc = oracle_expert_ffn(xt, H, I, w13 + e * e13, s13 + (int64_t)e * 2 * I, w2 + e * e2,
                                   s2 + (int64_t)e * H, wbits, NULL, y);
            for (int h = 0; h < H; ++h) o[h] += wts[k] * y[h];
        }
        if (rc == ORC_OK && Is > 0) {
            rc = oracle_expert_ffn(xt, H, Is, sh_w13, sh_s13, sh_w2, sh_s2, wbits, NULL, y);
            for (int h = 0; h < H; ++h) o[h] += y[h];
        }
        if (residual)
            for (int h = 0; h < H; ++h) o[h] += xt[h];
        if (idx_out) memcpy(idx_out + (int64_t)i * K, idx, sizeof(int32_t) * (size_t)K);
        if (w_out) memcpy(w_out + (int64_t)i * K, wts, sizeof(double) * (size_t)K);
        if (margin_out) margin_out[i] = margin;
    }
    free(xt); free(y); free(sc); free(items);
    return rc;
}
