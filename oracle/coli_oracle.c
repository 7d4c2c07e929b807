/*
 * coli_oracle.c -- the plain f64 CPU definition of the routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY (see coli_oracle.h): used by the tests, the smoke
 * check and the benchmark's CPU-baseline leg, never by the product path.
 *
 * Every step is written as its definition, in the pages' order
 * (Route -> Union -> expert compute), with no blocking, fusion or reordering.
 * The only parallelism is an OpenMP loop over the output rows of one
 * matrix-vector product, which does not change any result.
 */
#include "coli_oracle.h"

#include <float.h>
#include <math.h>
#include <stddef.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define COLI_ORACLE_GROUP 64

int coli_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * int4-gs64 storage ("gs64 build" of the int4 container: "colibri: 744B MoEを
 * ストレージから推論するCエンジン", section はじめにとソースが語らないこと).
 * The pages name the format only; this library reads it as: row-major [N, K],
 * two values per byte with the even k in the low nibble, each nibble a
 * two's-complement integer in [-8, 7], no zero point, and one fp32 scale per
 * 64 consecutive k of a row.  W[n, kk] = q * s[n, kk / 64].
 */
double coli_oracle_weight(const uint8_t* q, const float* s, int64_t K, int64_t n, int64_t kk)
{
    uint8_t byte = q[n * (K / 2) + kk / 2];
    int nib = (kk % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
    int value = (nib >= 8) ? nib - 16 : nib;
    double scale = (double)s[n * (K / COLI_ORACLE_GROUP) + kk / COLI_ORACLE_GROUP];
    return (double)value * scale;
}

int coli_oracle_dequant(const uint8_t* q, const float* s, int64_t N, int64_t K, double* W)
{
    if (!q || !s || !W || N < 0 || K <= 0 || K % COLI_ORACLE_GROUP != 0) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t kk = 0; kk < K; ++kk)
            W[n * K + kk] = coli_oracle_weight(q, s, K, n, kk);
    return 0;
}

int coli_oracle_matvec(const uint8_t* q, const float* s, int64_t N, int64_t K,
                       const double* x, double* y)
{
    if (!q || !s || !x || !y || N < 0 || K <= 0 || K % COLI_ORACLE_GROUP != 0) return -1;
    int64_t n;
#pragma omp parallel for schedule(static)
    for (n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t kk = 0; kk < K; ++kk)
            acc += coli_oracle_weight(q, s, K, n, kk) * x[kk];
        y[n] = acc;
    }
    return 0;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/*
 * Route ("Colibri 完全ガイド", section コア技術のハイライト: a DeepSeek-V3-style
 * sigmoid router; Korean getting-started page, section 토큰당 처리 경로, "Route").
 * Per token t:
 *   logit_e = sum_h x[t,h] * Wr[e,h]
 *   s_e     = 1 / (1 + exp(-logit_e))
 *   c_e     = s_e + b_e                      (bias-corrected selection score)
 *   idx     = the k experts of largest c, in descending c; equal c -> lower e first
 *   w_j     = routed_scale * s_idx[j] / sum_j' s_idx[j']
 * Readings: top-k is taken over all E experts (the pages mention no grouping);
 * the bias only selects, the weights use the unbiased s.
 */
int coli_oracle_route(const double* x, int64_t T, int64_t H,
                      const float* w_router, const float* sel_bias, int64_t E, int64_t k,
                      double routed_scale, int32_t* topk_idx, double* topk_w,
                      double* logits, double* sig, double* biased)
{
    if (!x || !w_router || !sel_bias || !topk_idx || !topk_w) return -1;
    if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return -1;

    double* l = (double*)malloc(sizeof(double) * (size_t)E);
    double* sv = (double*)malloc(sizeof(double) * (size_t)E);
    double* c = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    if (!l || !sv || !c || !taken) { free(l); free(sv); free(c); free(taken); return -1; }

    for (int64_t t = 0; t < T; ++t) {
        const double* xt = x + t * H;
        int64_t e;
#pragma omp parallel for schedule(static)
        for (e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h) acc += xt[h] * (double)w_router[e * H + h];
            l[e] = acc;
        }
        for (e = 0; e < E; ++e) {
            sv[e] = sigmoid(l[e]);
            c[e] = sv[e] + (double)sel_bias[e];
            taken[e] = 0;
            if (logits) logits[t * E + e] = l[e];
            if (sig) sig[t * E + e] = sv[e];
            if (biased) biased[t * E + e] = c[e];
        }
        /* selection: k rounds of "largest remaining c, lowest index on ties" */
        for (int64_t j = 0; j < k; ++j) {
            int64_t best = -1;
            for (e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || c[e] > c[best]) best = e;
            }
            taken[best] = 1;
            topk_idx[t * k + j] = (int32_t)best;
        }
        double denom = 0.0;
        for (int64_t j = 0; j < k; ++j) denom += sv[topk_idx[t * k + j]];
        for (int64_t j = 0; j < k; ++j)
            topk_w[t * k + j] = routed_scale * sv[topk_idx[t * k + j]] / denom;
    }
    free(l); free(sv); free(c); free(taken);
    return 0;
}

/*
 * Union (Korean getting-started page, section 토큰당 처리 경로, "Union": experts that
 * several tokens of a batch select are de-duplicated so each is processed once).
 * The pair p = t*k + j goes to bucket idx[p]; buckets are listed in ascending
 * expert order and, inside a bucket, pairs keep ascending p (a stable sort).
 */
int coli_oracle_union(const int32_t* topk_idx, int64_t T, int64_t k, int64_t E,
                      int32_t* count, int32_t* offset, int32_t* active, int32_t* n_active,
                      int32_t* perm, int32_t* inv_perm)
{
    if (!topk_idx || !count || !offset || !active || !n_active || !perm || !inv_perm) return -1;
    if (T < 0 || k <= 0 || E <= 0) return -1;
    int64_t P = T * k;
    for (int64_t p = 0; p < P; ++p)
        if (topk_idx[p] < 0 || topk_idx[p] >= E) return -1;

    for (int64_t e = 0; e < E; ++e) count[e] = 0;
    for (int64_t p = 0; p < P; ++p) count[topk_idx[p]] += 1;

    offset[0] = 0;
    for (int64_t e = 0; e < E; ++e) offset[e + 1] = offset[e] + count[e];

    int32_t na = 0;
    for (int64_t e = 0; e < E; ++e) active[e] = -1;
    for (int64_t e = 0; e < E; ++e)
        if (count[e] > 0) active[na++] = (int32_t)e;
    n_active[0] = na;

    int64_t pos = 0;
    for (int64_t e = 0; e < E; ++e)
        for (int64_t p = 0; p < P; ++p)
            if (topk_idx[p] == e) {
                perm[pos] = (int32_t)p;
                inv_perm[p] = (int32_t)pos;
                ++pos;
            }
    return 0;
}

/*
 * One expert on one token.  The pages describe each routed expert as an int4
 * FFN block of about 19 MB (Korean page, section 프로젝트 설명) but do not print
 * its form; this library reads it as SwiGLU:
 *   g = Wg x,  u = Wu x,  h = silu(g) * u  with silu(z) = z / (1 + exp(-z)),
 *   y = Wd h.
 */
int coli_oracle_expert_ffn(const double* x, int64_t H, int64_t F,
                           const uint8_t* gate_q, const float* gate_s,
                           const uint8_t* up_q, const float* up_s,
                           const uint8_t* down_q, const float* down_s,
                           double* y, double* h)
{
    if (!x || !gate_q || !gate_s || !up_q || !up_s || !down_q || !down_s || !y) return -1;
    if (H <= 0 || F <= 0 || H % COLI_ORACLE_GROUP != 0 || F % COLI_ORACLE_GROUP != 0) return -1;

    double* g = (double*)malloc(sizeof(double) * (size_t)F);
    double* u = (double*)malloc(sizeof(double) * (size_t)F);
    double* a = (double*)malloc(sizeof(double) * (size_t)F);
    if (!g || !u || !a) { free(g); free(u); free(a); return -1; }

    coli_oracle_matvec(gate_q, gate_s, F, H, x, g);
    coli_oracle_matvec(up_q, up_s, F, H, x, u);
    for (int64_t f = 0; f < F; ++f) {
        a[f] = g[f] * sigmoid(g[f]) * u[f];
        if (h) h[f] = a[f];
    }
    coli_oracle_matvec(down_q, down_s, H, F, a, y);

    free(g); free(u); free(a);
    return 0;
}

/*
 * The layer: Route, then the combine of the selected experts and the shared
 * expert.  out_t = sum_j w[t,j] * FFN_{idx[t,j]}(x_t) + FFN_E(x_t).
 * The shared expert ("Colibri 完全ガイド", DeepSeek-V3 router row: shared experts;
 * Korean page, section 프로젝트 설명) is always applied with weight one; the
 * pages do not say it is scaled, so it is not.
 */
int coli_oracle_moe_layer(const double* x, int64_t T, int64_t H, int64_t F,
                          int64_t E, int64_t k, double routed_scale,
                          const float* w_router, const float* sel_bias,
                          const uint8_t* const* gate_q, const float* const* gate_s,
                          const uint8_t* const* up_q, const float* const* up_s,
                          const uint8_t* const* down_q, const float* const* down_s,
                          int32_t* topk_idx, double* topk_w, double* out)
{
    if (!x || !gate_q || !gate_s || !up_q || !up_s || !down_q || !down_s) return -1;
    if (!topk_idx || !topk_w || !out) return -1;
    int rc = coli_oracle_route(x, T, H, w_router, sel_bias, E, k, routed_scale,
                               topk_idx, topk_w, NULL, NULL, NULL);
    if (rc != 0) return rc;

    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    if (!y) return -1;
    for (int64_t t = 0; t < T; ++t) {
        const double* xt = x + t * H;
        double* ot = out + t * H;
        for (int64_t n = 0; n < H; ++n) ot[n] = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            int64_t e = topk_idx[t * k + j];
            if (!gate_q[e] || !gate_s[e] || !up_q[e] || !up_s[e] || !down_q[e] || !down_s[e]) {
                free(y);
                return -1;
            }
            rc = coli_oracle_expert_ffn(xt, H, F, gate_q[e], gate_s[e], up_q[e], up_s[e],
                                        down_q[e], down_s[e], y, NULL);
            if (rc != 0) { free(y); return rc; }
            for (int64_t n = 0; n < H; ++n) ot[n] += topk_w[t * k + j] * y[n];
        }
        if (!gate_q[E] || !gate_s[E] || !up_q[E] || !up_s[E] || !down_q[E] || !down_s[E]) {
            free(y);
            return -1;
        }
        rc = coli_oracle_expert_ffn(xt, H, F, gate_q[E], gate_s[E], up_q[E], up_s[E],
                                    down_q[E], down_s[E], y, NULL);
        if (rc != 0) { free(y); return rc; }
        for (int64_t n = 0; n < H; ++n) ot[n] += y[n];
    }
    free(y);
    return 0;
}

/*
 * Adaptive expert top-p ("colibri解説", section 速度を稼ぐ実用ノブ: the --topp 0.7
 * knob, "adaptive expert top-p", which cuts expert reads by 30-40 %).  The page
 * names the knob and its effect but not its rule; this library reads it as a
 * cut of the routing distribution of the k experts the router selected:
 *   pi_j = s_j / sum_j' s_j'            (unbiased sigmoids of the selected experts)
 *   order the selected experts by pi descending (equal pi: lower expert first)
 *   keep the shortest prefix of that order whose cumulative pi reaches top_p
 *   (at least one expert; top_p >= 1 keeps all k)
 *   w_j = routed_scale * s_j / sum_{kept} s     for kept experts (the router's
 *         renormalisation, taken over the kept set)
 * A dropped expert keeps its slot with index -1 and weight 0.
 */
int coli_oracle_route_top_p(const double* x, int64_t T, int64_t H,
                            const float* w_router, const float* sel_bias, int64_t E, int64_t k,
                            double routed_scale, double top_p, int32_t* topk_idx, double* topk_w)
{
    if (!x || !w_router || !sel_bias || !topk_idx || !topk_w) return -1;
    if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E || !(top_p > 0.0)) return -1;
    double* sig = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * (size_t)E);
    int64_t* order = (int64_t*)malloc(sizeof(int64_t) * (size_t)k);
    char* keep = (char*)malloc((size_t)k);
    if (!sig || !order || !keep) { free(sig); free(order); free(keep); return -1; }
    int rc = coli_oracle_route(x, T, H, w_router, sel_bias, E, k, routed_scale, topk_idx, topk_w, NULL, sig, NULL);
    if (rc != 0) { free(sig); free(order); free(keep); return rc; }
    for (int64_t t = 0; t < T; ++t) {
        int32_t* idx = topk_idx + t * k;
        double* w = topk_w + t * k;
        const double* st = sig + t * E;
        double total = 0.0;
        for (int64_t j = 0; j < k; ++j) total += st[idx[j]];
        /* slots by pi descending, lower expert first on ties (selection sort) */
        for (int64_t j = 0; j < k; ++j) { order[j] = j; keep[j] = 0; }
        for (int64_t a = 0; a < k; ++a) {
            int64_t best = a;
            for (int64_t b = a + 1; b < k; ++b) {
                const double sb = st[idx[order[b]]], sx = st[idx[order[best]]];
                if (sb > sx || (sb == sx && idx[order[b]] < idx[order[best]])) best = b;
            }
            const int64_t tmp = order[a]; order[a] = order[best]; order[best] = tmp;
        }
        double cum = 0.0, kept = 0.0;
        for (int64_t a = 0; a < k; ++a) {
            keep[order[a]] = 1;
            cum += st[idx[order[a]]] / total;
            if (cum >= top_p) break;
        }
        for (int64_t j = 0; j < k; ++j)  /* the router's sum, in slot order, over the kept set */
            if (keep[j]) kept += st[idx[j]];
        for (int64_t j = 0; j < k; ++j) {
            if (keep[j]) {
                w[j] = routed_scale * st[idx[j]] / kept;
            } else {
                idx[j] = -1;
                w[j] = 0.0;
            }
        }
    }
    free(sig); free(order); free(keep);
    return 0;
}

/*
 * The layer with adaptive expert top-p routing: out_t = sum over the kept
 * slots of w[t,j] * FFN_{idx[t,j]}(x_t) + FFN_E(x_t).
 */
int coli_oracle_moe_layer_top_p(const double* x, int64_t T, int64_t H, int64_t F,
                                int64_t E, int64_t k, double routed_scale, double top_p,
                                const float* w_router, const float* sel_bias,
                                const uint8_t* const* gate_q, const float* const* gate_s,
                                const uint8_t* const* up_q, const float* const* up_s,
                                const uint8_t* const* down_q, const float* const* down_s,
                                int32_t* topk_idx, double* topk_w, double* out)
{
    if (!x || !gate_q || !gate_s || !up_q || !up_s || !down_q || !down_s) return -1;
    if (!topk_idx || !topk_w || !out) return -1;
    int rc = coli_oracle_route_top_p(x, T, H, w_router, sel_bias, E, k, routed_scale, top_p, topk_idx, topk_w);
    if (rc != 0) return rc;
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    if (!y) return -1;
    for (int64_t t = 0; t < T; ++t) {
        const double* xt = x + t * H;
        double* ot = out + t * H;
        for (int64_t n = 0; n < H; ++n) ot[n] = 0.0;
        for (int64_t j = 0; j <= k; ++j) {
            const int64_t e = j < k ? topk_idx[t * k + j] : E;
            if (e < 0) continue; /* dropped slot */
            if (!gate_q[e] || !gate_s[e] || !up_q[e] || !up_s[e] || !down_q[e] || !down_s[e]) {
                free(y);
                return -1;
            }
            rc = coli_oracle_expert_ffn(xt, H, F, gate_q[e], gate_s[e], up_q[e], up_s[e],
                                        down_q[e], down_s[e], y, NULL);
            if (rc != 0) { free(y); return rc; }
            const double wj = j < k ? topk_w[t * k + j] : 1.0;
            for (int64_t n = 0; n < H; ++n) ot[n] += wj * y[n];
        }
    }
    free(y);
    return 0;
}

/*
 * Integer-activation variant ("Colibri 完全ガイド", section コア技術のハイライト,
 * row 整数ドット積カーネル: int8 and packed-int4 integer products from u8 x s8
 * pairs, so the activations are int8; the same page's environment table lists
 * the IDOT switch).  The pages name the kernel but not its quantisation rule;
 * this library reads it as symmetric int8 per block of 32 consecutive values:
 *   m = max |x| over the block,  scale = m / 127,
 *   code = rint(x * (127 / m))   (round half to even), in [-127, 127],
 *   x_hat = code * scale;  an all-zero block (or one whose maximum is so small
 *   that 127 / m overflows fp32) has codes 0 and scale 0, and a block holding
 *   inf or NaN has codes 0 and scale NaN.
 * Every step is taken in fp32, the precision the kernel decides the codes in.
 */
#define COLI_ORACLE_I8_BLOCK 32

int coli_oracle_quant_i8(const float* x, int64_t n, int8_t* code, float* scale)
{
    if (!x || !code || !scale || n < 0 || n % COLI_ORACLE_I8_BLOCK != 0) return -1;
    for (int64_t b = 0; b < n / COLI_ORACLE_I8_BLOCK; ++b) {
        const float* xb = x + b * COLI_ORACLE_I8_BLOCK;
        int8_t* cb = code + b * COLI_ORACLE_I8_BLOCK;
        float m = 0.0f;
        int finite = 1;
        for (int i = 0; i < COLI_ORACLE_I8_BLOCK; ++i) {
            if (!isfinite(xb[i])) finite = 0;
            else if (fabsf(xb[i]) > m) m = fabsf(xb[i]);
        }
        if (!finite || m == 0.0f) {
            for (int i = 0; i < COLI_ORACLE_I8_BLOCK; ++i) cb[i] = 0;
            scale[b] = finite ? 0.0f : NAN;
            continue;
        }
        const float inv = 127.0f / m;
        if (!(inv <= FLT_MAX)) { /* a maximum below 127 / FLT_MAX: the block is taken as zero */
            for (int i = 0; i < COLI_ORACLE_I8_BLOCK; ++i) cb[i] = 0;
            scale[b] = 0.0f;
            continue;
        }
        for (int i = 0; i < COLI_ORACLE_I8_BLOCK; ++i) {
            float c = rintf(xb[i] * inv);
            if (c > 127.0f) c = 127.0f;
            if (c < -127.0f) c = -127.0f;
            cb[i] = (int8_t)c;
        }
        scale[b] = m / 127.0f;
    }
    return 0;
}

/* x_hat of a vector of n values (fp32 x given as f64, widened exactly from fp32). */
static int quant_i8_hat(const double* x, int64_t n, double* xh)
{
    if (n <= 0) return -1;
    float* xf = (float*)malloc(sizeof(float) * (size_t)n);
    int8_t* c = (int8_t*)malloc((size_t)n);
    float* s = (float*)malloc(sizeof(float) * (size_t)(n / COLI_ORACLE_I8_BLOCK + 1));
    if (!xf || !c || !s) { free(xf); free(c); free(s); return -1; }
    for (int64_t i = 0; i < n; ++i) xf[i] = (float)x[i];
    int rc = coli_oracle_quant_i8(xf, n, c, s);
    if (rc == 0)
        for (int64_t i = 0; i < n; ++i) xh[i] = (double)c[i] * (double)s[i / COLI_ORACLE_I8_BLOCK];
    free(xf); free(c); free(s);
    return rc;
}

/*
 * One expert with int8 activations: g = Wg x_hat, u = Wu x_hat,
 * h = silu(g) * u (f64, rounded to fp32 before it is quantised, as the kernel
 * holds it), y = Wd h_hat.
 */
static int expert_ffn_i8(const double* x, int64_t H, int64_t F,
                         const uint8_t* gate_q, const float* gate_s, const uint8_t* up_q, const float* up_s,
                         const uint8_t* down_q, const float* down_s, double* y)
{
    double* xh = (double*)malloc(sizeof(double) * (size_t)H);
    double* g = (double*)malloc(sizeof(double) * (size_t)F);
    double* u = (double*)malloc(sizeof(double) * (size_t)F);
    double* a = (double*)malloc(sizeof(double) * (size_t)F);
    double* ah = (double*)malloc(sizeof(double) * (size_t)F);
    int rc = -1;
    if (xh && g && u && a && ah && quant_i8_hat(x, H, xh) == 0) {
        coli_oracle_matvec(gate_q, gate_s, F, H, xh, g);
        coli_oracle_matvec(up_q, up_s, F, H, xh, u);
        for (int64_t f = 0; f < F; ++f) a[f] = (double)(float)(g[f] * sigmoid(g[f]) * u[f]);
        if (quant_i8_hat(a, F, ah) == 0) rc = coli_oracle_matvec(down_q, down_s, H, F, ah, y);
    }
    free(xh); free(g); free(u); free(a); free(ah);
    return rc;
}

/*
 * The layer with int8 activations in every expert: the route is the plain one
 * (the router reads the activations as stored), out_t = sum_j w[t,j] *
 * FFN8_{idx[t,j]}(x_t) + FFN8_E(x_t), FFN8 = expert_ffn_i8.
 */
int coli_oracle_moe_layer_i8(const double* x, int64_t T, int64_t H, int64_t F,
                             int64_t E, int64_t k, double routed_scale,
                             const float* w_router, const float* sel_bias,
                             const uint8_t* const* gate_q, const float* const* gate_s,
                             const uint8_t* const* up_q, const float* const* up_s,
                             const uint8_t* const* down_q, const float* const* down_s,
                             int32_t* topk_idx, double* topk_w, double* out)
{
    if (!x || !gate_q || !gate_s || !up_q || !up_s || !down_q || !down_s) return -1;
    if (!topk_idx || !topk_w || !out) return -1;
    if (H % COLI_ORACLE_I8_BLOCK != 0 || F % COLI_ORACLE_I8_BLOCK != 0) return -1;
    int rc = coli_oracle_route(x, T, H, w_router, sel_bias, E, k, routed_scale, topk_idx, topk_w, NULL, NULL, NULL);
    if (rc != 0) return rc;
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    if (!y) return -1;
    for (int64_t t = 0; t < T; ++t) {
        const double* xt = x + t * H;
        double* ot = out + t * H;
        for (int64_t n = 0; n < H; ++n) ot[n] = 0.0;
        for (int64_t j = 0; j <= k; ++j) {
            const int64_t e = j < k ? topk_idx[t * k + j] : E;
            if (!gate_q[e] || !gate_s[e] || !up_q[e] || !up_s[e] || !down_q[e] || !down_s[e]) {
                free(y);
                return -1;
            }
            rc = expert_ffn_i8(xt, H, F, gate_q[e], gate_s[e], up_q[e], up_s[e], down_q[e], down_s[e], y);
            if (rc != 0) { free(y); return rc; }
            const double wj = j < k ? topk_w[t * k + j] : 1.0;
            for (int64_t n = 0; n < H; ++n) ot[n] += wj * y[n];
        }
    }
    free(y);
    return 0;
}
