/*
 * coli_oracle.h -- plain, slow, f64 CPU statement of the routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This oracle exists to check the CUDA library
 * against the plain definition of what the layer computes.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg may load it.
 * The product path never calls it and it shares no code, header, table or
 * helper with the CUDA library.
 *
 * What is computed (sources are the colibri pages, cited by title and section):
 *   - Route: DeepSeek-V3-style sigmoid router, bias-corrected top-k
 *     ("Colibri 完全ガイド", section コア技術のハイライト, row "DeepSeek-V3 式 Router";
 *      Korean getting-started page, section 토큰당 처리 경로, step "Route").
 *   - Union: tokens of one batch that pick the same expert share one pass over it
 *     (same Korean page and section, step "Union"; "colibri: 744B MoEを
 *      ストレージから推論するCエンジン", section エンドツーエンドの測定で…, "batched expert union").
 *   - Expert FFN on int4 weights with one scale per group of 64 along K
 *     ("colibri: 744B MoE…", section はじめにとソースが語らないこと, "gs64 build";
 *      mcpfield "colibri" page, section コアアーキテクチャ, int4 experts).
 *   - Integer-activation variant: int8 activations per block of 32 into the
 *     expert products ("Colibri 完全ガイド", section コア技術のハイライト, row
 *     整数ドット積カーネル).
 *   - Shared expert, always on, added with weight one
 *     ("Colibri 完全ガイド", same row; Korean page, section 프로젝트 설명, shared experts).
 *
 * Readings where the pages are silent (each stated where it is used below):
 *   nibble order low-first, two's complement [-8,7], fp32 scale per 64 along K,
 *   no zero point; plain top-k over all experts (no group-limited routing);
 *   the bias selects but does not weight; weights renormalised over the k
 *   selected unbiased sigmoids and scaled by routed_scale; ties go to the lower
 *   expert index; expert FFN = SwiGLU, y = W_down (silu(W_gate x) * (W_up x));
 *   shared expert stored at expert index E with the same shapes.
 *
 * All functions return 0 on success and -1 on an invalid argument.
 */
#ifndef COLI_ORACLE_H
#define COLI_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* One element of an int4-gs64 matrix [N, K]: q bytes [N, K/2], s fp32 [N, K/64]. */
double coli_oracle_weight(const uint8_t* q, const float* s, int64_t K, int64_t n, int64_t kk);

/* Dense f64 copy W[N, K] of an int4-gs64 matrix. */
int coli_oracle_dequant(const uint8_t* q, const float* s, int64_t N, int64_t K, double* W);

/* y[N] = W x for an int4-gs64 matrix W [N, K]. */
int coli_oracle_matvec(const uint8_t* q, const float* s, int64_t N, int64_t K,
                       const double* x, double* y);

/* Router for T tokens.  x [T, H] (stored activations widened to f64), w_router
 * fp32 [E, H], sel_bias fp32 [E].  Writes topk_idx [T, k] (descending biased
 * score), topk_w [T, k]; optionally logits, sigmoid scores and biased scores,
 * each [T, E] (pass NULL to skip). */
int coli_oracle_route(const double* x, int64_t T, int64_t H,
                      const float* w_router, const float* sel_bias, int64_t E, int64_t k,
                      double routed_scale, int32_t* topk_idx, double* topk_w,
                      double* logits, double* sig, double* biased);

/* Batch union of the T*k (token, slot) pairs p = t*k + j by expert:
 * count [E], offset [E+1] (exclusive scan of count), active [E] (experts with
 * count > 0, ascending; unused tail set to -1), n_active [1], perm [T*k]
 * (pair ids in (expert, token, slot) order), inv_perm [T*k]. */
int coli_oracle_union(const int32_t* topk_idx, int64_t T, int64_t k, int64_t E,
                      int32_t* count, int32_t* offset, int32_t* active, int32_t* n_active,
                      int32_t* perm, int32_t* inv_perm);

/* One SwiGLU expert on one token: h = silu(Wg x) * (Wu x), y = Wd h.
 * Wg, Wu [F, H]; Wd [H, F]; h [F] optional (NULL to skip). */
int coli_oracle_expert_ffn(const double* x, int64_t H, int64_t F,
                           const uint8_t* gate_q, const float* gate_s,
                           const uint8_t* up_q, const float* up_s,
                           const uint8_t* down_q, const float* down_s,
                           double* y, double* h);

/* Whole layer for T tokens.  The per-expert arrays hold E+1 pointers each
 * (index E = shared expert); an entry may be NULL when no token selects that
 * expert (the call fails with -1 if a NULL expert is needed).
 * out [T, H] = sum_j topk_w[t,j] * FFN_{idx[t,j]}(x_t) + FFN_E(x_t). */
int coli_oracle_moe_layer(const double* x, int64_t T, int64_t H, int64_t F,
                          int64_t E, int64_t k, double routed_scale,
                          const float* w_router, const float* sel_bias,
                          const uint8_t* const* gate_q, const float* const* gate_s,
                          const uint8_t* const* up_q, const float* const* up_s,
                          const uint8_t* const* down_q, const float* const* down_s,
                          int32_t* topk_idx, double* topk_w, double* out);

/* Number of threads the oracle's parallel loops use (1 without OpenMP). */
int coli_oracle_threads(void);

/* Adaptive expert top-p on top of coli_oracle_route (see coli_oracle.c):
 * dropped slots get index -1 and weight 0; kept weights are renormalised over
 * the kept experts.  top_p >= 1 gives coli_oracle_route's result. */
int coli_oracle_route_top_p(const double* x, int64_t T, int64_t H,
                            const float* w_router, const float* sel_bias, int64_t E, int64_t k,
                            double routed_scale, double top_p, int32_t* topk_idx, double* topk_w);

/* The layer with top-p routing (dropped slots contribute nothing). */
int coli_oracle_moe_layer_top_p(const double* x, int64_t T, int64_t H, int64_t F,
                                int64_t E, int64_t k, double routed_scale, double top_p,
                                const float* w_router, const float* sel_bias,
                                const uint8_t* const* gate_q, const float* const* gate_s,
                                const uint8_t* const* up_q, const float* const* up_s,
                                const uint8_t* const* down_q, const float* const* down_s,
                                int32_t* topk_idx, double* topk_w, double* out);

/* Integer-activation variant (see coli_oracle.c): symmetric int8 codes of x
 * [n] (n a multiple of 32), one fp32 scale per block of 32. */
int coli_oracle_quant_i8(const float* x, int64_t n, int8_t* code, float* scale);

/* The layer with int8 activations into every expert matmul (x before gate/up,
 * h before down); the route reads the stored activations. */
int coli_oracle_moe_layer_i8(const double* x, int64_t T, int64_t H, int64_t F,
                             int64_t E, int64_t k, double routed_scale,
                             const float* w_router, const float* sel_bias,
                             const uint8_t* const* gate_q, const float* const* gate_s,
                             const uint8_t* const* up_q, const float* const* up_s,
                             const uint8_t* const* down_q, const float* const* down_s,
                             int32_t* topk_idx, double* topk_w, double* out);

#ifdef __cplusplus
}
#endif
#endif /* COLI_ORACLE_H */
