/*
 * tg_oracle.h -- plain CPU oracle for the TokenGate prefill hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This library is the checker that the CUDA path
 * (libtokengate) is compared against.  Only the test suite, the smoke check and
 * the CPU-baseline leg of the benchmark may load it; the product path never
 * does, and this code shares no source, header, table or helper with the CUDA
 * kernels.
 *
 * Every routine is single-threaded, written for a reader to check by eye, and
 * computes in fp64.  Floating-point inputs are fp32 arrays; values that are
 * bf16 on the GPU side are passed as their exact fp32 widening, so both sides
 * see the same numbers.
 *
 * Sources (web pages about "TokenGate: learned token pruning for long-context
 * prefill", Patel, Ranjan, Stoica, Zaharia, Guestrin):
 *   - three-phase forward, gate on the post-attention residual at layer L,
 *     top-K keeps the best-scored tokens, upper layers see only K tokens:
 *     aiproducthub.cn article (paragraph 事件详情), aisight.pl article
 *     (section Jak to działa), chathome.org article (section TokenGate の
 *     学習可能なトークンプルーニングの仕組み);
 *   - only the document part of the prompt is prunable, the question never:
 *     same three sections;
 *   - token-gated attention: each kept token's score becomes a bias on the
 *     attention logits above the gate, with a learned per-head gain and a
 *     learned temperature: aiproducthub.cn (paragraph 事件详情), aisight.pl
 *     (section Jak to działa), chathome.org (section トークンゲート付き
 *     アテンションとは).
 * The pages give the ingredients but not the formulas; the formulas below are
 * the task specification's:
 *   gate:  s_i = w2 . SiLU(r_i * (h_i . (gamma*W1)^T) + b1) + b2,
 *          r_i = (mean_c h_ic^2 + eps)^(-1/2)
 *   logit: l_{r,c} = tau * (q_r . k_c) / sqrt(d_h) + g_h * s_c,  c <= r.
 *
 * Parity pins: every routine is pinned by tests under tests/ (closed forms,
 * brute force, library special cases).  The one acknowledged gap is that the
 * absolute gate formula is a specification choice, not a page fact.
 */
#ifndef TG_ORACLE_H
#define TG_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Number of tokens kept: min(k_doc, doc_end-doc_begin) + (N - (doc_end-doc_begin)).
 * Returns -1 for an invalid span or k_doc < 0. */
int64_t tgo_kept_count(int64_t N, int64_t doc_begin, int64_t doc_end, int64_t k_doc);

/* Gate score, fp64.  h: [N, ld_h] row-major (first d columns used).
 * gamma: [d] RMSNorm weight or NULL (= ones).  If fold_gamma_bf16 != 0 the
 * weight actually used is W1'_jc = bf16_rne(fp32(gamma_c * W1_jc)) (the folded
 * bf16 weight that the GPU path feeds its tensor cores); otherwise the exact
 * product gamma_c*W1_jc is used.  W1: [d_g, d].  b1: [d_g] or NULL (= 0).
 * w2: [d_g].  Output: s[N] in fp64.  Returns 0, or -1 on bad arguments. */
int tgo_gate_score(const float* h, int64_t N, int d, int64_t ld_h,
                   const float* gamma, int fold_gamma_bf16, double eps,
                   const float* W1, const float* b1, const float* w2, double b2,
                   int d_g, double* s);

/* Top-K selection over the document span [doc_begin, doc_end).
 * Order: larger score first; -0 equals +0; NaN ranks below every number;
 * equal scores are ordered by lower index first.  The first min(k_doc, N_doc)
 * document tokens in that order are kept, every token outside the span is
 * kept, and the result is written in ascending index order.
 * kept: room for tgo_kept_count(...) entries.  Returns the count written, or
 * -1 on bad arguments. */
int64_t tgo_topk_select(const float* scores, int64_t N, int64_t doc_begin,
                        int64_t doc_end, int64_t k_doc, int32_t* kept);

/* The k_doc-th document score in the selection order (the threshold), as
 * fp64; NaN if k_doc == 0 or the span is empty.  Used to express the
 * "within 1e-4 of the K-th threshold" acceptance rule. */
/* Random-K selector: the k_doc document tokens with the largest keys, key of
 * token i = top 32 bits of the (i + 1)-th SplitMix64 output from state `seed`
 * (lower index first on equal keys), plus every token outside the span,
 * ascending.  Returns the count written or -1. */
int64_t tgo_random_select(int64_t N, int64_t doc_begin, int64_t doc_end, int64_t k_doc,
                          uint64_t seed, int32_t* kept);
/* n successive SplitMix64 outputs from `state` (the generator itself). */
int tgo_splitmix64_stream(uint64_t state, int64_t n, uint64_t* out);

double tgo_topk_threshold(const float* scores, int64_t N, int64_t doc_begin,
                          int64_t doc_end, int64_t k_doc);

/* Compaction: h_out[r,:] = h[idx[r],:] (raw 16-bit patterns, bit-exact),
 * pos_out[r] = pos_in ? pos_in[idx[r]] : idx[r],
 * s_out[r] = scores[idx[r]] when both pointers are non-NULL.
 * Returns 0, or -1 if an index is out of range. */
int tgo_gather_compact(const uint16_t* h, int64_t N, int d, int64_t ld_h,
                       const int32_t* idx, int64_t K, const int32_t* pos_in,
                       const float* scores, uint16_t* h_out, int32_t* pos_out,
                       float* s_out);

/* Rotate-half rotary embedding at the given positions, fp64.
 * x: [K, H, d_h]; pairs (t, t + d_h/2); angle = pos * base^(-2t/d_h).
 * out: [K, H, d_h] fp64. */
int tgo_rope(const float* x, int64_t K, int H, int d_h, const int32_t* pos,
             double base, double* out);

/* Projection of the kept rows, fp64: out[r, j] = sum_c x[r, c] * W[j, c].
 * x: [K, ld_x] row-major (first d columns used); W: [n_out, d] (one row per
 * output feature, so stacked Wq, Wk, Wv give Q, K, V as column blocks);
 * out: [K, n_out].  Returns 0, or -1 on bad arguments. */
int tgo_project(const float* x, int64_t K, int d, int64_t ld_x,
                const float* W, int n_out, double* out);

/* Token-gated causal GQA attention, fp64, for a subset of query rows.
 * q: [K, Hq, d_h], k and v: [K, Hkv, d_h]; query head h reads kv head
 * h / (Hq/Hkv).  s: [K] kept-token scores or NULL (= 0); g: [Hq] or NULL (= 0).
 * Key c is visible to query r iff pos[c] <= pos[r] (pos NULL: c <= r).
 * rows: [n_rows] query row indices, or NULL for all K rows (n_rows ignored).
 * out: [n_rows, Hq, d_h]; lse: [n_rows, Hq] natural-log sum of exp(logits),
 * or NULL.  Returns 0, or -1 on bad arguments. */
int tgo_gated_attention(const float* q, const float* k, const float* v,
                        int64_t K, int Hq, int Hkv, int d_h,
                        const int32_t* pos, const float* s, const float* g,
                        double tau, const int64_t* rows, int64_t n_rows,
                        double* out, double* lse);

/* Gradients of token-gated attention, fp64, over all K rows (test
 * infrastructure for the backward kernels).  The pages give the reason the
 * bias exists -- it is the scorer's gradient path, and the per-head gain and
 * the temperature are learned (aiproducthub.cn article, paragraph 事件详情;
 * aisight.pl article, section Jak to działa; chathome.org article, section
 * トークンゲート付きアテンションとは) -- so the quantities are the derivatives
 * of the loss sum_{r,h,t} dout[r,h,t] * out[r,h,t] with respect to q, k, v,
 * the kept scores s, the gains g and tau, by the chain rule through the
 * forward of tgo_gated_attention (same arguments, same visibility rule).
 * dout: [K, Hq, d_h].  Outputs: dq [K, Hq, d_h], dk and dv [K, Hkv, d_h],
 * ds [K], dg [Hq], dtau [1]; ds, dg, dtau may be NULL.  s NULL or g NULL
 * means 0 (their gradients are still defined and returned).
 * Returns 0, or -1 on bad arguments. */
int tgo_gated_attention_backward(const float* q, const float* k, const float* v,
                                 int64_t K, int Hq, int Hkv, int d_h,
                                 const int32_t* pos, const float* s, const float* g,
                                 double tau, const float* dout,
                                 double* dq, double* dk, double* dv,
                                 double* ds, double* dg, double* dtau);

/* Round an fp32 value to the nearest bf16 (ties to even), returned widened to
 * fp32.  NaN stays NaN.  Exposed so tests can state bf16 inputs exactly. */
float tgo_round_bf16(float x);

#ifdef __cplusplus
}
#endif

#endif /* TG_ORACLE_H */
