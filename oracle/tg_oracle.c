/*
 * tg_oracle.c -- plain fp64 CPU oracle for the TokenGate prefill hot path.
 *
 * TEST INFRASTRUCTURE ONLY (see tg_oracle.h): loaded by the tests, the smoke
 * check and the CPU-baseline leg of the benchmark, never by the product path.
 * Shares nothing with the CUDA sources.
 *
 * Each function follows one step of the method as the TokenGate pages state
 * it, with the specification's formulas where the pages only name the
 * ingredients.  No blocking, fusion or reordering: loops run in the order of
 * the definition so that a reader can check them by eye.
 */
#include "tg_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

int64_t tgo_kept_count(int64_t N, int64_t doc_begin, int64_t doc_end, int64_t k_doc)
{
    if (N < 0 || doc_begin < 0 || doc_end < doc_begin || doc_end > N || k_doc < 0)
        return -1;
    int64_t n_doc = doc_end - doc_begin;
    int64_t keep_doc = k_doc < n_doc ? k_doc : n_doc;
    return keep_doc + (N - n_doc);
}

float tgo_round_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
        u |= 0x00400000u; /* quiet NaN, keep it NaN after truncation */
        u &= 0xffff0000u;
    } else {
        /* round to nearest, ties to even, on the upper 16 bits */
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7fffu + lsb;
        u &= 0xffff0000u;
    }
    float y;
    memcpy(&y, &u, 4);
    return y;
}

/* ------------------------------------------------------------------------ */
/* Gate score.  The pages: a small MLP scores each token from its
 * post-attention residual at the gate layer (aiproducthub.cn article,
 * paragraph 事件详情; chathome.org article, section TokenGate の学習可能な
 * トークンプルーニングの仕組み).  The MLP shape is the specification's:
 * RMSNorm -> Linear(d -> d_g) -> SiLU -> Linear(d_g -> 1). */
int tgo_gate_score(const float* h, int64_t N, int d, int64_t ld_h,
                   const float* gamma, int fold_gamma_bf16, double eps,
                   const float* W1, const float* b1, const float* w2, double b2,
                   int d_g, double* s)
{
    if (!h || !W1 || !w2 || !s || N < 0 || d <= 0 || d_g <= 0 || ld_h < d)
        return -1;

    /* Effective first-layer weight: gamma folded in (RMSNorm weight times W1). */
    double* W = (double*)malloc(sizeof(double) * (size_t)d_g * (size_t)d);
    if (!W)
        return -1;
    for (int j = 0; j < d_g; ++j) {
        for (int c = 0; c < d; ++c) {
            double w = W1[(size_t)j * d + c];
            if (gamma) {
                if (fold_gamma_bf16)
                    w = tgo_round_bf16((float)(gamma[c] * W1[(size_t)j * d + c]));
                else
                    w = (double)gamma[c] * (double)W1[(size_t)j * d + c];
            }
            W[(size_t)j * d + c] = w;
        }
    }

    for (int64_t i = 0; i < N; ++i) {
        const float* hi = h + i * ld_h;
        /* RMSNorm: r_i = 1 / sqrt(mean_c h_ic^2 + eps) */
        double ss = 0.0;
        for (int c = 0; c < d; ++c)
            ss += (double)hi[c] * (double)hi[c];
        double r = 1.0 / sqrt(ss / (double)d + eps);

        double si = b2;
        for (int j = 0; j < d_g; ++j) {
            /* u_ij = r_i * sum_c h_ic * W_jc + b1_j */
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += (double)hi[c] * W[(size_t)j * d + c];
            double u = r * acc + (b1 ? (double)b1[j] : 0.0);
            /* SiLU(u) = u * sigmoid(u) */
            double a = u / (1.0 + exp(-u));
            si += a * (double)w2[j];
        }
        s[i] = si;
    }
    free(W);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Top-K over the document span; the question (and anything else outside the
 * span) is always kept (aiproducthub.cn article, paragraph 事件详情;
 * chathome.org article, section TokenGate の学習可能なトークンプルーニングの
 * 仕組み).  Tie rule and ascending output order
 * are the specification's. */
static const float* g_sort_scores; /* qsort has no context argument */

/* Negative when token a ranks before token b. */
static int rank_cmp(const void* pa, const void* pb)
{
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    float sa = g_sort_scores[a], sb = g_sort_scores[b];
    int na = isnan(sa), nb = isnan(sb);
    if (na != nb)
        return na ? 1 : -1;          /* every number ranks above NaN */
    if (!na && sa != sb)             /* C comparison: -0 == +0 */
        return sa > sb ? -1 : 1;     /* larger score first */
    return (a > b) - (a < b);        /* lower index first */
}

static int64_t sort_doc(const float* scores, int64_t doc_begin, int64_t doc_end, int32_t** out)
{
    int64_t n_doc = doc_end - doc_begin;
    int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_doc > 0 ? n_doc : 1));
    if (!order)
        return -1;
    for (int64_t i = 0; i < n_doc; ++i)
        order[i] = (int32_t)(doc_begin + i);
    g_sort_scores = scores;
    qsort(order, (size_t)n_doc, sizeof(int32_t), rank_cmp);
    *out = order;
    return n_doc;
}

int64_t tgo_topk_select(const float* scores, int64_t N, int64_t doc_begin,
                        int64_t doc_end, int64_t k_doc, int32_t* kept)
{
    int64_t K = tgo_kept_count(N, doc_begin, doc_end, k_doc);
    if (K < 0 || !kept || (N > 0 && !scores) || N > 2147483647)
        return -1;
    int32_t* order = NULL;
    int64_t n_doc = sort_doc(scores, doc_begin, doc_end, &order);
    if (n_doc < 0)
        return -1;
    int64_t keep_doc = k_doc < n_doc ? k_doc : n_doc;

    unsigned char* keep = (unsigned char*)calloc((size_t)(N > 0 ? N : 1), 1);
    if (!keep) {
        free(order);
        return -1;
    }
    for (int64_t i = 0; i < N; ++i)
        if (i < doc_begin || i >= doc_end)
            keep[i] = 1;
    for (int64_t r = 0; r < keep_doc; ++r)
        keep[order[r]] = 1;

    int64_t n = 0;
    for (int64_t i = 0; i < N; ++i)
        if (keep[i])
            kept[n++] = (int32_t)i;
    free(keep);
    free(order);
    return n;
}

/* ------------------------------------------------------------------------ */
/* Random-K selector.  The pages compare TokenGate with keeping K document
 * tokens chosen at random (a budget-matched random baseline).  The draw is
 * SplitMix64 (Steele, Lea and Flood; the constants of Vigna's reference code):
 * the state advances by 0x9E3779B97F4A7C15 per output, and an output is the
 * new state through z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
 * z *= 0x94D049BB133111EB; z ^= z >> 31.  Token i draws the (i + 1)-th output
 * of the stream started at state `seed`; a document token's key is that
 * output's top 32 bits, and the k_doc largest keys are kept (the lower index
 * first on equal keys), with every token outside the span. */
uint64_t tgo_splitmix64_next(uint64_t* state)
{
    *state += 0x9E3779B97F4A7C15ull;
    uint64_t z = *state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

int tgo_splitmix64_stream(uint64_t state, int64_t n, uint64_t* out)
{
    if (n < 0 || (n > 0 && !out))
        return -1;
    for (int64_t i = 0; i < n; ++i)
        out[i] = tgo_splitmix64_next(&state);
    return 0;
}

static const uint32_t* g_rkeys; /* comparator context (single-threaded oracle) */

static int cmp_rkey(const void* a, const void* b)
{
    int32_t i = *(const int32_t*)a, j = *(const int32_t*)b;
    if (g_rkeys[i] != g_rkeys[j])
        return g_rkeys[i] > g_rkeys[j] ? -1 : 1; /* larger key first */
    return i < j ? -1 : (i > j);                 /* then lower index */
}

int64_t tgo_random_select(int64_t N, int64_t doc_begin, int64_t doc_end, int64_t k_doc,
                          uint64_t seed, int32_t* kept)
{
    int64_t K = tgo_kept_count(N, doc_begin, doc_end, k_doc);
    if (K < 0 || !kept || N > 2147483647)
        return -1;
    uint32_t* keys = (uint32_t*)malloc((size_t)(N > 0 ? N : 1) * sizeof(uint32_t));
    int32_t* order = (int32_t*)malloc((size_t)(N > 0 ? N : 1) * sizeof(int32_t));
    unsigned char* keep = (unsigned char*)calloc((size_t)(N > 0 ? N : 1), 1);
    if (!keys || !order || !keep) {
        free(keys);
        free(order);
        free(keep);
        return -1;
    }
    uint64_t state = seed;
    for (int64_t i = 0; i < N; ++i)
        keys[i] = (uint32_t)(tgo_splitmix64_next(&state) >> 32);
    int64_t n_doc = doc_end - doc_begin;
    for (int64_t r = 0; r < n_doc; ++r)
        order[r] = (int32_t)(doc_begin + r);
    g_rkeys = keys;
    qsort(order, (size_t)n_doc, sizeof(int32_t), cmp_rkey);
    int64_t keep_doc = k_doc < n_doc ? k_doc : n_doc;
    for (int64_t r = 0; r < keep_doc; ++r)
        keep[order[r]] = 1;
    int64_t n = 0;
    for (int64_t i = 0; i < N; ++i)
        if (keep[i] || i < doc_begin || i >= doc_end) /* every token outside the span is kept */
            kept[n++] = (int32_t)i;
    free(keys);
    free(order);
    free(keep);
    return n;
}

double tgo_topk_threshold(const float* scores, int64_t N, int64_t doc_begin,
                          int64_t doc_end, int64_t k_doc)
{
    if (tgo_kept_count(N, doc_begin, doc_end, k_doc) < 0)
        return NAN;
    int32_t* order = NULL;
    int64_t n_doc = sort_doc(scores, doc_begin, doc_end, &order);
    if (n_doc <= 0 || k_doc == 0) {
        free(order);
        return NAN;
    }
    int64_t keep_doc = k_doc < n_doc ? k_doc : n_doc;
    double t = scores[order[keep_doc - 1]];
    free(order);
    return t;
}

/* ------------------------------------------------------------------------ */
/* Compaction: the layers above the gate see only the kept rows, and pruned
 * tokens get no KV entries (aiproducthub.cn article, paragraph 事件详情;
 * chathome.org article, section TokenGate の学習可能なトークンプルーニングの
 * 仕組み).  Original positions
 * travel with the rows so that RoPE stays correct (specification). */
int tgo_gather_compact(const uint16_t* h, int64_t N, int d, int64_t ld_h,
                       const int32_t* idx, int64_t K, const int32_t* pos_in,
                       const float* scores, uint16_t* h_out, int32_t* pos_out,
                       float* s_out)
{
    if (!h || !idx || !h_out || !pos_out || d <= 0 || ld_h < d || K < 0)
        return -1;
    for (int64_t r = 0; r < K; ++r) {
        int64_t i = idx[r];
        if (i < 0 || i >= N)
            return -1;
        memcpy(h_out + r * (int64_t)d, h + i * ld_h, sizeof(uint16_t) * (size_t)d);
        pos_out[r] = pos_in ? pos_in[i] : (int32_t)i;
        if (scores && s_out)
            s_out[r] = scores[i];
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Rotary embedding at original positions (rotate-half pairing, the Qwen3
 * convention; the pages are silent on positions, the specification keeps
 * the original position ids through compaction). */
int tgo_rope(const float* x, int64_t K, int H, int d_h, const int32_t* pos,
             double base, double* out)
{
    if (!x || !pos || !out || K < 0 || H <= 0 || d_h <= 0 || (d_h & 1))
        return -1;
    int half = d_h / 2;
    for (int64_t r = 0; r < K; ++r) {
        for (int hh = 0; hh < H; ++hh) {
            const float* xr = x + (r * H + hh) * (int64_t)d_h;
            double* o = out + (r * H + hh) * (int64_t)d_h;
            for (int t = 0; t < half; ++t) {
                double inv_freq = pow(base, -2.0 * (double)t / (double)d_h);
                double ang = (double)pos[r] * inv_freq;
                double c = cos(ang), s = sin(ang);
                double x1 = xr[t], x2 = xr[t + half];
                o[t] = x1 * c - x2 * s;
                o[t + half] = x2 * c + x1 * s;
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Q/K/V projection of the kept rows.  Above the gate only the kept tokens
 * are processed and only they produce keys and values (aiproducthub.cn
 * article, paragraph 事件详情; chathome.org article, section TokenGate の
 * 学習可能なトークンプルーニングの仕組み), so the next layer's projections
 * run on the compacted rows.  A linear map with no bias (Qwen3's attention
 * projections), weight in the nn.Linear layout, one row per output feature:
 *   out[r, j] = sum_c x[r, c] * W[j, c].
 * Stacking Wq, Wk, Wv as the rows of W gives Q, K and V as consecutive
 * column blocks of out. */
int tgo_project(const float* x, int64_t K, int d, int64_t ld_x,
                const float* W, int n_out, double* out)
{
    if (!x || !W || !out || K < 0 || d <= 0 || n_out <= 0 || ld_x < d)
        return -1;
    for (int64_t r = 0; r < K; ++r) {
        const float* xr = x + r * ld_x;
        for (int j = 0; j < n_out; ++j) {
            const float* wj = W + (size_t)j * (size_t)d;
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += (double)xr[c] * (double)wj[c];
            out[r * n_out + j] = acc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Token-gated attention: the kept token's score becomes a bias on the
 * attention logits, plus a learned per-head gain and a learned temperature
 * (aiproducthub.cn article, paragraph 事件详情; aisight.pl article, section
 * Jak to działa; chathome.org article, section トークンゲート付きアテンション
 * とは).  Formula from the specification:
 *   l_{r,c} = tau * (q_r . k_c) / sqrt(d_h) + g_h * s_c   for visible c,
 *   O_r = sum_c softmax_c(l_{r,.}) v_c. */
int tgo_gated_attention(const float* q, const float* k, const float* v,
                        int64_t K, int Hq, int Hkv, int d_h,
                        const int32_t* pos, const float* s, const float* g,
                        double tau, const int64_t* rows, int64_t n_rows,
                        double* out, double* lse)
{
    if (!q || !k || !v || !out || K < 0 || Hq <= 0 || Hkv <= 0 || d_h <= 0 || (Hq % Hkv))
        return -1;
    if (!rows)
        n_rows = K;
    int group = Hq / Hkv;
    double scale = tau / sqrt((double)d_h);
    double* logit = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    if (!logit)
        return -1;

    for (int64_t n = 0; n < n_rows; ++n) {
        int64_t r = rows ? rows[n] : n;
        if (r < 0 || r >= K) {
            free(logit);
            return -1;
        }
        for (int h = 0; h < Hq; ++h) {
            int kvh = h / group;
            const float* qr = q + (r * Hq + h) * (int64_t)d_h;
            double gain = g ? (double)g[h] : 0.0;

            /* logits of the visible keys, and their maximum */
            double m = -INFINITY;
            for (int64_t c = 0; c < K; ++c) {
                int visible = pos ? (pos[c] <= pos[r]) : (c <= r);
                if (!visible) {
                    logit[c] = -INFINITY;
                    continue;
                }
                const float* kc = k + (c * Hkv + kvh) * (int64_t)d_h;
                double dot = 0.0;
                for (int t = 0; t < d_h; ++t)
                    dot += (double)qr[t] * (double)kc[t];
                double l = scale * dot + gain * (s ? (double)s[c] : 0.0);
                logit[c] = l;
                if (l > m)
                    m = l;
            }

            /* softmax-weighted sum of values */
            double* o = out + (n * Hq + h) * (int64_t)d_h;
            for (int t = 0; t < d_h; ++t)
                o[t] = 0.0;
            double denom = 0.0;
            for (int64_t c = 0; c < K; ++c) {
                if (logit[c] == -INFINITY)
                    continue;
                double p = exp(logit[c] - m);
                denom += p;
                const float* vc = v + (c * Hkv + kvh) * (int64_t)d_h;
                for (int t = 0; t < d_h; ++t)
                    o[t] += p * (double)vc[t];
            }
            for (int t = 0; t < d_h; ++t)
                o[t] /= denom;
            if (lse)
                lse[n * Hq + h] = m + log(denom);
        }
    }
    free(logit);
    return 0;
}

/* Backward of the token-gated logit and the softmax-weighted sum, one query
 * row and head at a time, straight from the chain rule:
 *   P_c   = exp(l_c - lse)                      (softmax over visible keys)
 *   out   = sum_c P_c v_c
 *   dP_c  = dout . v_c                          (d loss / d P_c)
 *   dl_c  = P_c (dP_c - sum_c' P_c' dP_c')      (softmax Jacobian)
 *   l_c   = tau (q . k_c) / sqrt(d_h) + g_h s_c, so
 *   dq   += dl_c tau / sqrt(d_h) k_c,   dk_c += dl_c tau / sqrt(d_h) q,
 *   dv_c += P_c dout,                    ds_c += dl_c g_h,
 *   dg_h += dl_c s_c,                    dtau += dl_c (q . k_c) / sqrt(d_h). */
int tgo_gated_attention_backward(const float* q, const float* k, const float* v,
                                 int64_t K, int Hq, int Hkv, int d_h,
                                 const int32_t* pos, const float* s, const float* g,
                                 double tau, const float* dout,
                                 double* dq, double* dk, double* dv,
                                 double* ds, double* dg, double* dtau)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv || K < 0 || Hq <= 0 || Hkv <= 0 || d_h <= 0 ||
        (Hq % Hkv))
        return -1;
    int group = Hq / Hkv;
    double inv_sqrt_d = 1.0 / sqrt((double)d_h);
    double scale = tau * inv_sqrt_d;
    memset(dq, 0, sizeof(double) * (size_t)K * Hq * d_h);
    memset(dk, 0, sizeof(double) * (size_t)K * Hkv * d_h);
    memset(dv, 0, sizeof(double) * (size_t)K * Hkv * d_h);
    if (ds)
        memset(ds, 0, sizeof(double) * (size_t)K);
    if (dg)
        memset(dg, 0, sizeof(double) * (size_t)Hq);
    double dtau_sum = 0.0;
    size_t n = (size_t)(K > 0 ? K : 1);
    double* dot = (double*)malloc(sizeof(double) * n);   /* q . k_c */
    double* prob = (double*)malloc(sizeof(double) * n);  /* logit, then P_c */
    double* dprob = (double*)malloc(sizeof(double) * n); /* dP_c */
    if (!dot || !prob || !dprob) {
        free(dot);
        free(prob);
        free(dprob);
        return -1;
    }

    for (int h = 0; h < Hq; ++h) {
        int kv_head = h / group;
        double gain = g ? (double)g[h] : 0.0;
        for (int64_t r = 0; r < K; ++r) {
            const float* qr = q + (r * Hq + h) * (int64_t)d_h;
            const float* dor = dout + (r * Hq + h) * (int64_t)d_h;
            /* keys 0..last are the candidates; key c is visible iff VISIBLE(c) */
#define VISIBLE(c) (pos ? (pos[(c)] <= pos[r]) : ((c) <= r))

            /* forward again: logits of the visible keys, their maximum, the softmax */
            double m = -INFINITY;
            for (int64_t c = 0; c < K; ++c) {
                if (!VISIBLE(c))
                    continue;
                const float* kc = k + (c * Hkv + kv_head) * (int64_t)d_h;
                double d = 0.0;
                for (int t = 0; t < d_h; ++t)
                    d += (double)qr[t] * (double)kc[t];
                dot[c] = d;
                prob[c] = scale * d + gain * (s ? (double)s[c] : 0.0);
                if (prob[c] > m)
                    m = prob[c];
            }
            double denom = 0.0;
            for (int64_t c = 0; c < K; ++c) {
                if (!VISIBLE(c))
                    continue;
                prob[c] = exp(prob[c] - m);
                denom += prob[c];
            }

            /* P_c, d loss / d P_c, and the P-weighted mean of the latter */
            double mean = 0.0;
            for (int64_t c = 0; c < K; ++c) {
                if (!VISIBLE(c))
                    continue;
                prob[c] /= denom;
                const float* vc = v + (c * Hkv + kv_head) * (int64_t)d_h;
                double d = 0.0;
                for (int t = 0; t < d_h; ++t)
                    d += (double)dor[t] * (double)vc[t];
                dprob[c] = d;
                mean += prob[c] * d;
            }

            /* through the softmax and the logit to every input */
            double* dqr = dq + (r * Hq + h) * (int64_t)d_h;
            for (int64_t c = 0; c < K; ++c) {
                if (!VISIBLE(c))
                    continue;
                double dl = prob[c] * (dprob[c] - mean);
                const float* kc = k + (c * Hkv + kv_head) * (int64_t)d_h;
                double* dkc = dk + (c * Hkv + kv_head) * (int64_t)d_h;
                double* dvc = dv + (c * Hkv + kv_head) * (int64_t)d_h;
                for (int t = 0; t < d_h; ++t) {
                    dqr[t] += dl * scale * (double)kc[t];
                    dkc[t] += dl * scale * (double)qr[t];
                    dvc[t] += prob[c] * (double)dor[t];
                }
                if (ds)
                    ds[c] += dl * gain;
                if (dg)
                    dg[h] += dl * (s ? (double)s[c] : 0.0);
                dtau_sum += dl * dot[c] * inv_sqrt_d;
            }
#undef VISIBLE
        }
    }
    if (dtau)
        *dtau = dtau_sum;
    free(dot);
    free(prob);
    free(dprob);
    return 0;
}
