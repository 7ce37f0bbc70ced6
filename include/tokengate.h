/*
 * tokengate.h -- C ABI of libtokengate, the B200 (sm_100a) prefill hot path
 * of TokenGate (learned token pruning for long-context prefill).
 *
 * The method, as the TokenGate pages describe it (aiproducthub.cn article,
 * paragraph 事件详情; aisight.pl article, section Jak to działa; chathome.org
 * article, sections TokenGate の学習可能なトークンプルーニングの仕組み and
 * トークンゲート付きアテンションとは):
 *   1. layers below the gate layer L process all N prompt tokens;
 *   2. at layer L a small MLP scores every token from its post-attention
 *      residual, and a top-K selector keeps the best-scored document tokens;
 *      the question part of the prompt is never pruned;
 *   3. layers above L process only the K kept tokens and create no KV entries
 *      for the pruned ones;
 *   4. in every attention above the gate, a kept token's score is a bias on
 *      the attention logits, scaled by a learned per-head gain, with a learned
 *      temperature that accounts for each query seeing fewer keys.
 * The pages name these ingredients but print no formulas; the formulas used
 * here are fixed by the specification and restated at each entry point.
 *
 * The four calls below are steps 2-4; tg_rope_apply is the rotary embedding
 * applied at the tokens' original positions between the projections and the
 * attention.
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates or frees device memory.  Scratch space is a caller-owned
 *     device buffer of tg_workspace_bytes() bytes ("workspace"), zero-filled
 *     once before its first use; a successful call leaves it ready for the
 *     next call.  One workspace may be shared by all calls on one stream.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work and returns; none synchronizes, except
 *     tg_device_status, which reads the workspace's status word back.
 *   - bf16 tensors are passed as tg_bf16 (the 16-bit pattern of a bfloat16).
 *   - Arguments are checked on the host before anything is launched:
 *     TG_ERR_INVALID_ARG for NULL pointers, negative sizes, bad spans,
 *     misaligned pointers; TG_ERR_UNSUPPORTED for shapes the kernels do not
 *     implement (there is no fallback path); TG_ERR_CUDA when a launch fails.
 *   - Kernels that wait on other thread blocks or on asynchronous copies wait
 *     at most about one second; on timeout they set a bit in the workspace's
 *     status word and return early (results are then undefined).
 *     tg_device_status reports it as TG_ERR_TIMEOUT; re-zero the workspace
 *     before reusing it after a timeout.
 *   - tg_gate_score, tg_topk_select, tg_gather_compact, tg_rope_apply and
 *     tg_gated_attention may be captured in a CUDA graph: they neither
 *     synchronize nor allocate, and the kept count is known on the host.
 */
#ifndef TOKENGATE_H
#define TOKENGATE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t tg_bf16;

typedef enum {
    TG_OK = 0,
    TG_ERR_INVALID_ARG = 1,
    TG_ERR_UNSUPPORTED = 2,
    TG_ERR_CUDA = 3,
    TG_ERR_TIMEOUT = 4,
    TG_ERR_RANGE = 5
} tg_status;

typedef enum {
    TG_OP_GATE = 0,
    TG_OP_SELECT = 1,
    TG_OP_ATTENTION = 2,
    TG_OP_ALL = 3, /* one buffer usable by every call above */
    TG_OP_DECODE = 4,
    TG_OP_ATTENTION_BACKWARD = 5,
    TG_OP_PROJECT = 6
} tg_op;

/* Bits of the device status word (first 4 bytes of the workspace). */
#define TG_STATUS_SELECT_TIMEOUT 0x1u
#define TG_STATUS_GATE_TIMEOUT 0x2u
#define TG_STATUS_ATTENTION_TIMEOUT 0x4u
#define TG_STATUS_DECODE_TIMEOUT 0x8u
#define TG_STATUS_BACKWARD_TIMEOUT 0x10u
#define TG_STATUS_PROJECT_TIMEOUT 0x20u
/* Not a timeout: a value of V beyond fp16's range (|v| > 65504) was written
 * into an fp16 copy of V (tg_gated_attention, tg_project_rope); the outputs
 * that read it are not the specified values. */
#define TG_STATUS_V_RANGE 0x40u
/* Not a timeout: a row index outside [0, N) was given to
 * tg_project_rope_gather; that row was read from row 0 instead. */
#define TG_STATUS_INDEX_RANGE 0x80u
#define TG_STATUS_TIMEOUT_BITS 0x3fu

/* Static description of a status code.  Never NULL. */
const char* tg_status_string(tg_status status);

/* Library version as major*10000 + minor*100 + patch. */
int32_t tg_version(void);

/* Number of kept tokens (host-only, pure): min(k_doc, doc_end - doc_begin)
 * document tokens plus every token outside the document span.  Returns -1 if
 * the span is not inside [0, N] or k_doc < 0. */
int64_t tg_kept_count(int64_t N, int64_t doc_begin, int64_t doc_end, int64_t k_doc);

/* Workspace bytes needed by `op` (arguments an op does not use are ignored):
 *   TG_OP_GATE       N tokens of hidden size d, gate width d_g
 *   TG_OP_SELECT     N scores
 *   TG_OP_ATTENTION  N = K kept tokens, d = Hkv * d_h (the width of one
 *                    token's V row; the workspace holds an fp16 copy of V)
 *   TG_OP_ALL        every op above with these N, d, d_g (attention over at
 *                    most N tokens whose V rows are at most d wide)
 *   TG_OP_DECODE     tg_gated_decode with d = Hq query heads (N, d_g unused)
 *   TG_OP_ATTENTION_BACKWARD  tg_gated_attention_backward with N = K kept
 *                    tokens, d = Hq query heads, d_g = Hkv KV heads
 *   TG_OP_PROJECT    tg_project_rope with N = K kept tokens, d = d_h
 * Returns 0 for bad arguments. */
size_t tg_workspace_bytes(tg_op op, int64_t N, int32_t d, int32_t d_g);

/* Gate score (step 2: a small MLP on the post-attention residual):
 *   r_i = (mean_c h_ic^2 + eps)^(-1/2)
 *   u_ij = r_i * sum_c h_ic * W_jc + b1_j,   W = W1, or bf16(rms_weight (.) W1)
 *   s_i = sum_j SiLU(u_ij) * w2_j + b2,      SiLU(u) = u / (1 + e^-u)
 * h: [N, d] bf16, row stride ld_h elements (ld_h >= d, multiple of 8).
 * rms_weight: [d] bf16 RMSNorm weight, or NULL for ones.  When given it is
 *   folded into W1 once per call as bf16(rms_weight_c * W1_jc) (one rounding).
 * W1: [d_g, d] bf16 row-major.  b1: [d_g] fp32 or NULL (zeros).
 * w2: [d_g] fp32.  b2: scalar.  scores: [N] fp32 output.
 * Supported: d a multiple of 64 (64..16384), d_g in {64, 128, 256},
 * N in [0, 2^31).  h, W1 16-byte aligned.
 * Tensor cores (tcgen05, bf16 in, fp32 accumulate in TMEM); the RMS factor,
 * bias, SiLU and the d_g -> 1 projection are applied in the epilogue.  With
 * d_g = 256 two CTAs of a cluster share each 256-row tile (one M = 256 MMA per
 * step, each CTA holding half of W1), where the device offers clusters of 2. */
tg_status tg_gate_score(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h,
                        const tg_bf16* rms_weight, float eps,
                        const tg_bf16* W1, const float* b1, const float* w2, float b2,
                        int32_t d_g, float* scores,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Top-K selection (step 2: top-K keeps the best-scored tokens; only the
 * document part of the prompt is prunable, the question never is):
 * keeps the first min(k_doc, doc_end - doc_begin) document tokens in the
 * order (score descending, index ascending), where -0 == +0 and NaN ranks
 * below every number, plus every token outside [doc_begin, doc_end).
 * kept_idx: int32 output of tg_kept_count(...) entries, ascending.
 * The result is unique, so it is bit-exact with any correct implementation.
 * Supported: N < 2^31 and doc_end - doc_begin <= 2424832 (148 * 1024 * 16).
 * Multi-pass radix select (11/11/10-bit digits of the order-preserving key
 * of each fp32 score) in one launch: spans of up to 16 * 1024 * 16 = 262144
 * tokens (131072 on a device that offers clusters of 8 only) in one
 * thread-block cluster that merges its histograms through distributed shared
 * memory, longer spans in one cooperative grid that merges them in the
 * workspace.  The cluster shape writes nothing but kept_idx and waits only at
 * hardware cluster barriers; the workspace is still required. */
tg_status tg_topk_select(const float* scores, int64_t N, int64_t doc_begin,
                         int64_t doc_end, int64_t k_doc, int32_t* kept_idx,
                         void* workspace, size_t workspace_bytes, void* stream);

/* The gate and the select as a pair on one workspace, for the path where the
 * select runs right after the gate: tg_gate_score_for_select is tg_gate_score
 * (same arguments, same scores bit for bit) that also counts, in its
 * epilogue, the scores of the rows in [doc_begin, doc_end) by the top 11 bits
 * of their order-preserving key -- the select's first radix pass -- into the
 * workspace's select scratch; tg_topk_select_after_gate is tg_topk_select
 * (same arguments and result) that starts from that count instead of making
 * the first pass itself, and leaves the count at zero again.  Call them in
 * this order, on the same stream and workspace, with the same scores, N and
 * span; a tg_topk_select_after_gate without its gate call, or two gate calls
 * in a row, select from a wrong count.  The workspace is the gate's
 * (tg_workspace_bytes(TG_OP_GATE, N, d, d_g), which holds the select
 * scratch); after a timeout it must be zero-filled again, as for every call. */
tg_status tg_gate_score_for_select(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h,
                                   const tg_bf16* rms_weight, float eps,
                                   const tg_bf16* W1, const float* b1, const float* w2, float b2,
                                   int32_t d_g, float* scores, int64_t doc_begin, int64_t doc_end,
                                   void* workspace, size_t workspace_bytes, void* stream);
tg_status tg_topk_select_after_gate(const float* scores, int64_t N, int64_t doc_begin,
                                    int64_t doc_end, int64_t k_doc, int32_t* kept_idx,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* tg_topk_select_after_gate that also writes the kept tokens' scores:
 * s_kept[i] = scores[kept_idx[i]] ([tg_kept_count(...)] fp32, in the order of
 * kept_idx) -- the compacted scores the attention's key bias reads, so no
 * separate compaction pass is needed for them.  Same call order, workspace
 * and errors as tg_topk_select_after_gate; s_kept must not be NULL when the
 * kept count is positive. */
tg_status tg_topk_select_after_gate_kept_scores(const float* scores, int64_t N, int64_t doc_begin, int64_t doc_end,
                                                int64_t k_doc, int32_t* kept_idx, float* s_kept, void* workspace,
                                                size_t workspace_bytes, void* stream);

/* Top-K selection that allocates nothing and takes no workspace.
 * There is no counterpart on the TokenGate pages: this is a calling-convention
 * variant of tg_topk_select for callers that cannot allocate device memory
 * when they select (code running inside an allocator or memory-pool callback,
 * a serving process whose device memory is fully reserved up front by its own
 * pool, a host environment that only lends the library the buffers it owns).
 * Same arguments (minus the workspace), same result, bit for bit, as
 * tg_topk_select.
 * Scratch: a static device array of 34,560 bytes inside the library, which
 * every GPU that loads the library keeps until the process exits.  The first
 * call on each device looks up that array's device address (with the device
 * current), so make the first call on a device before any stream capture.
 * Every call shares the array and clears it on the stream before use; calls
 * that overlap on the GPU (different streams, or several host threads) race
 * on it and must be serialised by the caller.  It never calls cudaMalloc,
 * cudaFree or any allocating routine.
 * Limit: doc_end - doc_begin <= #SMs * 1024 * 16 (2,424,832 on a 148-SM B200,
 * the largest grid the select kernel uses); longer spans return
 * TG_ERR_UNSUPPORTED before anything is launched.
 * A device-side wait that times out leaves kept_idx undefined and sets
 * TG_STATUS_SELECT_TIMEOUT in the array's status word, which
 * tg_topk_select_noalloc_status reads back; this entry point itself reports
 * launch errors only. */
tg_status tg_topk_select_noalloc(const float* scores, int64_t N, int64_t doc_begin,
                                 int64_t doc_end, int64_t k_doc, int32_t* kept_idx,
                                 void* stream);

/* The status word the last tg_topk_select_noalloc call on the current device
 * left in its static array (each call clears it first): synchronizes `stream`
 * (the stream of that call), writes the raw TG_STATUS_* bits to *status_word
 * (may be NULL) and returns TG_ERR_TIMEOUT if a timeout bit is set, TG_OK
 * otherwise.  Allocates nothing. */
tg_status tg_topk_select_noalloc_status(uint32_t* status_word, void* stream);

/* Random-K selector (the pages' budget-matched random baseline): keeps
 * min(k_doc, doc_end - doc_begin) document tokens chosen at random, plus every
 * token outside [doc_begin, doc_end), as ascending indices (the same output as
 * tg_topk_select).  Token i's key is the top 32 bits of the (i + 1)-th output
 * of a SplitMix64 stream started at state `seed` (state += 0x9E3779B97F4A7C15;
 * z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
 * z ^= z >> 31); the largest keys are kept, the lower index first on equal
 * keys, so the result is a deterministic function of the seed.  Workspace,
 * sizes, errors and limits as tg_topk_select (the same kernel, keys drawn in
 * registers instead of read from scores). */
tg_status tg_random_select(int64_t N, int64_t doc_begin, int64_t doc_end, int64_t k_doc, uint64_t seed,
                           int32_t* kept_idx, void* workspace, size_t workspace_bytes, void* stream);

/* Compaction (step 3: layers above the gate see only the K kept tokens):
 *   h_out[r, :] = h[kept_idx[r], :]           (bit-exact copy)
 *   pos_out[r]  = pos_in ? pos_in[kept_idx[r]] : kept_idx[r]
 *   s_out[r]    = scores[kept_idx[r]]          (if both are non-NULL)
 * h: [N, d] bf16 with row stride ld_h; h_out: [K, d] contiguous.
 * kept_idx entries are checked on the device: an entry outside [0, N) is not
 * read; its h_out row is zero-filled, pos_out gets -1 and s_out (if given)
 * NaN, so any negative pos_out marks a bad index (-2: a row copy that did not
 * complete within the library's wait limit).
 * Supported: d a multiple of 8; h, h_out 16-byte aligned, ld_h multiple of 8.
 * One launch: rows up to 20 KB (d <= 10240) move by the bulk-copy engine, one
 * row per lane and 32 rows per SM in flight; wider rows by 16-byte loads. */
tg_status tg_gather_compact(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h,
                            const int32_t* kept_idx, int64_t K, const int32_t* pos_in,
                            const float* scores, tg_bf16* h_out, int32_t* pos_out,
                            float* s_out, void* stream);

/* Rotary embedding at the original positions, in place (rotate-half pairing
 * (t, t + d_h/2), angle pos * base^(-2t/d_h) computed in fp64, cos/sin
 * rounded to fp32, rotation in fp32, result rounded to bf16).
 * q: [K, Hq, d_h] with token stride ld_q; k: [K, Hkv, d_h] with stride ld_k
 * (strides in elements, multiples of 8; heads contiguous inside a token).
 * pos: [K] int32.  Supported: d_h in {64, 128}. */
tg_status tg_rope_apply(tg_bf16* q, int64_t ld_q, tg_bf16* k, int64_t ld_k,
                        const int32_t* pos, int64_t K, int32_t Hq, int32_t Hkv,
                        int32_t d_h, double base, void* stream);

/* Token-gated causal GQA attention over the K kept tokens (step 4):
 *   l_{r,c} = tau * (q_{r,h} . k_{c,kv(h)}) / sqrt(d_h) + gain_h * s_c,  c <= r
 *   out_{r,h} = sum_c softmax_c(l_{r,.}) v_{c,kv(h)},  kv(h) = h / (Hq / Hkv)
 * Causality on compacted indices equals causality on original positions
 * because the kept indices are ascending.
 * q: [K, Hq, d_h], k and v: [K, Hkv, d_h] bf16, token strides ld_q, ld_k,
 * ld_v (elements, multiples of 8).  s_kept: [K] fp32 or NULL (no bias).
 * gain: [Hq] fp32 or NULL (zeros).  out: [K, Hq, d_h] bf16 contiguous.
 * lse: [Hq, K] fp32 natural-log sum of exp of the logits, or NULL.
 * tau > 0 (TG_ERR_INVALID_ARG otherwise).  workspace: at least
 * tg_workspace_bytes(TG_OP_ATTENTION, K, Hkv * d_h, 0) bytes.
 * Supported: d_h in {64, 128}, Hq a multiple of Hkv, K < 2^31.
 * Two launches: V to fp16 into the workspace, then the attention kernel:
 * tensor cores for Q K^T (the key bias added by one extra MMA step) and P V
 * (tcgen05, accumulators in TMEM), K/V tiles staged by TMA, online softmax in
 * fp32, P and V in fp16 for the P V product.
 * Range: V goes through fp16, so |v| must stay within 65504 (fp16's largest
 * finite value; bf16 reaches 3.4e38).  A larger finite v has no fp16 value:
 * the conversion sets TG_STATUS_V_RANGE in the workspace's status word
 * (tg_device_status then returns TG_ERR_RANGE), and the outputs of the query
 * heads that read that KV head are undefined (any of their rows may hold
 * non-finite values). */
tg_status tg_gated_attention(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                             const tg_bf16* v, int64_t ld_v, int64_t K, int32_t Hq,
                             int32_t Hkv, int32_t d_h, const float* s_kept,
                             const float* gain, float tau, tg_bf16* out, float* lse,
                             void* workspace, size_t workspace_bytes, void* stream);

/* tg_gated_attention over a V that is already an fp16 copy, as
 * tg_project_rope writes it: one launch, no conversion pass.
 * v16: [K, Hkv, d_h] fp16 (uint16_t bit patterns), dense, 16-byte aligned.
 * workspace: at least tg_workspace_bytes(TG_OP_ATTENTION, 0, Hkv * d_h, 0)
 * bytes (the status word; no per-call region).  Every other argument, the
 * formula and the limits are those of tg_gated_attention. */
tg_status tg_gated_attention_f16v(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                  const uint16_t* v16, int64_t K, int32_t Hq, int32_t Hkv, int32_t d_h,
                                  const float* s_kept, const float* gain, float tau, tg_bf16* out,
                                  float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* One decoding step of token-gated attention over a KV cache (the layers
 * above the gate layer keep only the kept tokens' keys, each with its gate
 * score as a logit bias; a new token's key carries its own score):
 *   l_c = tau * (q_h . k_{c,kv(h)}) / sqrt(d_h) + gain_h * s_c,   c < T
 *   out_h = sum_c softmax_c(l_c) v_{c,kv(h)},  kv(h) = h / (Hq / Hkv)
 * The query attends to all T keys in the cache (the new token's own key is
 * the last one), so there is no mask.
 * q: [Hq, d_h] bf16 (one token, heads contiguous).  k_cache, v_cache:
 * [T, Hkv, d_h] bf16 with token strides ld_k, ld_v (elements, multiples of
 * 8).  s_cache: [T] fp32 or NULL (no bias); gain: [Hq] fp32 or NULL.
 * out: [Hq, d_h] bf16.  lse: [Hq] fp32 natural-log sum of exp, or NULL.
 * workspace: tg_workspace_bytes(TG_OP_DECODE, 0, Hq, 0) bytes, zero-filled
 * once; concurrent calls must not share one.
 * Supported: d_h in {64, 128}, Hq / Hkv in {1, 2, 4, 8}, Hkv <= 64, 1 <= T <
 * 2^31; q, k_cache, v_cache, s_cache 16-byte aligned.  One launch;
 * every cache row is read once (HBM-bound), fp32 softmax and accumulation.
 * Waits on copies are bounded (TG_STATUS_DECODE_TIMEOUT in the workspace's
 * status word; re-zero the workspace after a timeout). */
tg_status tg_gated_decode(const tg_bf16* q, const tg_bf16* k_cache, int64_t ld_k, const tg_bf16* v_cache,
                          int64_t ld_v, int64_t T, int32_t Hq, int32_t Hkv, int32_t d_h,
                          const float* s_cache, const float* gain, float tau, tg_bf16* out, float* lse,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Gradients of tg_gated_attention (the gradient path the key bias gives the
 * scorer, with the learned per-head gain and temperature: aiproducthub.cn
 * article, paragraph 事件详情; aisight.pl article, section Jak to działa;
 * chathome.org article, section トークンゲート付きアテンションとは).  With
 * l_{r,c} = tau q_r.k_c / sqrt(d_h) + g_h s_c (c <= r), P = softmax_c(l),
 * O = P V, an upstream gradient dO and D_r = dO_r . O_r:
 *   dl = P (dO V^T - D)
 *   dq = tau / sqrt(d_h) dl K,   dk = tau / sqrt(d_h) dl^T Q,   dv = P^T dO
 *   ds_c = sum_h g_h sum_r dl_{h,r,c},   dg_h = sum_{r,c} dl_{h,r,c} s_c,
 *   dtau = sum_{h,r,c} dl_{h,r,c} q_r.k_c / sqrt(d_h)
 * (GQA: dk and dv sum over the query heads of each KV head).
 * q, k, v, K, Hq, Hkv, d_h, s_kept, gain, tau: as given to the forward call.
 * out: the forward's output, dout: the gradient of the loss with respect to
 * it, both [K, Hq, d_h] bf16 dense; lse: the forward's [Hq, K] fp32
 * log-sum-exp (required).  Outputs: dq [K, Hq, d_h], dk and dv [K, Hkv, d_h]
 * bf16 dense; ds [K], dg [Hq], dtau [1] fp32, each may be NULL.  Without a
 * bias (s_kept or gain NULL) the missing one counts as 0: ds is then 0 and dg
 * is still defined.
 * workspace: tg_workspace_bytes(TG_OP_ATTENTION_BACKWARD, K, Hq, Hkv) bytes,
 * 16-byte aligned; every part of it is rewritten by each call (no zeroing).
 * Supported: d_h in {64, 128}, Hq / Hkv <= 8, tau > 0; every bf16 tensor
 * 16-byte aligned, strides multiples of 8 elements.  Four launches: D and the
 * log2 lse; the dq kernel (per query tile and head); the dk/dv kernel (per key
 * tile and KV head, which also sums ds and dg); the final fixed-order sums.
 * Both main kernels recompute S on the tensor cores (tcgen05, TMEM
 * accumulators, TMA-staged tiles) with P and dS in bf16.  Deterministic: the
 * same inputs give the same bits.  Waits are bounded
 * (TG_STATUS_BACKWARD_TIMEOUT in the workspace's status word). */
tg_status tg_gated_attention_backward(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                      const tg_bf16* v, int64_t ld_v, int64_t K, int32_t Hq, int32_t Hkv,
                                      int32_t d_h, const float* s_kept, const float* gain, float tau,
                                      const tg_bf16* out, const tg_bf16* dout, const float* lse,
                                      tg_bf16* dq, tg_bf16* dk, tg_bf16* dv, float* ds, float* dg,
                                      float* dtau, void* workspace, size_t workspace_bytes, void* stream);

/* The Q/K/V projection of the kept rows with the rotary embedding fused into
 * the GEMM epilogue (layers above the gate see only the kept tokens, rotated
 * at their original positions; aiproducthub.cn article, paragraph 事件详情):
 *   qkv[r, :] = x[r, :] W^T, then for every query and key head the
 *   rotate-half pairs (t, t + d_h/2) turned by pos[r] * base^(-2t/d_h),
 *   from the fp32 accumulators (the angle formed and reduced modulo 2 pi in
 *   fp64, its cos / sin in fp32: within 6e-7 of tg_rope_apply's);
 *   value heads are stored as they are, and also in fp16 into v16.
 * x: [K, d] bf16, row stride ld_x (multiple of 8).  W: [(Hq + 2 Hkv) d_h, d]
 * bf16 (query heads, then key heads, then value heads, as an nn.Linear
 * weight).  pos: [K] int32.  qkv: [K, (Hq + 2 Hkv) d_h] bf16, row stride
 * ld_qkv (multiple of 8).  v16: [K, Hkv d_h] fp16 (uint16 bit patterns)
 * dense, or NULL.  workspace: tg_workspace_bytes(TG_OP_PROJECT, K, d_h, 0)
 * bytes (the status word).
 * Supported: d a multiple of 64; (Hq + 2 Hkv) d_h a multiple of 256; d_h in
 * {64, 128}; x, W, qkv, v16 16-byte aligned.  One launch: a persistent
 * tcgen05 GEMM over CTA pairs (256 x 256 tiles, each CTA of a pair loading
 * its own rows and half of W's tile by TMA, TMEM accumulators double-buffered
 * against the epilogue), or over single CTAs (128 x 256 tiles) where a pair
 * cannot be resident.
 * Waits are bounded (TG_STATUS_PROJECT_TIMEOUT).  A value head element above
 * fp16's range (|v| > 65504) written into v16 sets TG_STATUS_V_RANGE. */
tg_status tg_project_rope(const tg_bf16* x, int64_t K, int32_t d, int64_t ld_x, const tg_bf16* W, int32_t Hq,
                          int32_t Hkv, int32_t d_h, const int32_t* pos, double base, tg_bf16* qkv, int64_t ld_qkv,
                          uint16_t* v16, void* workspace, size_t workspace_bytes, void* stream);

/* tg_project_rope whose rows are gathered from h on the way into the GEMM
 * (the compaction of the kept rows fused into the projection's operand
 * loads): x[r, :] = h[rows[r], :], fetched by TMA gather4 copies (four rows
 * of 128 bytes per copy) straight into the tensor-core operand tiles, so the
 * compacted rows are never written out.
 * h: [N, d] bf16, row stride ld_h (multiple of 8), 16-byte aligned.
 * rows: [K] int32 indices into h (the kept indices from the select).  An
 * index outside [0, N) is not followed: row 0 is read in its place and
 * TG_STATUS_INDEX_RANGE is set in the workspace's status word.
 * Every other argument, the outputs, the workspace and the limits are those
 * of tg_project_rope (pos: the rows' original positions; pass `rows` itself
 * when the positions are the indices). */
tg_status tg_project_rope_gather(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h, const int32_t* rows, int64_t K,
                                 const tg_bf16* W, int32_t Hq, int32_t Hkv, int32_t d_h, const int32_t* pos,
                                 double base, tg_bf16* qkv, int64_t ld_qkv, uint16_t* v16, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Test hook (fault injection without a fault): sets the time limit of the
 * grid barrier inside tg_topk_select, tg_topk_select_noalloc and
 * tg_random_select on the current device to `ns` nanoseconds of %globaltimer
 * (0 restores the default of about one second).  With a limit of a few
 * nanoseconds a call's blocks stop waiting for one another, set
 * TG_STATUS_SELECT_TIMEOUT and return before writing any result; the
 * workspace must then be zero-filled again.  No other wait in the library is
 * affected (the others also guard asynchronous copies in flight).
 * Synchronous; not for use while a select may be running. */
tg_status tg_debug_set_select_wait_limit(uint64_t ns);

/* Test hook: with enabled = 0 the gate (d_g = 256) and the projection
 * (tg_project_rope, tg_project_rope_gather) run their one-CTA kernels instead
 * of the CTA-pair kernels they use where the device offers clusters of 2, so
 * that tests can check both shapes on one device; 1 restores the default.
 * Process-wide; not for use while another thread launches those calls. */
tg_status tg_debug_set_cta_pairs(int enabled);

/* Reads the workspace's status word after synchronizing `stream`.
 * *status_word receives the raw TG_STATUS_* bits (may be NULL).
 * Returns TG_ERR_TIMEOUT if a timeout bit is set, else TG_ERR_RANGE if
 * TG_STATUS_V_RANGE or TG_STATUS_INDEX_RANGE is set, TG_OK otherwise. */
tg_status tg_device_status(const void* workspace, uint32_t* status_word, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TOKENGATE_H */
