// gated_attention.cu -- token-gated causal GQA attention over the kept tokens.
//
// TokenGate (aiproducthub.cn article, paragraph 事件详情; aisight.pl article,
// section Jak to działa; chathome.org article, section トークンゲート付き
// アテンションとは): every attention above the gate layer sees only the K kept
// tokens; each kept token's gate score is a bias on the attention logits,
// scaled by a learned per-head gain, and a learned temperature corrects for
// each query seeing fewer keys.  Formula (the specification's):
//   l_{r,c} = tau * (q_r . k_c) / sqrt(d_h) + g_h * s_c,   c <= r
//   O_r = sum_c softmax_c(l_{r,.}) v_c
//
// Kernel: one CTA per (128-query tile, NQ query heads of one GQA group), the
// heaviest query tiles first.  NQ = 2 when the group size is even: the two
// heads share every K/V tile and their softmax warpgroups run side by side, so
// the tensor pipe works on one head while the other head's softmax runs.
// Tiles are 128 queries x 128 keys.
//   warp 0      TMA: the NQ Q tiles once, then K and V tiles into two rings
//               (K runs one tile ahead of V)
//   warp 1      TMEM allocation and the single MMA-issuing thread, per key
//               tile j and head h:
//                 O_h += P_h(j) V_j      (kind::f16, fp16 x fp16 -> fp32; P_h
//                                          read from TMEM, V_j MN-major in smem)
//                 S_h(j+1) = Q_h K_{j+1}^T  (kind::f16, bf16 x bf16 -> fp32)
//               P_h(j) is written over S_h(j)'s own columns, so S_h(j+1) is
//               issued right behind P_h(j) V_j; the tensor pipe runs one
//               thread's MMAs in order, so S_h(j+1) finishing also means
//               P_h(j) V_j has finished and O_h may be rescaled.
//   warp 2      the key-bias operand of each K tile (below)
//   warps 3-6, 7-10   softmax of head 0, head 1 (one query row per thread;
//               warp w owns TMEM lanes 32 (w mod 4) ..): the row's 128 S values
//               are read from TMEM into registers, row max, then
//               P = 2^(S c - m) with c = tau / sqrt(d_h) log2(e), as fp16 into
//               the S columns.
//               Lazy rescaling: O is rescaled (in TMEM) only when a row max
//               grows by more than 2^8, so P <= 256.  Causal masking only on
//               the diagonal tile.  At the end O / l to bf16 and the
//               log-sum-exp.
// The key bias rides in the tensor core: S is computed as
//   S_h = Q_h K^T + A_h B^T,   A_h[r, 3i+k] = gamma_h^(i),   B[c, 3i+k] = s_c^(k)
// (one extra K = 16 MMA step; gamma_h = g_h sqrt(d_h) / tau and s_c each split
// into three bf16 parts whose sum is the fp32 value, so the nine products add
// up to gamma_h s_c to fp32 accuracy), hence S c = tau q.k / sqrt(d_h) log2(e)
// + g_h s_c log2(e): the logit in log2 units, with no per-element bias work.
// This needs c > 0 (tau > 0).
// P in fp16 (11 significant bits) rather than bf16 keeps the P V product's
// relative error below 2^-11 per weight, which bounds the output error for
// large-magnitude values.  V is converted to fp16 once, by a small pass into
// the workspace before the attention kernel (bf16 values in fp16's normal
// range convert without rounding); converting inside the attention kernel would
// redo it for every query tile that reads the V tile.
//
// TMEM columns: S_h (and P_h over it) at 128 h, O_h at 128 NQ + d_h h.  Every
// wait is bounded (TG_STATUS_ATTENTION_TIMEOUT).
#include <cmath>

#include <cfloat>

#include "tg_host.cuh"

namespace tg {
namespace attn {

constexpr int kBM = 128;        // query rows per tile
constexpr int kBN = 128;        // keys per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8

template <int D, int NQ>
struct Cfg {
    static constexpr int kStages = (D == 64) ? 4 : 2;  // depth of the K ring and of the V ring
    static constexpr int kQTile = kBM * D * 2;   // bytes of a 128 x D 16-bit tile
    static constexpr int kKVTile = kBN * D * 2;  // bytes of a 128 x D 16-bit tile
    static constexpr int kChunks = D / 64;       // 64-column (128-byte) swizzle chunks per row
    static constexpr int kSoftmaxWarp0 = 3;
    static constexpr int kThreads = 32 * (kSoftmaxWarp0 + 4 * NQ);
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + NQ * kQTile;
    static constexpr int kOffV = kOffK + kStages * kKVTile;
    // bias operands, 128 rows x 16 bf16 each in the no-swizzle K-major layout (4 KB)
    static constexpr int kAugTile = 4096;
    static constexpr int kOffAugA = kOffV + kStages * kKVTile;  // [NQ]      gamma_h parts, every row alike
    static constexpr int kOffAugB = kOffAugA + NQ * kAugTile;   // [kStages] s_c parts of a K tile's keys
    static constexpr int kOffBar = kOffAugB + kStages * kAugTile;
    static constexpr int kNumBars = 2 + 4 * kStages + 4 * NQ + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmem = kOffMisc + 16 + 1024;
    static constexpr uint32_t kTmemCols = (NQ * kBN + NQ * D > 256) ? 512 : 256;
    static __device__ __forceinline__ uint32_t col_s(int h) { return static_cast<uint32_t>(h * kBN); }
    static __device__ __forceinline__ uint32_t col_o(int h) { return static_cast<uint32_t>(NQ * kBN + h * D); }
};

struct Args {
    int64_t K;
    int Hq, Hkv;
    int num_q_tiles;
    int pairs_per_group;  // (Hq / Hkv) / NQ
    float scale_log2;     // tau / sqrt(d_h) * log2(e)
    const float* s_kept;
    const float* gain;
    __nv_bfloat16* out;
    float* lse;
    unsigned int* status;
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 up2(uint64_t u) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(u));
    return r;
}
// Blackwell paired fp32 arithmetic: two lanes of work per issue slot.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(pk2(a.x, a.y)), "l"(pk2(b.x, b.y)), "l"(pk2(c.x, c.y)));
    return up2(d);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pk2(a.x, a.y)), "l"(pk2(b.x, b.y)));
    return up2(d);
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ uint32_t f16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// x as three bf16 parts (round to nearest at each step); their exact sum is x
// to within fp32's own precision.
__device__ __forceinline__ void split3_bf16(float x, __nv_bfloat16 (&p)[3]) {
    p[0] = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(p[0]);
    p[1] = __float2bfloat16_rn(r1);
    p[2] = __float2bfloat16_rn(r1 - __bfloat162float(p[1]));
}
__device__ __forceinline__ uint32_t bf2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}
// Row r's two 16-byte core-matrix rows of a 128 x 16 no-swizzle K-major tile
// (LBO 128 bytes, SBO 256 bytes), in uint4 units from the tile start.
__device__ __forceinline__ int aug_slot(int r, int chunk) { return (r >> 3) * 16 + chunk * 8 + (r & 7); }

// Instruction descriptor for kind::f16 with fp16 A and B, fp32 accumulator
// (A/B format field 0 = f16; same layout as idesc_bf16_f32 otherwise).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool b_mn_major) {
    return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// Bounded wait whose result is the same on every lane of the warp, so that the
// warp-collective tcgen05.ld/st and shuffles that follow never see a partial warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          unsigned int* status) {
    const bool ok = mbar_wait(bar, parity, abort, status, TG_STATUS_ATTENTION_TIMEOUT);
    return __all_sync(0xffffffffu, ok);
}

template <int D, int NQ>
__global__ void __launch_bounds__(Cfg<D, NQ>::kThreads, 1)
gated_attention_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const Args a) {
    using C = Cfg<D, NQ>;
    constexpr int kStages = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars;                        // TMA -> MMA (one phase per work item)
    uint64_t* q_empty = bars + 1;                   // commit after an item's last S -> TMA (next Q), bias warp
    uint64_t* k_full = bars + 2;                    // [kStages] TMA bytes of K + the bias warp's 32 lanes -> MMA
    uint64_t* k_empty = k_full + kStages;           // [kStages] commit after the last S of a K tile -> TMA
    uint64_t* v_full = k_empty + kStages;           // [kStages] TMA -> MMA
    uint64_t* v_empty = v_full + kStages;           // [kStages] commit after the last P V of a V tile -> TMA
    uint64_t* s_full = v_empty + kStages;           // [NQ] commit after S_h(j) (and P_h(j-1) V) -> softmax h
    uint64_t* p_full = s_full + NQ;                 // [NQ] 128 softmax threads wrote P_h(j) -> MMA
    uint64_t* o_full = p_full + NQ;                 // [NQ] commit after an item's last P_h V -> epilogue h
    uint64_t* o_empty = o_full + NQ;                // [NQ] 128 epilogue threads read O_h -> MMA (next item)
    uint64_t* drain = o_empty + NQ;                 // abort path
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Work items: (128-query tile, NQ query heads of one KV head), heaviest (most key tiles) first.
    // Persistent CTAs take them in snake order -- round r hands item r G + b to CTA b on even
    // rounds and r G + G - 1 - b on odd ones -- which evens out the triangular causal work.
    const int per_tile = a.Hkv * a.pairs_per_group;
    const int n_items = a.num_q_tiles * per_tile;
    const int G = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
    auto item_of = [&](int r) -> int { return r * G + ((r & 1) ? (G - 1 - b) : b); };
    struct Item {
        int m_tile, kvh, head0, n_kv;
    };
    auto decode = [&](int idx) -> Item {
        Item it;
        it.m_tile = a.num_q_tiles - 1 - idx / per_tile;
        const int rem = idx % per_tile;
        it.kvh = rem / a.pairs_per_group;
        it.head0 = it.kvh * (a.Hq / a.Hkv) + (rem % a.pairs_per_group) * NQ;
        it.n_kv = it.m_tile + 1;  // causal: key tiles 0..m_tile, the last one on the diagonal
        return it;
    };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1 + 32);  // the TMA bytes of K, and the 32 lanes writing its bias operand B
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int h = 0; h < NQ; ++h) {
            mbar_init(&s_full[h], 1);
            mbar_init(&p_full[h], 128);
            mbar_init(&o_full[h], 1);
            mbar_init(&o_empty[h], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_trigger();
    pdl_wait();  // global memory is shared with the kernels before this one from here on

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int k_last[kStages], v_last[kStages];  // parity of the last phase loaded per stage, -1 if none
            for (int i = 0; i < kStages; ++i) k_last[i] = v_last[i] = -1;
            int q_last = -1;
            // K (is_k) or V tile j of an item whose first tile is number g0 of this CTA: wait for its ring
            // slot, then one TMA box per 64-column chunk
            auto load_kv = [&](int g0, int j, int kvh, bool is_k) -> bool {
                const int g = g0 + j;
                const int st = g % kStages;
                const uint32_t ph = static_cast<uint32_t>(g / kStages) & 1;
                uint64_t* full = is_k ? k_full : v_full;
                if (!mbar_wait(is_k ? &k_empty[st] : &v_empty[st], ph ^ 1, abort_flag, a.status,
                               TG_STATUS_ATTENTION_TIMEOUT))
                    return false;
                uint8_t* dst = smem + (is_k ? C::kOffK : C::kOffV) + st * C::kKVTile;
                mbar_arrive_expect_tx(&full[st], C::kKVTile);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(dst + c * (kBN * 128), is_k ? &tmap_k : &tmap_v, &full[st], c * 64, kvh, j * kBN,
                                kEvictLast);
                (is_k ? k_last : v_last)[st] = static_cast<int>(ph);
                return true;
            };
            bool ok = true;
            int g0 = 0;
            for (int r = 0, it = 0; ok && r * G < n_items; ++r) {
                const int idx = item_of(r);
                if (idx >= n_items) continue;
                const Item w = decode(idx);
                // Q of this item once the previous item's last S no longer reads the Q tiles
                if (!(ok = mbar_wait(q_empty, (static_cast<uint32_t>(it) & 1) ^ 1, abort_flag, a.status,
                                     TG_STATUS_ATTENTION_TIMEOUT)))
                    break;
                mbar_arrive_expect_tx(q_full, NQ * C::kQTile);
                for (int h = 0; h < NQ; ++h)
#pragma unroll
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(smem + C::kOffQ + h * C::kQTile + c * (kBM * 128), &tmap_q, q_full, c * 64,
                                    w.head0 + h, w.m_tile * kBM, kEvictFirst);
                q_last = it & 1;
                // K runs one tile ahead of V: S(j+1) needs only K(j+1); P(j) V(j) waits for softmax j anyway.
                ok = load_kv(g0, 0, w.kvh, true);
                for (int j = 0; j < w.n_kv && ok; ++j) {
                    if (j + 1 < w.n_kv) ok = load_kv(g0, j + 1, w.kvh, true);
                    if (ok) ok = load_kv(g0, j, w.kvh, false);
                }
                g0 += w.n_kv;
                ++it;
            }
            // Every issued copy must land before shared memory is released (matters on abort only).
            volatile int no_abort = 0;
            if (q_last >= 0)
                mbar_wait(q_full, static_cast<uint32_t>(q_last), &no_abort, a.status, TG_STATUS_ATTENTION_TIMEOUT);
            for (int i = 0; i < kStages; ++i) {
                if (k_last[i] >= 0)
                    mbar_wait(&k_full[i], static_cast<uint32_t>(k_last[i]), &no_abort, a.status,
                              TG_STATUS_ATTENTION_TIMEOUT);
                if (v_last[i] >= 0)
                    mbar_wait(&v_full[i], static_cast<uint32_t>(v_last[i]), &no_abort, a.status,
                              TG_STATUS_ATTENTION_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, false);  // Q K^T: both K-major
            constexpr uint32_t idesc_o = idesc_f16_f32(kBM, D, true);      // P V: V MN-major
            // Descriptors as 32-bit start/LBO words over one shared high word (SBO 1024,
            // 128-byte swizzle): every MMA below moves its operands by compile-time
            // offsets, so the issuing thread keeps ahead of the tensor pipe.
            const uint32_t dhi = sw128_desc_hi(1024);
            const uint32_t q_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffQ), 16);
            const uint32_t k_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffK), 16);
            const uint32_t v_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffV), kBN * 128);
            const uint32_t ahi = noswz_desc_hi(256);
            const uint32_t aa_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffAugA), 128);
            const uint32_t ab_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffAugB), 128);
            const bool bias = a.gain != nullptr && a.s_kept != nullptr;
            // K tile g and its bias operand B both in shared memory (one barrier counts both)
            auto wait_k = [&](int g) -> bool {
                const uint32_t ph = static_cast<uint32_t>(g / kStages) & 1;
                return mbar_wait(&k_full[g % kStages], ph, abort_flag, a.status, TG_STATUS_ATTENTION_TIMEOUT);
            };
            // S_h = Q_h K_g^T into head h's S columns, then signal softmax h (the commit
            // also covers every earlier MMA of this thread, P_h(g-1) V_{g-1} included)
            auto issue_s = [&](int h, int g) {
                const uint32_t q_lo = q_lo0 + static_cast<uint32_t>(h * (C::kQTile >> 4));
                const uint32_t k_lo = k_lo0 + static_cast<uint32_t>((g % kStages) * (C::kKVTile >> 4));
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    // K step k: 64-column chunk k / 4, 32-byte column offset k % 4 inside the swizzle atom
                    const uint32_t qo = static_cast<uint32_t>(((k >> 2) * (kBM * 128) + (k & 3) * 32) >> 4);
                    const uint32_t ko = static_cast<uint32_t>(((k >> 2) * (kBN * 128) + (k & 3) * 32) >> 4);
                    mma_ss_lo(tmem + C::col_s(h), q_lo + qo, k_lo + ko, dhi, idesc_s, k > 0);
                }
                // + A_h B^T: the key bias g_h s_c / c, one more K step (none without a bias)
                if (bias)
                    mma_ss_lo(tmem + C::col_s(h), aa_lo0 + static_cast<uint32_t>(h * (C::kAugTile >> 4)),
                              ab_lo0 + static_cast<uint32_t>((g % kStages) * (C::kAugTile >> 4)), ahi, idesc_s, 1u);
                mma_commit(&s_full[h]);
            };
            bool ok = true;
            int g0 = 0;
            for (int r = 0, it = 0; ok && r * G < n_items; ++r) {
                const int idx = item_of(r);
                if (idx >= n_items) continue;
                const int n_kv = decode(idx).n_kv;
                if (!(ok = mbar_wait(q_full, static_cast<uint32_t>(it) & 1, abort_flag, a.status,
                                     TG_STATUS_ATTENTION_TIMEOUT)))
                    break;
                if (!(ok = wait_k(g0))) break;
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < NQ; ++h) issue_s(h, g0);
                mma_commit(&k_empty[g0 % kStages]);
                if (n_kv == 1) mma_commit(q_empty);
                for (int j = 0; j < n_kv && ok; ++j) {
                    const int g = g0 + j;
                    const int st = g % kStages;
                    const bool more = j + 1 < n_kv;
                    if (!(ok = mbar_wait(&v_full[st], static_cast<uint32_t>(g / kStages) & 1, abort_flag,
                                         a.status, TG_STATUS_ATTENTION_TIMEOUT)))
                        break;
                    if (more && !(ok = wait_k(g + 1))) break;
                    const uint32_t v_lo = v_lo0 + static_cast<uint32_t>(st * (C::kKVTile >> 4));
#pragma unroll
                    for (int h = 0; h < NQ && ok; ++h) {
                        // O_h += P_h(j) V_j once softmax h has written P_h(j) (and, on the item's first
                        // tile, once the previous item's epilogue has read O_h out) ...
                        if (!(ok = mbar_wait(&p_full[h], static_cast<uint32_t>(g) & 1, abort_flag, a.status,
                                             TG_STATUS_ATTENTION_TIMEOUT)))
                            break;
                        if (j == 0 && !(ok = mbar_wait(&o_empty[h], (static_cast<uint32_t>(it) & 1) ^ 1, abort_flag,
                                                       a.status, TG_STATUS_ATTENTION_TIMEOUT)))
                            break;
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < kBN / 16; ++k)  // 16 keys per step: 16 rows of 128 bytes in each chunk
                            mma_ts_lo(tmem + C::col_o(h), tmem + C::col_s(h) + static_cast<uint32_t>(k * 8),
                                      v_lo + static_cast<uint32_t>(k * (2048 >> 4)), dhi, idesc_o,
                                      (j > 0 || k > 0) ? 1u : 0u);
                        // ... then, behind it in the same pipe, S_h(j+1) over the same columns
                        if (more)
                            issue_s(h, g + 1);
                        else
                            mma_commit(&o_full[h]);
                    }
                    if (!ok) break;
                    mma_commit(&v_empty[st]);
                    if (more) mma_commit(&k_empty[(g + 1) % kStages]);
                    if (more && j + 2 == n_kv) mma_commit(q_empty);  // the item's last S is issued
                }
                g0 += n_kv;
                ++it;
            }
            if (!ok) {
                mma_commit(drain);
                volatile int no_abort = 0;
                mbar_wait(drain, 0, &no_abort, a.status, TG_STATUS_ATTENTION_TIMEOUT);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ bias operands A and B
        uint4* aug_a = reinterpret_cast<uint4*>(smem + C::kOffAugA);
        uint4* aug_b = reinterpret_cast<uint4*>(smem + C::kOffAugB);
        // B for K tile g (key tile j of the item): row c holds s_c's parts (k = col mod 3 for col < 9)
        auto fill_aug = [&](int g, int j, const Item& w, int it) -> bool {
            const int st = g % kStages;
            // the tile's key scores are loaded first, so their latency overlaps the wait for the slot
            float sv[kBN / 32];
#pragma unroll
            for (int i = 0; i < kBN / 32; ++i) {
                const int64_t key = static_cast<int64_t>(j) * kBN + i * 32 + lane;
                sv[i] = (a.s_kept && key < a.K) ? __ldg(a.s_kept + key) : 0.0f;
            }
            // the slot is free once the S MMAs of tile g - kStages are done (same release as K)
            if (!mbar_wait(&k_empty[st], (static_cast<uint32_t>(g / kStages) & 1) ^ 1, abort_flag, a.status,
                           TG_STATUS_ATTENTION_TIMEOUT))
                return false;
            if (j == 0) {
                // A_h of this item: every row holds gamma_h's parts (i = col / 3 for col < 9, zeros after),
                // written once the previous item's S MMAs are done (q_empty)
                if (!mbar_wait(q_empty, (static_cast<uint32_t>(it) & 1) ^ 1, abort_flag, a.status,
                               TG_STATUS_ATTENTION_TIMEOUT))
                    return false;
#pragma unroll
                for (int h = 0; h < NQ; ++h) {
                    __nv_bfloat16 gp[3];
                    split3_bf16(a.gain ? a.gain[w.head0 + h] * kLog2e / a.scale_log2 : 0.0f, gp);
                    const __nv_bfloat16 z = __float2bfloat16_rn(0.0f);
                    const uint4 c0 = make_uint4(bf2(gp[0], gp[0]), bf2(gp[0], gp[1]), bf2(gp[1], gp[1]),
                                                bf2(gp[2], gp[2]));
                    const uint4 c1 = make_uint4(bf2(gp[2], z), 0u, 0u, 0u);
                    for (int rr = lane; rr < kBM; rr += 32) {
                        aug_a[h * (C::kAugTile / 16) + aug_slot(rr, 0)] = c0;
                        aug_a[h * (C::kAugTile / 16) + aug_slot(rr, 1)] = c1;
                    }
                }
            }
            uint4* dst = aug_b + st * (C::kAugTile / 16);
#pragma unroll
            for (int i = 0; i < kBN / 32; ++i) {
                const int c = i * 32 + lane;
                __nv_bfloat16 p[3];
                split3_bf16(sv[i], p);
                const __nv_bfloat16 z = __float2bfloat16_rn(0.0f);
                dst[aug_slot(c, 0)] = make_uint4(bf2(p[0], p[1]), bf2(p[2], p[0]), bf2(p[1], p[2]), bf2(p[0], p[1]));
                dst[aug_slot(c, 1)] = make_uint4(bf2(p[2], z), 0u, 0u, 0u);
            }
            fence_proxy_async_smem();  // generic-proxy writes -> tensor-core (async proxy) reads
            mbar_arrive(&k_full[st]);  // B written: with K's bytes this completes the tile's k_full phase
            return true;
        };
        bool ok = true;
        int g0 = 0;
        for (int r = 0, it = 0; ok && r * G < n_items; ++r) {
            const int idx = item_of(r);
            if (idx >= n_items) continue;
            const Item w = decode(idx);
            for (int j = 0; j < w.n_kv && ok; ++j) ok = fill_aug(g0 + j, j, w, it);
            g0 += w.n_kv;
            ++it;
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue of head h
        const int sw = warp - C::kSoftmaxWarp0;
        const int h = sw >> 2;
        const int q = warp & 3;         // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;  // query row inside the tile == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + C::col_s(h);
        const uint32_t o_addr = tmem + lane_off + C::col_o(h);
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
        bool ok = true;
        int g0 = 0;
        for (int r = 0, it = 0; ok && r * G < n_items; ++r) {
            const int idx = item_of(r);
            if (idx >= n_items) continue;
            const int n_kv = a.num_q_tiles - idx / per_tile;  // the item's key tiles (its query tile + 1)
            float m_run = -INFINITY, l_run = 0.0f;
            for (int j = 0; j < n_kv && ok; ++j) {
                if (!(ok = warp_wait(&s_full[h], static_cast<uint32_t>(g0 + j) & 1, abort_flag, a.status))) break;
                tc_fence_after();
                // the row's 128 S values (bias included)
                float x[kBN];
                {
                    uint32_t* xv = reinterpret_cast<uint32_t*>(x);
#pragma unroll
                    for (int c = 0; c < kBN; c += 32)
                        tmem_ld32(s_addr + c, *reinterpret_cast<uint32_t(*)[32]>(xv + c));
                    tmem_ld_wait();
                }
                // on the diagonal tile, key c is in the future of query row r when c > r
                if (j == n_kv - 1) {
#pragma unroll
                    for (int c = 0; c < kBN; ++c)
                        if (c > row) x[c] = -INFINITY;
                }
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < kBN; c += 2) mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], x[c], x[c + 1]);
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * a.scale_log2;
                // lazy rescaling: keep the stale max unless this row's max grew by more than 2^8
                const bool need = mx > m_run + kRescaleThreshold;
                float alpha = 1.0f;
                if (need) {
                    alpha = ex2(m_run - mx);  // 0 on the first tile (m_run = -inf)
                    m_run = mx;
                    l_run *= alpha;
                }
                // S_h(j) complete implies P_h(j-1) V_{j-1} complete: O_h may be rescaled now
                if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld16(o_addr + c0, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                        tmem_st16(o_addr + c0, v);
                    }
                }
                // P = 2^(S c - m) as fp16 over the first kBN / 2 S columns (already read)
                const float2 neg_m = make_float2(-m_run, -m_run);
                float2 ls[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
                for (int c0 = 0; c0 < kBN; c0 += 32) {
                    uint32_t p16[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float2 y0 = ffma2(make_float2(x[c0 + i], x[c0 + i + 1]), sc2, neg_m);
                        const float2 y1 = ffma2(make_float2(x[c0 + i + 2], x[c0 + i + 3]), sc2, neg_m);
                        const float2 p0 = make_float2(ex2(y0.x), ex2(y0.y));
                        const float2 p1 = make_float2(ex2(y1.x), ex2(y1.y));
                        ls[0] = fadd2(ls[0], p0);
                        ls[1] = fadd2(ls[1], p1);
                        p16[i / 2] = f16x2(p0.x, p0.y);
                        p16[i / 2 + 1] = f16x2(p1.x, p1.y);
                    }
                    tmem_st16(s_addr + (c0 >> 1), p16);
                }
                const float2 lsum = fadd2(ls[0], ls[1]);
                tmem_st_wait();
                l_run += lsum.x + lsum.y;
                tc_fence_before();
                mbar_arrive(&p_full[h]);
            }
            if (!ok || !warp_wait(&o_full[h], static_cast<uint32_t>(it) & 1, abort_flag, a.status)) {
                ok = false;
                break;
            }
            // epilogue: normalise, store bf16 rows and the log-sum-exp; O_h's columns are free for the
            // next item once every row has been read out
            tc_fence_after();
            const Item w = decode(idx);
            const int head = w.head0 + h;
            const int64_t grow = static_cast<int64_t>(w.m_tile) * kBM + row;
            const float inv_l = 1.0f / l_run;
            __nv_bfloat16* orow = a.out + (grow * a.Hq + head) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(o_addr + c0, v);
                tmem_ld_wait();
                if (c0 + 32 == D) {
                    tc_fence_before();
                    mbar_arrive(&o_empty[h]);
                }
                if (grow < a.K) {
                    uint32_t o[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        o[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l, __uint_as_float(v[2 * i + 1]) * inv_l);
                    uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                }
            }
            if (a.lse && grow < a.K)
                a.lse[static_cast<int64_t>(head) * a.K + grow] = (m_run + log2f(l_run)) / kLog2e;
            g0 += n_kv;
            ++it;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// V [K, Hkv d_h] bf16 (token stride ld_v) -> dense fp16 [K, Hkv d_h], eight
// elements per 16-byte load and store.  A finite value above fp16's range
// (|v| > 65504) becomes +-inf in the copy; the kernel then sets
// TG_STATUS_V_RANGE in the status word so the caller learns of it.
__global__ void __launch_bounds__(128) v_to_f16_kernel(const uint4* __restrict__ v, int64_t ld_v8, int64_t K,
                                                       int w8, uint4* __restrict__ v16, unsigned int* status) {
    bool out_of_range = false;
    for (int64_t r = blockIdx.x; r < K; r += gridDim.x) {
        for (int c = threadIdx.x; c < w8; c += blockDim.x) {
            const uint4 x = v[r * ld_v8 + c];
            uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xffff0000u);
                out_of_range |= (fabsf(lo) > 65504.0f && fabsf(lo) <= FLT_MAX) || (fabsf(hi) > 65504.0f && fabsf(hi) <= FLT_MAX);
                w[e] = f16x2(lo, hi);
            }
            v16[r * w8 + c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    if (out_of_range) atomicOr(status, TG_STATUS_V_RANGE);
}

template <int D, int NQ>
static tg_status launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, Args a,
                        cudaStream_t st) {
    using C = Cfg<D, NQ>;
    auto kern = gated_attention_kernel<D, NQ>;
    static std::atomic<int> smem_set[64];  // zero before first use (static storage)
    if (!set_max_dynamic_smem(kern, C::kSmem, smem_set))
        return TG_ERR_CUDA;
    a.pairs_per_group = (a.Hq / a.Hkv) / NQ;
    const int64_t items = static_cast<int64_t>(a.num_q_tiles) * a.Hkv * a.pairs_per_group;
    if (items > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    // persistent: one CTA per SM (TMEM and shared memory allow no more), each taking several items
    const int grid = static_cast<int>(std::min<int64_t>(items, num_sms()));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, a) == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

}  // namespace attn
}  // namespace tg

using namespace tg;

// Shared by both entry points: checks, tensor maps and the launch over a dense
// fp16 V ([K, Hkv, d_h]) that is already in device memory.
static tg_status attention_over_v16(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k, const void* v16,
                                    int64_t K, int32_t Hq, int32_t Hkv, int32_t d_h, const float* s_kept,
                                    const float* gain, float tau, tg_bf16* out, float* lse, void* workspace,
                                    cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    const uint32_t qbox[3] = {64, 1, 128};
    const uint32_t kvbox[3] = {64, 1, static_cast<uint32_t>(attn::kBN)};
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(d_h), static_cast<uint64_t>(Hq), static_cast<uint64_t>(K)};
        const uint64_t str[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_q) * 2};
        if (!make_tmap_bf16(&mq, q, 3, dims, str, qbox)) return TG_ERR_CUDA;
    }
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(d_h), static_cast<uint64_t>(Hkv), static_cast<uint64_t>(K)};
        const uint64_t sk[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_k) * 2};
        const uint64_t sv[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(Hkv) * d_h * 2};
        // (the map's element type only matters for fills; the fp16 bits are copied as they are)
        if (!make_tmap_bf16(&mk, k, 3, dims, sk, kvbox) || !make_tmap_bf16(&mv, v16, 3, dims, sv, kvbox))
            return TG_ERR_CUDA;
    }
    attn::Args a;
    a.K = K;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.num_q_tiles = static_cast<int>((K + attn::kBM - 1) / attn::kBM);
    a.pairs_per_group = 1;
    a.scale_log2 = tau / std::sqrt(static_cast<float>(d_h)) * attn::kLog2e;
    a.s_kept = s_kept;
    a.gain = gain;
    a.out = reinterpret_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.status = status_word(workspace);
    const bool pairs = ((Hq / Hkv) % 2) == 0;
    if (d_h == 128) return pairs ? attn::launch<128, 2>(mq, mk, mv, a, st) : attn::launch<128, 1>(mq, mk, mv, a, st);
    return pairs ? attn::launch<64, 2>(mq, mk, mv, a, st) : attn::launch<64, 1>(mq, mk, mv, a, st);
}

static tg_status check_attention_args(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k, int64_t K,
                                      int32_t Hq, int32_t Hkv, int32_t d_h, float tau, const tg_bf16* out) {
    if (K < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || !std::isfinite(tau) || !(tau > 0.0f))
        return TG_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return TG_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(out)) return TG_ERR_INVALID_ARG;
    if (K > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    if (ld_q < static_cast<int64_t>(Hq) * d_h || ld_k < static_cast<int64_t>(Hkv) * d_h || (ld_q % 8) || (ld_k % 8))
        return TG_ERR_INVALID_ARG;
    return TG_OK;
}

extern "C" tg_status tg_gated_attention(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                        const tg_bf16* v, int64_t ld_v, int64_t K, int32_t Hq, int32_t Hkv,
                                        int32_t d_h, const float* s_kept, const float* gain, float tau,
                                        tg_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    const tg_status chk = check_attention_args(q, ld_q, k, ld_k, K, Hq, Hkv, d_h, tau, out);
    if (chk != TG_OK) return chk;
    if (!aligned16(v)) return TG_ERR_INVALID_ARG;
    if (K == 0) return TG_OK;
    if (!q || !k || !v || !out || !workspace || !aligned16(workspace)) return TG_ERR_INVALID_ARG;
    if (workspace_bytes < tg_workspace_bytes(TG_OP_ATTENTION, K, Hkv * d_h, 0)) return TG_ERR_INVALID_ARG;
    if (ld_v < static_cast<int64_t>(Hkv) * d_h || (ld_v % 8)) return TG_ERR_INVALID_ARG;

    // fp16 copy of V in the workspace, dense [K, Hkv, d_h]
    void* v16 = static_cast<char*>(workspace) + ws_gate_offset();
    cudaStream_t st = as_stream(stream);
    {
        const int w8 = Hkv * d_h / 8;
        const int64_t grid = K < static_cast<int64_t>(num_sms()) * 16 ? K : static_cast<int64_t>(num_sms()) * 16;
        attn::v_to_f16_kernel<<<static_cast<unsigned>(grid), 128, 0, st>>>(
            reinterpret_cast<const uint4*>(v), ld_v / 8, K, w8, reinterpret_cast<uint4*>(v16), status_word(workspace));
        if (launch_status() != TG_OK) return TG_ERR_CUDA;
    }
    return attention_over_v16(q, ld_q, k, ld_k, v16, K, Hq, Hkv, d_h, s_kept, gain, tau, out, lse, workspace, st);
}

extern "C" tg_status tg_gated_attention_f16v(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                             const uint16_t* v16, int64_t K, int32_t Hq, int32_t Hkv, int32_t d_h,
                                             const float* s_kept, const float* gain, float tau, tg_bf16* out,
                                             float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    const tg_status chk = check_attention_args(q, ld_q, k, ld_k, K, Hq, Hkv, d_h, tau, out);
    if (chk != TG_OK) return chk;
    if (!aligned16(v16)) return TG_ERR_INVALID_ARG;
    if (K == 0) return TG_OK;
    if (!q || !k || !v16 || !out || !workspace || !aligned16(workspace)) return TG_ERR_INVALID_ARG;
    if (workspace_bytes < tg_workspace_bytes(TG_OP_ATTENTION, 0, Hkv * d_h, 0)) return TG_ERR_INVALID_ARG;
    return attention_over_v16(q, ld_q, k, ld_k, v16, K, Hq, Hkv, d_h, s_kept, gain, tau, out, lse, workspace,
                              as_stream(stream));
}
