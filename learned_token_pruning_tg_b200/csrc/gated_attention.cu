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
// heads share every K/V tile and their softmax warpgroups run side by side.
//   warp 0      TMA: the NQ Q tiles once, then K and V tiles of 64 keys into
//               two 4-stage rings (K runs one tile ahead of V)
//   warp 1      TMEM allocation and the single MMA-issuing thread:
//                 S_h = Q_h K_j^T   (kind::f16 bf16 x bf16 -> fp32, N = 64)
//                 O_h += P_h V_j    (kind::f16 fp16 x fp16 -> fp32; P_h read
//                                    from TMEM, V_j MN-major from smem)
//               S_h(j+1) is issued as soon as softmax h has read S_h(j), so it
//               runs while softmax h computes P_h(j): the MMA latency stays off
//               the softmax's critical path.
//   warps 2-3   convert each V tile to fp16 in place in shared memory (the
//               swizzled layout is unchanged because both types are 2 bytes)
//   warps 4+4h  softmax of head h, one query row per thread: the 64 S values of
//               the row are read from TMEM once into registers, x = S tau /
//               sqrt(d_h) log2(e) + g_h s_c log2(e) (key bias from a per-tile
//               shared vector whose scores are prefetched a tile ahead), row
//               max, P = 2^(x - m) as fp16 into TMEM.  Lazy rescaling: O is
//               rescaled (in TMEM) only when a row max grows by more than 2^8,
//               so P <= 256.  Causal masking only on the diagonal tiles.  At
//               the end O / l to bf16 and the log-sum-exp.
// P in fp16 (11 significant bits) rather than bf16 keeps the P V product's
// relative error below 2^-11 per weight, which bounds the output error for
// large-magnitude values; V is converted exactly (bf16 values in fp16's normal
// range convert without rounding).
//
// TMEM columns: S_h at 64 h, P_h at 128 + 32 h, O_h at 256 + d_h h (512 in all
// for two heads of 128).  Every wait is bounded (TG_STATUS_ATTENTION_TIMEOUT).
#include <cmath>

#include "tg_host.cuh"

namespace tg {
namespace attn {

constexpr int kBM = 128;    // query rows per tile
constexpr int kBN = 64;     // keys per tile
constexpr int kStages = 4;  // depth of the K ring and of the V ring
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8

template <int D, int NQ>
struct Cfg {
    static constexpr int kQTile = kBM * D * 2;   // bytes of a 128 x D 16-bit tile
    static constexpr int kKVTile = kBN * D * 2;  // bytes of a 64 x D 16-bit tile
    static constexpr int kChunks = D / 64;       // 64-column (128-byte) swizzle chunks per row
    static constexpr int kThreads = 32 * (4 + 4 * NQ);
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + NQ * kQTile;
    static constexpr int kOffV = kOffK + kStages * kKVTile;
    static constexpr int kOffBias = kOffV + kStages * kKVTile;  // float [NQ][2][64]
    static constexpr int kOffBar = kOffBias + NQ * 2 * kBN * 4;
    static constexpr int kNumBars = 1 + 5 * kStages + 6 * NQ + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmem = kOffMisc + 16 + 1024;
    static constexpr uint32_t kTmemCols = (NQ == 2) ? 512 : 256;
    static __device__ __forceinline__ uint32_t col_s(int h) { return static_cast<uint32_t>(h * kBN); }
    static __device__ __forceinline__ uint32_t col_p(int h) { return static_cast<uint32_t>(NQ * kBN + h * (kBN / 2)); }
    static __device__ __forceinline__ uint32_t col_o(int h) {
        return static_cast<uint32_t>((NQ == 2 ? 256 : 128) + h * D);
    }
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
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* bias_s = reinterpret_cast<float*>(smem + C::kOffBias);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars;                      // TMA -> MMA
    uint64_t* k_full = bars + 1;                  // [kStages] TMA -> MMA
    uint64_t* k_empty = k_full + kStages;         // [kStages] commit after the last S of a K tile -> TMA
    uint64_t* v_full = k_empty + kStages;         // [kStages] TMA -> converters
    uint64_t* v_ready = v_full + kStages;         // [kStages] 64 converter threads -> MMA
    uint64_t* v_empty = v_ready + kStages;        // [kStages] commit after the last P V of a V tile -> TMA
    uint64_t* s_full = v_empty + kStages;         // [NQ] commit after S_h(j) -> softmax h
    uint64_t* s_empty = s_full + NQ;              // [NQ] 128 softmax threads read S_h(j) -> MMA
    uint64_t* p_full = s_empty + NQ;              // [NQ] 128 softmax threads wrote P_h(j) -> MMA
    uint64_t* pv_done = p_full + NQ;              // [NQ] commit after P_h(j) V_j -> softmax h, epilogue
    uint64_t* bias_full = pv_done + NQ;           // [NQ][2] 128 softmax threads (key-bias vector written)
    uint64_t* drain = bias_full + 2 * NQ;         // abort path
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_tile = a.Hkv * a.pairs_per_group;
    const int m_tile = a.num_q_tiles - 1 - static_cast<int>(blockIdx.x / per_tile);  // heaviest first
    const int rem = static_cast<int>(blockIdx.x % per_tile);
    const int kvh = rem / a.pairs_per_group;
    const int head0 = kvh * (a.Hq / a.Hkv) + (rem % a.pairs_per_group) * NQ;
    // causal: key tiles 0..n_kv-1; the last kBM / kBN of them touch the diagonal
    const int n_kv = static_cast<int>((static_cast<int64_t>(m_tile + 1) * kBM + kBN - 1) / kBN);
    const int first_diag = (m_tile * kBM) / kBN;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_ready[s], 64);
            mbar_init(&v_empty[s], 1);
        }
        for (int h = 0; h < NQ; ++h) {
            mbar_init(&s_full[h], 1);
            mbar_init(&s_empty[h], 128);
            mbar_init(&p_full[h], 128);
            mbar_init(&pv_done[h], 1);
            mbar_init(&bias_full[2 * h], 128);
            mbar_init(&bias_full[2 * h + 1], 128);
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int k_last[kStages], v_last[kStages];  // parity of the last phase loaded per stage, -1 if none
            for (int i = 0; i < kStages; ++i) k_last[i] = v_last[i] = -1;
            mbar_arrive_expect_tx(q_full, NQ * C::kQTile);
            for (int h = 0; h < NQ; ++h)
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(smem + C::kOffQ + h * C::kQTile + c * (kBM * 128), &tmap_q, q_full, c * 64,
                                head0 + h, m_tile * kBM, kEvictFirst);
            auto load = [&](int j, uint64_t* empty, uint64_t* full, int off, const CUtensorMap* map,
                            int* last) -> bool {
                const int st = j % kStages;
                const uint32_t ph = static_cast<uint32_t>(j / kStages) & 1;
                if (!mbar_wait(&empty[st], ph ^ 1, abort_flag, a.status, TG_STATUS_ATTENTION_TIMEOUT))
                    return false;
                uint8_t* dst = smem + off + st * C::kKVTile;
                mbar_arrive_expect_tx(&full[st], C::kKVTile);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(dst + c * (kBN * 128), map, &full[st], c * 64, kvh, j * kBN, kEvictLast);
                last[st] = static_cast<int>(ph);
                return true;
            };
            // K runs one tile ahead of V: S(j+1) needs only K(j+1); P(j) V(j) waits for softmax j anyway.
            bool ok = load(0, k_empty, k_full, C::kOffK, &tmap_k, k_last);
            for (int j = 0; j < n_kv && ok; ++j) {
                if (j + 1 < n_kv) ok = load(j + 1, k_empty, k_full, C::kOffK, &tmap_k, k_last);
                if (ok) ok = load(j, v_empty, v_full, C::kOffV, &tmap_v, v_last);
            }
            // Every issued copy must land before shared memory is released (matters on abort only).
            volatile int no_abort = 0;
            mbar_wait(q_full, 0, &no_abort, a.status, TG_STATUS_ATTENTION_TIMEOUT);
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
            bool ok = mbar_wait(q_full, 0, abort_flag, a.status, TG_STATUS_ATTENTION_TIMEOUT);
            auto wait_k = [&](int j) -> bool {
                return mbar_wait(&k_full[j % kStages], static_cast<uint32_t>(j / kStages) & 1, abort_flag,
                                 a.status, TG_STATUS_ATTENTION_TIMEOUT);
            };
            // Descriptors as 32-bit start/LBO words over one shared high word (SBO 1024,
            // 128-byte swizzle): every MMA below moves its operands by compile-time
            // offsets, so the issuing thread keeps ahead of the tensor pipe.
            const uint32_t dhi = sw128_desc_hi(1024);
            const uint32_t q_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffQ), 16);
            const uint32_t k_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffK), 16);
            const uint32_t v_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffV), kBN * 128);
            // S_h = Q_h K_j^T into head h's S columns, then signal softmax h
            auto issue_s = [&](int h, int j) {
                const uint32_t q_lo = q_lo0 + static_cast<uint32_t>(h * (C::kQTile >> 4));
                const uint32_t k_lo = k_lo0 + static_cast<uint32_t>((j % kStages) * (C::kKVTile >> 4));
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    // K step k: 64-column chunk k / 4, 32-byte column offset k % 4 inside the swizzle atom
                    const uint32_t qo = static_cast<uint32_t>(((k >> 2) * (kBM * 128) + (k & 3) * 32) >> 4);
                    const uint32_t ko = static_cast<uint32_t>(((k >> 2) * (kBN * 128) + (k & 3) * 32) >> 4);
                    mma_ss_lo(tmem + C::col_s(h), q_lo + qo, k_lo + ko, dhi, idesc_s, k > 0);
                }
                mma_commit(&s_full[h]);
            };
            if (ok) ok = wait_k(0);
            if (ok) {
                tc_fence_after();
                for (int h = 0; h < NQ; ++h) issue_s(h, 0);
                mma_commit(&k_empty[0]);
            }
            for (int j = 0; j < n_kv && ok; ++j) {
                const int st = j % kStages;
                // next S of each head as soon as its softmax has read the current one
                if (j + 1 < n_kv) {
                    if (!(ok = wait_k(j + 1))) break;
#pragma unroll
                    for (int h = 0; h < NQ && ok; ++h) {
                        if (!(ok = mbar_wait(&s_empty[h], static_cast<uint32_t>(j) & 1, abort_flag, a.status,
                                             TG_STATUS_ATTENTION_TIMEOUT)))
                            break;
                        tc_fence_after();
                        issue_s(h, j + 1);
                    }
                    if (!ok) break;
                    mma_commit(&k_empty[(j + 1) % kStages]);
                }
                // P_h(j) V_j for each head once its softmax has written P_h(j)
                if (!(ok = mbar_wait(&v_ready[st], static_cast<uint32_t>(j / kStages) & 1, abort_flag, a.status,
                                     TG_STATUS_ATTENTION_TIMEOUT)))
                    break;
                const uint32_t v_lo = v_lo0 + static_cast<uint32_t>(st * (C::kKVTile >> 4));
#pragma unroll
                for (int h = 0; h < NQ && ok; ++h) {
                    if (!(ok = mbar_wait(&p_full[h], static_cast<uint32_t>(j) & 1, abort_flag, a.status,
                                         TG_STATUS_ATTENTION_TIMEOUT)))
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < kBN / 16; ++k)  // 16 keys per step: 16 rows of 128 bytes in each chunk
                        mma_ts_lo(tmem + C::col_o(h), tmem + C::col_p(h) + static_cast<uint32_t>(k * 8),
                                  v_lo + static_cast<uint32_t>(k * (2048 >> 4)), dhi, idesc_o,
                                  (j > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&pv_done[h]);
                }
                if (!ok) break;
                mma_commit(&v_empty[st]);
            }
            if (!ok) {
                mma_commit(drain);
                volatile int no_abort = 0;
                mbar_wait(drain, 0, &no_abort, a.status, TG_STATUS_ATTENTION_TIMEOUT);
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ V tile -> fp16, in place
        const int t = threadIdx.x - 64;
        for (int j = 0; j < n_kv; ++j) {
            const int st = j % kStages;
            if (!mbar_wait(&v_full[st], static_cast<uint32_t>(j / kStages) & 1, abort_flag, a.status,
                           TG_STATUS_ATTENTION_TIMEOUT))
                break;
            uint4* vt = reinterpret_cast<uint4*>(smem + C::kOffV + st * C::kKVTile);
#pragma unroll 4
            for (int i = t; i < C::kKVTile / 16; i += 64) {
                uint4 x = vt[i];
                uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = f16x2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
                vt[i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            fence_proxy_async_smem();  // generic-proxy writes -> tensor-core (async proxy) reads
            mbar_arrive(&v_ready[st]);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue of head h
        const int h = (warp - 4) >> 2;
        const int q = warp & 3;
        const int row = q * 32 + lane;  // query row inside the tile == TMEM lane
        const int t = threadIdx.x - 128 - 128 * h;
        const int head = head0 + h;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + C::col_s(h);
        const uint32_t p_addr = tmem + lane_off + C::col_p(h);
        const uint32_t o_addr = tmem + lane_off + C::col_o(h);
        const float gain = a.gain ? a.gain[head] * kLog2e : 0.0f;
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
        float* bias_h = bias_s + h * 2 * kBN;
        float s_pref = (a.s_kept && t < kBN && t < a.K) ? a.s_kept[t] : 0.0f;
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int j = 0; j < n_kv && ok; ++j) {
            const int b = j & 1;
            // this tile's key bias g_h * s_c in log2 units (one key per thread), next tile's score prefetched
            if (t < kBN) bias_h[b * kBN + t] = gain * s_pref;
            mbar_arrive(&bias_full[2 * h + b]);
            {
                const int64_t cn = static_cast<int64_t>(j + 1) * kBN + t;
                s_pref = (a.s_kept && t < kBN && j + 1 < n_kv && cn < a.K) ? a.s_kept[cn] : 0.0f;
            }
            if (!(ok = warp_wait(&bias_full[2 * h + b], static_cast<uint32_t>(j >> 1) & 1, abort_flag, a.status)))
                break;
            if (!(ok = warp_wait(&s_full[h], static_cast<uint32_t>(j) & 1, abort_flag, a.status))) break;
            tc_fence_after();
            // the row's 64 S values, then hand the S columns back to the MMA warp
            float x[kBN];
            {
                uint32_t* xv = reinterpret_cast<uint32_t*>(x);
                tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(xv));
                tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(xv + 32));
                tmem_ld_wait();
            }
            tc_fence_before();
            mbar_arrive(&s_empty[h]);
            const float* bias = bias_h + b * kBN;
            // keys c with j * kBN + c > m_tile * kBM + row are in the future of this query row
            const int lim = m_tile * kBM + row - j * kBN;
            const bool diag = j >= first_diag;
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < kBN; c += 4) {
                const float4 bb = *reinterpret_cast<const float4*>(bias + c);
                float2 x0 = ffma2(make_float2(x[c], x[c + 1]), sc2, make_float2(bb.x, bb.y));
                float2 x1 = ffma2(make_float2(x[c + 2], x[c + 3]), sc2, make_float2(bb.z, bb.w));
                if (diag) {
                    if (c > lim) x0.x = -INFINITY;
                    if (c + 1 > lim) x0.y = -INFINITY;
                    if (c + 2 > lim) x1.x = -INFINITY;
                    if (c + 3 > lim) x1.y = -INFINITY;
                }
                x[c] = x0.x;
                x[c + 1] = x0.y;
                x[c + 2] = x1.x;
                x[c + 3] = x1.y;
                mx4[(c >> 2) & 3] = fmax3(mx4[(c >> 2) & 3], fmaxf(x0.x, x0.y), fmaxf(x1.x, x1.y));
            }
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            // lazy rescaling: keep the stale max unless this row's max grew by more than 2^8
            const bool need = mx > m_run + kRescaleThreshold;
            float alpha = 1.0f;
            if (need) {
                alpha = ex2(m_run - mx);  // 0 on the first tile (m_run = -inf)
                m_run = mx;
                l_run *= alpha;
            }
            // P_h(j-1) V_{j-1} must be complete before O is rescaled and P_h is overwritten
            if (j > 0) {
                if (!(ok = warp_wait(&pv_done[h], static_cast<uint32_t>(j - 1) & 1, abort_flag, a.status))) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, need)) {
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
            }
            // P = 2^(x - m) as fp16 into P_h
            const float2 neg_m = make_float2(-m_run, -m_run);
            float2 ls[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t p16[16];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float2 y0 = fadd2(make_float2(x[c0 + i], x[c0 + i + 1]), neg_m);
                    const float2 y1 = fadd2(make_float2(x[c0 + i + 2], x[c0 + i + 3]), neg_m);
                    const float2 p0 = make_float2(ex2(y0.x), ex2(y0.y));
                    const float2 p1 = make_float2(ex2(y1.x), ex2(y1.y));
                    ls[0] = fadd2(ls[0], p0);
                    ls[1] = fadd2(ls[1], p1);
                    p16[i / 2] = f16x2(p0.x, p0.y);
                    p16[i / 2 + 1] = f16x2(p1.x, p1.y);
                }
                tmem_st16(p_addr + (c0 >> 1), p16);
            }
            const float2 lsum = fadd2(ls[0], ls[1]);
            tmem_st_wait();
            l_run += lsum.x + lsum.y;
            tc_fence_before();
            mbar_arrive(&p_full[h]);
        }
        if (ok && warp_wait(&pv_done[h], static_cast<uint32_t>(n_kv - 1) & 1, abort_flag, a.status)) {
            // epilogue: normalise, store bf16 rows and the log-sum-exp
            tc_fence_after();
            const int64_t grow = static_cast<int64_t>(m_tile) * kBM + row;
            const float inv_l = 1.0f / l_run;
            __nv_bfloat16* orow = a.out + (grow * a.Hq + head) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(o_addr + c0, v);
                tmem_ld_wait();
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
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D, int NQ>
static tg_status launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, Args a,
                        cudaStream_t st) {
    using C = Cfg<D, NQ>;
    auto kern = gated_attention_kernel<D, NQ>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) != cudaSuccess)
        return TG_ERR_CUDA;
    a.pairs_per_group = (a.Hq / a.Hkv) / NQ;
    const int64_t grid = static_cast<int64_t>(a.num_q_tiles) * a.Hkv * a.pairs_per_group;
    if (grid > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    kern<<<static_cast<unsigned>(grid), C::kThreads, C::kSmem, st>>>(mq, mk, mv, a);
    return launch_status();
}

}  // namespace attn
}  // namespace tg

using namespace tg;

extern "C" tg_status tg_gated_attention(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                        const tg_bf16* v, int64_t ld_v, int64_t K, int32_t Hq, int32_t Hkv,
                                        int32_t d_h, const float* s_kept, const float* gain, float tau,
                                        tg_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    if (K < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || !std::isfinite(tau)) return TG_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return TG_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return TG_ERR_INVALID_ARG;
    if (K == 0) return TG_OK;
    if (K > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    if (!q || !k || !v || !out || !workspace || !aligned16(workspace)) return TG_ERR_INVALID_ARG;
    if (workspace_bytes < tg_workspace_bytes(TG_OP_ATTENTION, K, 0, 0)) return TG_ERR_INVALID_ARG;
    if (ld_q < static_cast<int64_t>(Hq) * d_h || ld_k < static_cast<int64_t>(Hkv) * d_h ||
        ld_v < static_cast<int64_t>(Hkv) * d_h || (ld_q % 8) || (ld_k % 8) || (ld_v % 8))
        return TG_ERR_INVALID_ARG;

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
        const uint64_t sv[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_v) * 2};
        if (!make_tmap_bf16(&mk, k, 3, dims, sk, kvbox) || !make_tmap_bf16(&mv, v, 3, dims, sv, kvbox))
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
    cudaStream_t st = as_stream(stream);
    const bool pairs = ((Hq / Hkv) % 2) == 0;
    if (d_h == 128) return pairs ? attn::launch<128, 2>(mq, mk, mv, a, st) : attn::launch<128, 1>(mq, mk, mv, a, st);
    return pairs ? attn::launch<64, 2>(mq, mk, mv, a, st) : attn::launch<64, 1>(mq, mk, mv, a, st);
}
