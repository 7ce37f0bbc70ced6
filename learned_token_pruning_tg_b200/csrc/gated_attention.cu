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
// Kernel (one CTA per (128-query tile, query head); heaviest tiles first):
//   warp 0     TMA: the Q tile once, then K and V tiles (128 keys) into a
//              2-stage ring (separate K and V barriers so S can start early)
//   warp 1     TMEM allocation and the single MMA-issuing thread:
//                S_j = Q K_j^T   (tcgen05 kind::f16, M=128, N=128, K=d_h)
//                O  += P_j V_j   (A = P_j read from TMEM, B = V_j MN-major)
//              S is double-buffered in TMEM so S_{j+1} overlaps softmax j
//   warps 4-7  softmax, one query row per thread: tcgen05.ld of the S row,
//              x = S * tau/sqrt(d_h) * log2(e) + g_h s_c log2(e) (bias added
//              in registers from a per-tile shared-memory vector), causal mask
//              on the diagonal tile only, online max with lazy rescaling (O is
//              rescaled only when a row max grows by more than 2^8), P = 2^(x-m)
//              written to TMEM as two bf16 halves P_hi + P_lo (P_lo = the
//              rounding residual), so the P V product (two MMAs per step) sees P
//              to ~16 significant bits: the output error no longer grows with
//              the magnitude of v; at the end O / l to bf16 and the log-sum-exp.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+d_h) P_hi, P_lo (64 each).
// Every wait is bounded (TG_STATUS_ATTENTION_TIMEOUT).
#include <cmath>

#include "tg_host.cuh"

namespace tg {
namespace attn {

constexpr int kBM = 128;       // query rows per tile
constexpr int kBN = 128;       // keys per tile
constexpr int kStages = 2;     // K/V ring depth
constexpr int kThreads = 256;  // 8 warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8

template <int D>
struct Cfg {
    static constexpr int kTile = kBM * D * 2;  // bytes of one 128 x D bf16 tile
    static constexpr int kChunks = D / 64;     // 64-column (128-byte) swizzle chunks per row
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTile;
    static constexpr int kOffV = kOffK + kStages * kTile;
    static constexpr int kOffBias = kOffV + kStages * kTile;  // float [2][128]
    static constexpr int kOffBar = kOffBias + 2 * kBN * 4;
    static constexpr int kNumBars = 1 + 4 * kStages + 2 * 3 + 2 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmem = kOffMisc + 16 + 1024;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColPhi = 256 + D, kColPlo = 256 + D + 64;
    static constexpr uint32_t kTmemCols = 512;
};

struct Args {
    int64_t K;
    int Hq, Hkv;
    int num_q_tiles;
    float scale_log2;  // tau / sqrt(d_h) * log2(e)
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

// Bounded wait whose result is the same on every lane of the warp, so that the
// warp-collective tcgen05.ld/st and shuffles that follow never see a partial warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          unsigned int* status) {
    const bool ok = mbar_wait(bar, parity, abort, status, TG_STATUS_ATTENTION_TIMEOUT);
    return __all_sync(0xffffffffu, ok);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
gated_attention_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const Args a) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* bias_s = reinterpret_cast<float*>(smem + C::kOffBias);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars;                     // TMA -> MMA
    uint64_t* k_full = bars + 1;                 // [kStages] TMA -> MMA
    uint64_t* k_empty = k_full + kStages;        // [kStages] MMA commit after S_j -> TMA
    uint64_t* v_full = k_empty + kStages;        // [kStages] TMA -> MMA
    uint64_t* v_empty = v_full + kStages;        // [kStages] MMA commit after P_j V_j -> TMA
    uint64_t* s_full = v_empty + kStages;        // [2] MMA commit -> softmax
    uint64_t* s_empty = s_full + 2;              // [2] 128 softmax threads -> MMA
    uint64_t* p_full = s_empty + 2;              // 128 softmax threads -> MMA (P_j written)
    uint64_t* pv_done = p_full + 1;              // MMA commit after P_j V_j (completion j)
    uint64_t* bias_full = pv_done + 1;           // [2] 128 softmax threads (key-bias vector written)
    uint64_t* drain = bias_full + 2;             // abort path
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // heaviest (last) query tiles first
    const int m_tile = a.num_q_tiles - 1 - static_cast<int>(blockIdx.x / a.Hq);
    const int h = static_cast<int>(blockIdx.x % a.Hq);
    const int kvh = h / (a.Hq / a.Hkv);
    const int n_kv = m_tile + 1;  // causal: kv tiles 0..m_tile, the last one on the diagonal

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 128);
            mbar_init(&bias_full[b], 128);
        }
        mbar_init(p_full, 128);
        mbar_init(pv_done, 1);
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
            mbar_arrive_expect_tx(q_full, C::kTile);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
                tma_load_3d(smem + C::kOffQ + c * (kBM * 128), &tmap_q, q_full, c * 64, h, m_tile * kBM,
                            kEvictFirst);
            auto load_k = [&](int j) -> bool {
                const int st = j % kStages;
                const uint32_t ph = static_cast<uint32_t>(j / kStages) & 1;
                if (!mbar_wait(&k_empty[st], ph ^ 1, abort_flag, a.status, TG_STATUS_ATTENTION_TIMEOUT))
                    return false;
                uint8_t* dst = smem + C::kOffK + st * C::kTile;
                mbar_arrive_expect_tx(&k_full[st], C::kTile);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(dst + c * (kBN * 128), &tmap_k, &k_full[st], c * 64, kvh, j * kBN, kEvictLast);
                k_last[st] = static_cast<int>(ph);
                return true;
            };
            auto load_v = [&](int j) -> bool {
                const int st = j % kStages;
                const uint32_t ph = static_cast<uint32_t>(j / kStages) & 1;
                if (!mbar_wait(&v_empty[st], ph ^ 1, abort_flag, a.status, TG_STATUS_ATTENTION_TIMEOUT))
                    return false;
                uint8_t* dst = smem + C::kOffV + st * C::kTile;
                mbar_arrive_expect_tx(&v_full[st], C::kTile);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(dst + c * (kBN * 128), &tmap_v, &v_full[st], c * 64, kvh, j * kBN, kEvictLast);
                v_last[st] = static_cast<int>(ph);
                return true;
            };
            // K runs one tile ahead of V: S_{j+1} only needs K_{j+1}, P_j V_j comes after softmax j.
            bool ok = load_k(0);
            for (int j = 0; j < n_kv && ok; ++j) {
                if (j + 1 < n_kv) ok = load_k(j + 1);
                if (ok) ok = load_v(j);
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
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBM, D, true);     // P V: B (= V) MN-major
            const uint32_t q_addr = smem_u32(smem + C::kOffQ);
            bool ok = mbar_wait(q_full, 0, abort_flag, a.status, TG_STATUS_ATTENTION_TIMEOUT);
            tc_fence_after();
            // S_j = Q K_j^T into S buffer j % 2; the K stage is released when these MMAs finish
            auto issue_s = [&](int j) -> bool {
                const int st = j % kStages;
                const uint32_t ph = static_cast<uint32_t>(j / kStages) & 1;
                const int b = j & 1;
                if (!mbar_wait(&k_full[st], ph, abort_flag, a.status, TG_STATUS_ATTENTION_TIMEOUT)) return false;
                if (!mbar_wait(&s_empty[b], (static_cast<uint32_t>(j >> 1) & 1) ^ 1, abort_flag, a.status,
                               TG_STATUS_ATTENTION_TIMEOUT))
                    return false;
                tc_fence_after();
                const uint32_t k_addr = smem_u32(smem + C::kOffK + st * C::kTile);
                const uint32_t d_tmem = tmem + (b ? C::kColS1 : C::kColS0);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = static_cast<uint32_t>((k >> 2) * (kBM * 128) + (k & 3) * 32);
                    mma_ss(d_tmem, smem_desc_sw128(q_addr + off, 16, 1024),
                           smem_desc_sw128(k_addr + off, 16, 1024), idesc_s, k > 0);
                }
                mma_commit(&s_full[b]);
                mma_commit(&k_empty[st]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 0; j < n_kv && ok; ++j) {
                if (j + 1 < n_kv && !(ok = issue_s(j + 1))) break;
                const int st = j % kStages;
                const uint32_t ph = static_cast<uint32_t>(j / kStages) & 1;
                const int b = j & 1;
                (void)b;
                if (!(ok = mbar_wait(p_full, static_cast<uint32_t>(j) & 1, abort_flag, a.status,
                                     TG_STATUS_ATTENTION_TIMEOUT)))
                    break;
                if (!(ok = mbar_wait(&v_full[st], ph, abort_flag, a.status, TG_STATUS_ATTENTION_TIMEOUT))) break;
                tc_fence_after();
                const uint32_t v_addr = smem_u32(smem + C::kOffV + st * C::kTile);
#pragma unroll
                for (int k = 0; k < kBN / 16; ++k) {  // 16 keys per step: 16 rows of 128 bytes in each chunk
                    const uint64_t vd =
                        smem_desc_sw128(v_addr + static_cast<uint32_t>(k * 2048), kBN * 128, 1024);
                    // P = P_hi + P_lo: two bf16 products keep P at ~16 significant bits
                    mma_ts(tmem + C::kColO, tmem + C::kColPhi + static_cast<uint32_t>(k * 8), vd, idesc_o,
                           (j > 0 || k > 0) ? 1u : 0u);
                    mma_ts(tmem + C::kColO, tmem + C::kColPlo + static_cast<uint32_t>(k * 8), vd, idesc_o, 1u);
                }
                mma_commit(&v_empty[st]);
                mma_commit(pv_done);
            }
            if (!ok) {
                mma_commit(drain);
                volatile int no_abort = 0;
                mbar_wait(drain, 0, &no_abort, a.status, TG_STATUS_ATTENTION_TIMEOUT);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax + epilogue
        const int q = warp & 3;
        const int row = q * 32 + lane;  // query row inside the tile == TMEM lane
        const int tid = threadIdx.x - 128;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const float gain = a.gain ? a.gain[h] * kLog2e : 0.0f;
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int j = 0; j < n_kv && ok; ++j) {
            const int b = j & 1;
            const uint32_t par = static_cast<uint32_t>(j >> 1) & 1;
            // this tile's key bias g_h * s_c, in log2 units (one key per thread)
            {
                const int64_t c = static_cast<int64_t>(j) * kBN + tid;
                bias_s[b * kBN + tid] = (a.s_kept && c < a.K) ? gain * a.s_kept[c] : 0.0f;
                mbar_arrive(&bias_full[b]);
            }
            if (!(ok = warp_wait(&bias_full[b], par, abort_flag, a.status))) break;
            if (!(ok = warp_wait(&s_full[b], par, abort_flag, a.status))) break;
            tc_fence_after();
            float x[kBN];
            {
                const uint32_t sa = tmem + lane_off + (b ? C::kColS1 : C::kColS0);
#pragma unroll
                for (int c0 = 0; c0 < kBN; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(sa + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[c0 + i] = __uint_as_float(v[i]);
                }
                tmem_ld_wait();
            }
            tc_fence_before();
            mbar_arrive(&s_empty[b]);

            const float* bias = bias_s + b * kBN;
            const bool diag = (j == n_kv - 1);
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kBN; ++c) {
                float v = fmaf(x[c], a.scale_log2, bias[c]);
                if (diag && c > row) v = -INFINITY;
                x[c] = v;
                mx = fmaxf(mx, v);
            }
            // lazy rescaling: keep the stale max unless this row's max grew by more than 2^8
            const bool need = mx > m_run + kRescaleThreshold;
            float alpha = 1.0f;
            if (need) {
                alpha = ex2(m_run - mx);  // 0 on the first tile (m_run = -inf)
                m_run = mx;
                l_run *= alpha;
            }
            // P_{j-1} V_{j-1} must be complete before O is rescaled and before P is overwritten
            if (j > 0) {
                if (!(ok = warp_wait(pv_done, static_cast<uint32_t>(j - 1) & 1, abort_flag, a.status))) break;
                tc_fence_after();
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                const uint32_t oa = tmem + lane_off + C::kColO;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(oa + c0, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                    tmem_st16(oa + c0, v);
                }
            }
            float lsum = 0.0f;
            const uint32_t pa_hi = tmem + lane_off + C::kColPhi;
            const uint32_t pa_lo = tmem + lane_off + C::kColPlo;
#pragma unroll
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float p0 = ex2(x[c0 + 2 * i] - m_run);
                    const float p1 = ex2(x[c0 + 2 * i + 1] - m_run);
                    lsum += p0 + p1;
                    hi[i] = pack_bf16x2(p0, p1);
                    lo[i] = pack_bf16x2(p0 - __uint_as_float(hi[i] << 16), p1 - __uint_as_float(hi[i] & 0xffff0000u));
                }
                tmem_st16(pa_hi + (c0 >> 1), hi);
                tmem_st16(pa_lo + (c0 >> 1), lo);
            }
            tmem_st_wait();
            l_run += lsum;
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok) {
            // epilogue: wait for the last P V, normalise, store bf16 rows and the log-sum-exp
            const int jl = n_kv - 1;
            if (warp_wait(pv_done, static_cast<uint32_t>(jl) & 1, abort_flag, a.status)) {
                tc_fence_after();
                const int64_t grow = static_cast<int64_t>(m_tile) * kBM + row;
                const float inv_l = 1.0f / l_run;
                __nv_bfloat16* orow = a.out + (grow * a.Hq + h) * D;
                const uint32_t oa = tmem + lane_off + C::kColO;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(oa + c0, v);
                    tmem_ld_wait();
                    if (grow < a.K) {
                        uint32_t o[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            o[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l,
                                               __uint_as_float(v[2 * i + 1]) * inv_l);
                        uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                    }
                }
                if (a.lse && grow < a.K)
                    a.lse[static_cast<int64_t>(h) * a.K + grow] = (m_run + log2f(l_run)) / kLog2e;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D>
static tg_status launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const Args& a,
                        cudaStream_t st) {
    using C = Cfg<D>;
    auto kern = gated_attention_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) != cudaSuccess)
        return TG_ERR_CUDA;
    const int64_t grid = static_cast<int64_t>(a.num_q_tiles) * a.Hq;
    if (grid > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    kern<<<static_cast<unsigned>(grid), kThreads, C::kSmem, st>>>(mq, mk, mv, a);
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
    const uint32_t box[3] = {64, 1, 128};
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(d_h), static_cast<uint64_t>(Hq), static_cast<uint64_t>(K)};
        const uint64_t str[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_q) * 2};
        if (!make_tmap_bf16(&mq, q, 3, dims, str, box)) return TG_ERR_CUDA;
    }
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(d_h), static_cast<uint64_t>(Hkv), static_cast<uint64_t>(K)};
        const uint64_t sk[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_k) * 2};
        const uint64_t sv[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_v) * 2};
        if (!make_tmap_bf16(&mk, k, 3, dims, sk, box) || !make_tmap_bf16(&mv, v, 3, dims, sv, box))
            return TG_ERR_CUDA;
    }
    attn::Args a;
    a.K = K;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.num_q_tiles = static_cast<int>((K + attn::kBM - 1) / attn::kBM);
    a.scale_log2 = tau / std::sqrt(static_cast<float>(d_h)) * attn::kLog2e;
    a.s_kept = s_kept;
    a.gain = gain;
    a.out = reinterpret_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.status = status_word(workspace);
    cudaStream_t st = as_stream(stream);
    return d_h == 128 ? attn::launch<128>(mq, mk, mv, a, st) : attn::launch<64>(mq, mk, mv, a, st);
}
