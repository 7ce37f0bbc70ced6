// gated_attention_bwd.cu -- gradients of token-gated causal GQA attention.
//
// TokenGate (aiproducthub.cn article, paragraph 事件详情; aisight.pl article,
// section Jak to działa; chathome.org article, section トークンゲート付き
// アテンションとは): the kept tokens' scores enter the attention logits above
// the gate as a bias precisely so that the loss has a gradient path back to the
// scorer, and the per-head gain and the temperature are learned with it.  For
//   l_{r,c} = tau (q_r . k_c) / sqrt(d_h) + g_h s_c,  c <= r,
//   P = softmax_c(l),  O_r = sum_c P_{r,c} v_c,
// and an upstream gradient dO, the chain rule gives (D_r = dO_r . O_r)
//   dP_{r,c} = dO_r . v_c,            dl_{r,c} = P_{r,c} (dP_{r,c} - D_r)
//   dq_r = tau / sqrt(d_h) sum_c dl_{r,c} k_c,   dk_c = tau / sqrt(d_h) sum_r dl_{r,c} q_r
//   dv_c = sum_r P_{r,c} dO_r,        ds_c = sum_h g_h sum_r dl_{h,r,c}
//   dg_h = sum_{r,c} dl_{h,r,c} s_c,  dtau = 1 / sqrt(d_h) sum_{h,r} q_{h,r} . (sum_c dl_{h,r,c} k_c)
// (the last because tau enters only through q . k).
//
// Four launches, all on the caller's stream:
//   bwd_prep_kernel   D_r = dO_r . O_r and lse in log2 units, per (head, row), into
//                     the workspace, rows padded to a multiple of 128 (padding rows
//                     get lse = +inf, so every weight they produce is 0)
//   bwd_dq_kernel     one CTA per (128-row query tile, query head), heaviest first;
//                     per 128-key tile j (tcgen05, accumulators in TMEM):
//                       S  = Q K_j^T (+ the key bias as one extra K = 16 step, the
//                            same three-part split as the forward), dP = dO V_j^T,
//                       dS = P (dP - D) in bf16 over S's own columns,
//                       dQ += dS K_j   (dS read from TMEM, K_j MN-major in smem)
//                     epilogue: dq in bf16, and q . (sum_c dS k_c) per CTA for dtau
//   bwd_dkdv_kernel   one CTA per (128-key tile, KV head), heaviest first; per
//                     (query head of the group, query tile i) the transposed products
//                       S^T = K Q_i^T (+ bias), dP^T = V dO_i^T, P^T and dS^T in bf16,
//                       dV += P^T dO_i,  dK += dS^T Q_i
//                     with the keys in the TMEM lanes, so the column sums of dS that
//                     ds and dg need are per-thread register sums
//   bwd_finish_kernel ds over the KV heads, dg over the key tiles, dtau over the
//                     dq CTAs, in a fixed order (deterministic)
// Warps of both big kernels: 0 TMA, 1 TMEM allocation and the single MMA-issuing
// thread, 2 the bias operands, 3-10 two softmax warpgroups (one row per thread).
// The dq kernel's warpgroups split each tile's 128 keys (64 each); the dk/dv kernel
// takes each step's 128 queries in two 64-query halves with their own S^T / dP^T
// columns, so one half's products overlap the other half's softmax (32 queries of
// a half per warpgroup).  P and dS are bf16 because dO,
// Q and K are (kind::f16 multiplies operands of one type).  Every wait is bounded
// (TG_STATUS_BACKWARD_TIMEOUT).
#include <algorithm>
#include <cmath>

#include "tg_host.cuh"

namespace tg {
namespace bwd {

constexpr int kB = 128;  // rows of every tile (queries or keys)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kAugTile = 4096;   // 128 rows x 16 bf16, no-swizzle K-major
constexpr int kMaxGroup = 8;     // query heads per KV head
constexpr int kHalf = 64;        // the dk/dv kernel takes each step's 128 query columns in two halves
constexpr int kWG = 2;           // softmax warpgroups; each takes kWGCols of a half's 64 columns
constexpr int kWGCols = kHalf / kWG;
constexpr int kSoftWarps = 4 * kWG;
constexpr int kThreads = 32 * (3 + kSoftWarps);

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void split3_bf16(float x, __nv_bfloat16 (&p)[3]) {
    p[0] = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(p[0]);
    p[1] = __float2bfloat16_rn(r1);
    p[2] = __float2bfloat16_rn(r1 - __bfloat162float(p[1]));
}
__device__ __forceinline__ uint32_t bf2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}
// Row r's two 16-byte core-matrix rows of a 128 x 16 no-swizzle K-major tile (LBO 128, SBO 256), in uint4 units.
__device__ __forceinline__ int aug_slot(int r, int chunk) { return (r >> 3) * 16 + chunk * 8 + (r & 7); }
// The two products of the bias step: one operand's rows hold a per-row value x split in three parts
// as {x0 x1 x2 x0 x1 x2 x0 x1 x2}, the other's rows a per-head value y as {y0 y0 y0 y1 y1 y1 y2 y2 y2};
// the nine products add up to x y.
__device__ __forceinline__ void aug_row_cycled(uint4* tile, int r, float x) {
    __nv_bfloat16 p[3];
    split3_bf16(x, p);
    const __nv_bfloat16 z = __float2bfloat16_rn(0.0f);
    tile[aug_slot(r, 0)] = make_uint4(bf2(p[0], p[1]), bf2(p[2], p[0]), bf2(p[1], p[2]), bf2(p[0], p[1]));
    tile[aug_slot(r, 1)] = make_uint4(bf2(p[2], z), 0u, 0u, 0u);
}
__device__ __forceinline__ void aug_row_repeated(uint4* tile, int r, const __nv_bfloat16 (&g)[3]) {
    const __nv_bfloat16 z = __float2bfloat16_rn(0.0f);
    tile[aug_slot(r, 0)] = make_uint4(bf2(g[0], g[0]), bf2(g[0], g[1]), bf2(g[1], g[1]), bf2(g[2], g[2]));
    tile[aug_slot(r, 1)] = make_uint4(bf2(g[2], z), 0u, 0u, 0u);
}

// Plain (untiled) bulk copy global -> shared, completing on an mbarrier; both
// addresses 16-byte aligned and the size a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned int* status) {
    const bool ok = mbar_wait(bar, parity, abort, status, TG_STATUS_BACKWARD_TIMEOUT);
    return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ bool wait1(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned int* status) {
    return mbar_wait(bar, parity, abort, status, TG_STATUS_BACKWARD_TIMEOUT);
}

// K-step k (16 elements of a 128-byte-swizzled K-major tile of 128 rows): chunk k / 4, 32-byte column k % 4.
__device__ __forceinline__ uint32_t kstep_off(int k) {
    return static_cast<uint32_t>(((k >> 2) * (kB * 128) + (k & 3) * 32) >> 4);
}
// TMEM column of the A operand for K-step k (16 elements) of a bf16 P / dS tile that each softmax
// warpgroup wrote, packed two to a column, at the start of its own kWGCols-column range.
// The dq kernel's whole-tile variant: two warpgroups of 64 keys, keys 0-63 at columns 0-31, 64-127 at 64-95.
__device__ __forceinline__ uint32_t a_col_full(int k) { return static_cast<uint32_t>(k < 4 ? 8 * k : 64 + 8 * (k - 4)); }
__device__ __forceinline__ uint32_t a_col(int k) {
    constexpr int steps = kWGCols / 16;  // K-steps per warpgroup
    return static_cast<uint32_t>((k / steps) * kWGCols + (k % steps) * 8);
}

// ============================================================== prep: D and lse in log2 units
// One thread per (row, head), rows padded to Kp: D = dO . O from 16-byte loads of both rows.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ out,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse, int64_t K, int64_t Kp, int Hq,
                                                       float* __restrict__ lse2, float* __restrict__ dvec) {
    const int64_t total = Kp * Hq;
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < total;
         w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = w / Hq;
        const int h = static_cast<int>(w - r * Hq);
        float acc = 0.0f;
        if (r < K) {
            const uint4* o = reinterpret_cast<const uint4*>(out + w * D);   // row r, head h: w = r Hq + h
            const uint4* g = reinterpret_cast<const uint4*>(dout + w * D);
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                const uint4 a = o[i], b = g[i];
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(bw[e] << 16), acc);
                    acc = fmaf(__uint_as_float(aw[e] & 0xffff0000u), __uint_as_float(bw[e] & 0xffff0000u), acc);
                }
            }
        }
        lse2[h * Kp + r] = r < K ? lse[h * K + r] * kLog2e : INFINITY;
        dvec[h * Kp + r] = acc;
    }
}

// ============================================================== dQ
// Whole 128-key tiles: S and dP of one tile, then dQ += dS K_j.  (Taking the tile in 64-key halves
// to overlap the softmax with the products made S and dP N = 64 MMAs, which read the full Q / dO
// tile from shared memory for half the work each, and measured slower.)
template <int D>
struct CfgQ {
    static constexpr int kStages = (D == 64) ? 4 : 2;
    static constexpr int kTile = kB * D * 2;
    static constexpr int kChunks = D / 64;
    static constexpr int kOffQ = 0;
    static constexpr int kOffDO = kTile;
    static constexpr int kOffK = 2 * kTile;
    static constexpr int kOffV = kOffK + kStages * kTile;
    static constexpr int kOffAugA = kOffV + kStages * kTile;
    static constexpr int kOffAugB = kOffAugA + kAugTile;
    static constexpr int kOffBar = kOffAugB + kStages * kAugTile;
    static constexpr int kNumBars = 1 + 3 * kStages + 4;
    static constexpr int kOffRed = kOffBar + kNumBars * 8;
    static constexpr int kOffMisc = kOffRed + kSoftWarps * 4;
    static constexpr int kSmem = kOffMisc + 16 + 1024;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;
};

// 128-byte-swizzled TMA destinations start on 1024-byte boundaries; everything fits in 227 KB.
template <int D>
constexpr bool layout_ok_q() {
    using C = CfgQ<D>;
    return C::kOffDO % 1024 == 0 && C::kOffK % 1024 == 0 && C::kOffV % 1024 == 0 && C::kTile % 1024 == 0 &&
           C::kOffAugA % 16 == 0 && C::kOffAugB % 16 == 0 && C::kOffBar % 8 == 0 && C::kSmem <= 232448;
}
static_assert(layout_ok_q<64>() && layout_ok_q<128>(), "dq kernel shared-memory layout");

struct ArgsQ {
    int64_t K, Kp;
    int Hq, G, num_q_tiles;
    float scale_log2;  // tau / sqrt(d_h) * log2(e)
    float scale;       // tau / sqrt(d_h)
    const float* s_kept;
    const float* gain;
    const float* lse2;
    const float* dvec;
    const __nv_bfloat16* q;
    int64_t ld_q;
    __nv_bfloat16* dq;
    float* dtau_part;
    unsigned int* status;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_do,
              const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v, const ArgsQ a) {
    using C = CfgQ<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars;              // Q and dO tiles landed
    uint64_t* kv_full = bars + 1;         // [S] K_j and V_j landed
    uint64_t* kv_empty = kv_full + S;     // [S] commit after dQ += dS K_j
    uint64_t* aug_full = kv_empty + S;    // [S] bias operand of K_j written (32 lanes)
    uint64_t* s_full = aug_full + S;      // commit after S and dP of a tile
    uint64_t* ds_full = s_full + 1;       // 256 softmax threads wrote dS
    uint64_t* o_full = ds_full + 1;       // commit after the last dQ MMA
    uint64_t* drain = o_full + 1;
    float* red = reinterpret_cast<float*>(smem + C::kOffRed);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tile = a.num_q_tiles - 1 - static_cast<int>(blockIdx.x / a.Hq);  // heaviest first
    const int head = static_cast<int>(blockIdx.x % a.Hq);
    const int kvh = head / a.G;
    const int n_kv = m_tile + 1;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&aug_full[s], 32);
        }
        mbar_init(s_full, 1);
        mbar_init(ds_full, 32 * kSoftWarps);
        mbar_init(o_full, 1);
        mbar_init(drain, 1);
        for (int w = 0; w < kSoftWarps; ++w) red[w] = 0.0f;
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_do);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == 2) {
        // A of the bias step: every row holds gamma_h = g_h sqrt(d_h) / tau in three parts
        __nv_bfloat16 g[3];
        split3_bf16(a.gain ? a.gain[head] * kLog2e / a.scale_log2 : 0.0f, g);
        uint4* aug_a = reinterpret_cast<uint4*>(smem + C::kOffAugA);
        for (int r = lane; r < kB; r += 32) aug_row_repeated(aug_a, r, g);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int last[S];
            for (int i = 0; i < S; ++i) last[i] = -1;
            mbar_arrive_expect_tx(q_full, 2 * C::kTile);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) {
                tma_load_3d(smem + C::kOffQ + c * (kB * 128), &tmap_q, q_full, c * 64, head, m_tile * kB, kEvictFirst);
                tma_load_3d(smem + C::kOffDO + c * (kB * 128), &tmap_do, q_full, c * 64, head, m_tile * kB,
                            kEvictFirst);
            }
            for (int j = 0; j < n_kv; ++j) {
                const int st = j % S;
                const uint32_t ph = static_cast<uint32_t>(j / S) & 1;
                if (!wait1(&kv_empty[st], ph ^ 1, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(&kv_full[st], 2 * C::kTile);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) {
                    tma_load_3d(smem + C::kOffK + st * C::kTile + c * (kB * 128), &tmap_k, &kv_full[st], c * 64, kvh,
                                j * kB, kEvictLast);
                    tma_load_3d(smem + C::kOffV + st * C::kTile + c * (kB * 128), &tmap_v, &kv_full[st], c * 64, kvh,
                                j * kB, kEvictLast);
                }
                last[st] = static_cast<int>(ph);
            }
            // every issued copy lands before shared memory is released (matters on abort only)
            volatile int no_abort = 0;
            wait1(q_full, 0, &no_abort, a.status);
            for (int i = 0; i < S; ++i)
                if (last[i] >= 0) wait1(&kv_full[i], static_cast<uint32_t>(last[i]), &no_abort, a.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kB, kB, false);  // both operands K-major
            constexpr uint32_t idesc_q = idesc_bf16_f32(kB, D, true);    // dS (TMEM) x K_j MN-major
            const uint32_t dhi = sw128_desc_hi(1024);
            const uint32_t q_lo = sw128_desc_lo(smem_u32(smem + C::kOffQ), 16);
            const uint32_t do_lo = sw128_desc_lo(smem_u32(smem + C::kOffDO), 16);
            const uint32_t k_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffK), 16);
            const uint32_t kmn_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffK), kB * 128);
            const uint32_t v_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffV), 16);
            const uint32_t ahi = noswz_desc_hi(256);
            const uint32_t aa_lo = sw128_desc_lo(smem_u32(smem + C::kOffAugA), 128);
            const uint32_t ab_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffAugB), 128);
            const bool bias = a.gain != nullptr && a.s_kept != nullptr;
            auto ready = [&](int j) -> bool {
                const uint32_t ph = static_cast<uint32_t>(j / S) & 1;
                return wait1(&kv_full[j % S], ph, abort_flag, a.status) &&
                       wait1(&aug_full[j % S], ph, abort_flag, a.status);
            };
            // S = Q K_j^T (+ bias) and dP = dO V_j^T, then signal the softmax warps
            auto issue_sdp = [&](int j) {
                const uint32_t so = static_cast<uint32_t>((j % S) * (C::kTile >> 4));
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_ss_lo(tmem + C::kColS, q_lo + kstep_off(k), k_lo0 + so + kstep_off(k), dhi, idesc_s, k > 0);
                if (bias)
                    mma_ss_lo(tmem + C::kColS, aa_lo, ab_lo0 + static_cast<uint32_t>((j % S) * (kAugTile >> 4)), ahi,
                              idesc_s, 1u);
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_ss_lo(tmem + C::kColDP, do_lo + kstep_off(k), v_lo0 + so + kstep_off(k), dhi, idesc_s, k > 0);
                mma_commit(s_full);
            };
            bool ok = wait1(q_full, 0, abort_flag, a.status) && ready(0);
            if (ok) {
                tc_fence_after();
                issue_sdp(0);
            }
            for (int j = 0; j < n_kv && ok; ++j) {
                const int st = j % S;
                if (!(ok = wait1(ds_full, static_cast<uint32_t>(j) & 1, abort_flag, a.status))) break;
                tc_fence_after();
                // dQ += dS K_j: 16 keys per step (16 rows of the MN-major K tile)
                const uint32_t ko = kmn_lo0 + static_cast<uint32_t>(st * (C::kTile >> 4));
#pragma unroll
                for (int k = 0; k < kB / 16; ++k)
                    mma_ts_lo(tmem + C::kColDQ, tmem + C::kColS + a_col_full(k), ko + static_cast<uint32_t>(k * (2048 >> 4)),
                              dhi, idesc_q, (j > 0 || k > 0) ? 1u : 0u);
                mma_commit(&kv_empty[st]);
                if (j + 1 < n_kv) {
                    // behind dQ in the same in-order pipe: the next S and dP over the same columns
                    if (!(ok = ready(j + 1))) break;
                    issue_sdp(j + 1);
                } else {
                    mma_commit(o_full);
                }
            }
            if (!ok) {
                mma_commit(drain);
                volatile int no_abort = 0;
                wait1(drain, 0, &no_abort, a.status);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ bias operand B: s_c of K_j's keys
        uint4* aug_b = reinterpret_cast<uint4*>(smem + C::kOffAugB);
        for (int j = 0; j < n_kv; ++j) {
            const int st = j % S;
            if (!wait1(&kv_empty[st], (static_cast<uint32_t>(j / S) & 1) ^ 1, abort_flag, a.status)) break;
            uint4* dst = aug_b + st * (kAugTile / 16);
#pragma unroll
            for (int i = 0; i < kB / 32; ++i) {
                const int c = i * 32 + lane;
                const int64_t key = static_cast<int64_t>(j) * kB + c;
                aug_row_cycled(dst, c, (a.s_kept && key < a.K) ? a.s_kept[key] : 0.0f);
            }
            fence_proxy_async_smem();
            mbar_arrive(&aug_full[st]);
        }
    } else {
        // ------------------------------------------------------------ dS = P (dP - D), then the dq epilogue
        const int wg = (warp - 3) >> 2;      // which 64 keys of the tile
        const int qd = warp & 3;             // TMEM lane quarter
        const int row = qd * 32 + lane;      // query row in the tile == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
        const int64_t grow = static_cast<int64_t>(m_tile) * kB + row;
        const float lse2_r = a.lse2[head * a.Kp + grow];
        const float d_r = a.dvec[head * a.Kp + grow];
        bool ok = true;
        for (int j = 0; j < n_kv && ok; ++j) {
            if (!(ok = warp_wait(s_full, static_cast<uint32_t>(j) & 1, abort_flag, a.status))) break;
            tc_fence_after();
            const bool diag = j == n_kv - 1;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                const int c0 = 64 * wg + 32 * ch;
                uint32_t sv[32], pv[32];
                tmem_ld32(tmem + lane_off + C::kColS + c0, sv);
                tmem_ld32(tmem + lane_off + C::kColDP + c0, pv);
                tmem_ld_wait();
                uint32_t d16[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float p0 = ex2(fmaf(__uint_as_float(sv[e]), a.scale_log2, -lse2_r));
                    float p1 = ex2(fmaf(__uint_as_float(sv[e + 1]), a.scale_log2, -lse2_r));
                    if (diag) {  // key c of the diagonal tile is in the future of row r when c > r
                        if (c0 + e > row) p0 = 0.0f;
                        if (c0 + e + 1 > row) p1 = 0.0f;
                    }
                    d16[e >> 1] = pack_bf16x2(p0 * (__uint_as_float(pv[e]) - d_r), p1 * (__uint_as_float(pv[e + 1]) - d_r));
                }
                // into this warpgroup's own S columns, already read
                tmem_st16(tmem + lane_off + C::kColS + 64 * wg + 16 * ch, d16);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(ds_full);
        }
        if (ok && warp_wait(o_full, 0, abort_flag, a.status)) {
            tc_fence_after();
            float qdot = 0.0f;
            const __nv_bfloat16* qrow = a.q + grow * a.ld_q + static_cast<int64_t>(head) * D;
            __nv_bfloat16* drow = a.dq + (grow * a.Hq + head) * D;
#pragma unroll
            for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + C::kColDQ + c0, v);
                tmem_ld_wait();
                if (grow < a.K) {
                    uint32_t o[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 qq = *reinterpret_cast<const uint4*>(qrow + c0 + 8 * i);
                        const uint32_t qw[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float a0 = __uint_as_float(v[8 * i + 2 * e]), a1 = __uint_as_float(v[8 * i + 2 * e + 1]);
                            qdot = fmaf(__uint_as_float(qw[e] << 16), a0, qdot);
                            qdot = fmaf(__uint_as_float(qw[e] & 0xffff0000u), a1, qdot);
                            o[4 * i + e] = pack_bf16x2(a0 * a.scale, a1 * a.scale);
                        }
                    }
                    uint4* dst = reinterpret_cast<uint4*>(drow + c0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) qdot += __shfl_xor_sync(0xffffffffu, qdot, o);
            if (lane == 0) red[warp - 3] = qdot;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0) {
        float t = 0.0f;
        for (int w = 0; w < kSoftWarps; ++w) t += red[w];
        a.dtau_part[blockIdx.x] = t;
    }
}

__device__ __forceinline__ uint32_t col_s(int x) { return static_cast<uint32_t>(128 * x); }
__device__ __forceinline__ uint32_t col_dp(int x) { return static_cast<uint32_t>(128 * x + kHalf); }

// ============================================================== dK, dV, column sums
// Each step's 128 query columns are taken in two 64-query halves with their own S^T / dP^T
// columns, so one half's products overlap the other half's softmax.
template <int D>
struct CfgKV {
    static constexpr int kStages = (D == 64) ? 3 : 2;
    static constexpr int kTile = kB * D * 2;
    static constexpr int kChunks = D / 64;
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kTile;
    static constexpr int kOffQ = 2 * kTile;                      // [S]
    static constexpr int kOffDO = kOffQ + kStages * kTile;       // [S]
    static constexpr int kOffVec = kOffDO + kStages * kTile;     // [S] lse2[128], then D[128]
    static constexpr int kOffAugA = kOffVec + kStages * 1024;    // s_c of the CTA's keys
    static constexpr int kOffAugB = kOffAugA + kAugTile;         // [S] gamma_h of the step's head
    static constexpr int kOffBar = kOffAugB + kStages * kAugTile;
    static constexpr int kNumBars = 1 + 3 * kStages + 6;
    static constexpr int kOffDs = kOffBar + kNumBars * 8;        // [kWG][128] per-warpgroup ds
    static constexpr int kOffDg = kOffDs + kWG * kB * 4;         // [kSoftWarps][kMaxGroup]
    static constexpr int kOffMisc = kOffDg + kSoftWarps * kMaxGroup * 4;
    static constexpr int kSmem = kOffMisc + 16 + 1024;
    static constexpr uint32_t kColDV = 256, kColDK = 256 + D;
};

template <int D>
constexpr bool layout_ok_kv() {
    using C = CfgKV<D>;
    return C::kOffV % 1024 == 0 && C::kOffQ % 1024 == 0 && C::kOffDO % 1024 == 0 && C::kTile % 1024 == 0 &&
           C::kOffVec % 16 == 0 && C::kOffAugA % 16 == 0 && C::kOffAugB % 16 == 0 && C::kOffBar % 8 == 0 &&
           C::kSmem <= 232448;
}
static_assert(layout_ok_kv<64>() && layout_ok_kv<128>(), "dk/dv kernel shared-memory layout");

struct ArgsKV {
    int64_t K, Kp;
    int Hq, Hkv, G, num_q_tiles, num_k_tiles;
    float scale_log2, scale;
    const float* s_kept;
    const float* gain;
    const float* lse2;
    const float* dvec;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    float* ds_part;   // [Hkv, Kp]
    float* dg_part;   // [Hq, num_k_tiles]
    unsigned int* status;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_do,
                const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                const ArgsKV a) {
    using C = CfgKV<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* kv_full = bars;             // K and V tiles of the CTA landed
    uint64_t* st_full = bars + 1;         // [S] Q_i, dO_i, lse2 and D slices landed
    uint64_t* st_empty = st_full + S;     // [S] commit after the second half's dV and dK
    uint64_t* aug_full = st_empty + S;    // [S] gamma operand of the step written (32 lanes)
    uint64_t* s_full = aug_full + S;      // [2] commit after a half's S^T and dP^T
    uint64_t* p_full = s_full + 2;        // [2] the softmax threads wrote that half's P^T and dS^T
    uint64_t* o_full = p_full + 2;        // commit after the last dV / dK MMA
    uint64_t* drain = o_full + 1;
    float* dsw = reinterpret_cast<float*>(smem + C::kOffDs);
    float* dgw = reinterpret_cast<float*>(smem + C::kOffDg);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tile = static_cast<int>(blockIdx.x / a.Hkv);  // key tile; tile 0 has the most queries
    const int kvh = static_cast<int>(blockIdx.x % a.Hkv);
    const int nq = a.num_q_tiles - n_tile;                    // query tiles n_tile .. last
    const int T = nq * a.G;                                   // steps: (head of the group, query tile)
    const int U = 2 * T;                                      // halves: u = 2 t + (0 | 1)

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(&st_full[s], 1);
            mbar_init(&st_empty[s], 1);
            mbar_init(&aug_full[s], 32);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s_full[x], 1);
            mbar_init(&p_full[x], 32 * kSoftWarps);
        }
        mbar_init(o_full, 1);
        mbar_init(drain, 1);
        for (int i = 0; i < kSoftWarps * kMaxGroup; ++i) dgw[i] = 0.0f;
        for (int i = 0; i < kWG * kB; ++i) dsw[i] = 0.0f;
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_do);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == 2) {
        // A of the bias step: row c holds s_c of this CTA's key c in three parts
        uint4* aug_a = reinterpret_cast<uint4*>(smem + C::kOffAugA);
        for (int c = lane; c < kB; c += 32) {
            const int64_t key = static_cast<int64_t>(n_tile) * kB + c;
            aug_row_cycled(aug_a, c, (a.s_kept && key < a.K) ? a.s_kept[key] : 0.0f);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int last[S];
            for (int i = 0; i < S; ++i) last[i] = -1;
            mbar_arrive_expect_tx(kv_full, 2 * C::kTile);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) {
                tma_load_3d(smem + C::kOffK + c * (kB * 128), &tmap_k, kv_full, c * 64, kvh, n_tile * kB, kEvictFirst);
                tma_load_3d(smem + C::kOffV + c * (kB * 128), &tmap_v, kv_full, c * 64, kvh, n_tile * kB, kEvictFirst);
            }
            for (int t = 0; t < T; ++t) {
                const int st = t % S;
                const uint32_t ph = static_cast<uint32_t>(t / S) & 1;
                const int head = kvh * a.G + t / nq;
                const int i = n_tile + t % nq;
                if (!wait1(&st_empty[st], ph ^ 1, abort_flag, a.status)) break;
                mbar_arrive_expect_tx(&st_full[st], 2 * C::kTile + 1024);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) {
                    tma_load_3d(smem + C::kOffQ + st * C::kTile + c * (kB * 128), &tmap_q, &st_full[st], c * 64, head,
                                i * kB, kEvictLast);
                    tma_load_3d(smem + C::kOffDO + st * C::kTile + c * (kB * 128), &tmap_do, &st_full[st], c * 64,
                                head, i * kB, kEvictLast);
                }
                const int64_t vo = static_cast<int64_t>(head) * a.Kp + static_cast<int64_t>(i) * kB;
                bulk_load(smem + C::kOffVec + st * 1024, a.lse2 + vo, 512, &st_full[st]);
                bulk_load(smem + C::kOffVec + st * 1024 + 512, a.dvec + vo, 512, &st_full[st]);
                last[st] = static_cast<int>(ph);
            }
            volatile int no_abort = 0;
            wait1(kv_full, 0, &no_abort, a.status);
            for (int i = 0; i < S; ++i)
                if (last[i] >= 0) wait1(&st_full[i], static_cast<uint32_t>(last[i]), &no_abort, a.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kB, kHalf, false);  // 128 keys x 64 queries
            constexpr uint32_t idesc_o = idesc_bf16_f32(kB, D, true);
            const uint32_t dhi = sw128_desc_hi(1024);
            const uint32_t k_lo = sw128_desc_lo(smem_u32(smem + C::kOffK), 16);
            const uint32_t v_lo = sw128_desc_lo(smem_u32(smem + C::kOffV), 16);
            const uint32_t q_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffQ), 16);
            const uint32_t do_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffDO), 16);
            const uint32_t qmn_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffQ), kB * 128);
            const uint32_t domn_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffDO), kB * 128);
            const uint32_t ahi = noswz_desc_hi(256);
            const uint32_t aa_lo = sw128_desc_lo(smem_u32(smem + C::kOffAugA), 128);
            const uint32_t ab_lo0 = sw128_desc_lo(smem_u32(smem + C::kOffAugB), 128);
            const bool bias = a.gain != nullptr && a.s_kept != nullptr;
            auto ready = [&](int t) -> bool {
                const uint32_t ph = static_cast<uint32_t>(t / S) & 1;
                return wait1(&st_full[t % S], ph, abort_flag, a.status) &&
                       wait1(&aug_full[t % S], ph, abort_flag, a.status);
            };
            // half u (queries 64 (u & 1) .. of step u / 2): S^T = K Q^T (+ bias), dP^T = V dO^T
            auto issue_sdp = [&](int u) {
                const int t = u >> 1, hf = u & 1;
                const uint32_t so = static_cast<uint32_t>((t % S) * (C::kTile >> 4) + ((hf * kHalf * 128) >> 4));
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_ss_lo(tmem + col_s(hf), k_lo + kstep_off(k), q_lo0 + so + kstep_off(k), dhi, idesc_s, k > 0);
                if (bias)
                    mma_ss_lo(tmem + col_s(hf), aa_lo,
                              ab_lo0 + static_cast<uint32_t>((t % S) * (kAugTile >> 4) + ((hf * 2048) >> 4)), ahi,
                              idesc_s, 1u);
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    mma_ss_lo(tmem + col_dp(hf), v_lo + kstep_off(k), do_lo0 + so + kstep_off(k), dhi, idesc_s, k > 0);
                mma_commit(&s_full[hf]);
            };
            bool ok = wait1(kv_full, 0, abort_flag, a.status) && ready(0);
            if (ok) {
                tc_fence_after();
                issue_sdp(0);
                issue_sdp(1);
            }
            for (int u = 0; u < U && ok; ++u) {
                const int t = u >> 1, hf = u & 1;
                const int st = t % S;
                if (!(ok = wait1(&p_full[hf], static_cast<uint32_t>(t) & 1, abort_flag, a.status))) break;
                tc_fence_after();
                // dV += P^T dO and dK += dS^T Q over the half's 64 queries (16 rows of the MN-major tiles per step)
                const uint32_t so = static_cast<uint32_t>(st * (C::kTile >> 4) + ((hf * kHalf * 128) >> 4));
#pragma unroll
                for (int k = 0; k < kHalf / 16; ++k)
                    mma_ts_lo(tmem + C::kColDV, tmem + col_s(hf) + a_col(k),
                              domn_lo0 + so + static_cast<uint32_t>(k * (2048 >> 4)), dhi, idesc_o,
                              (u > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < kHalf / 16; ++k)
                    mma_ts_lo(tmem + C::kColDK, tmem + col_dp(hf) + a_col(k),
                              qmn_lo0 + so + static_cast<uint32_t>(k * (2048 >> 4)), dhi, idesc_o,
                              (u > 0 || k > 0) ? 1u : 0u);
                if (hf == 1) mma_commit(&st_empty[st]);  // both halves of the step consumed
                if (u + 2 < U) {
                    if (hf == 0 && !(ok = ready(t + 1))) break;
                    issue_sdp(u + 2);
                } else if (u == U - 1) {
                    mma_commit(o_full);
                }
            }
            if (!ok) {
                mma_commit(drain);
                volatile int no_abort = 0;
                wait1(drain, 0, &no_abort, a.status);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ bias operand B: gamma_h of each step
        uint4* aug_b = reinterpret_cast<uint4*>(smem + C::kOffAugB);
        for (int t = 0; t < T; ++t) {
            const int st = t % S;
            if (!wait1(&st_empty[st], (static_cast<uint32_t>(t / S) & 1) ^ 1, abort_flag, a.status)) break;
            const int head = kvh * a.G + t / nq;
            __nv_bfloat16 g[3];
            split3_bf16(a.gain ? a.gain[head] * kLog2e / a.scale_log2 : 0.0f, g);
            uint4* dst = aug_b + st * (kAugTile / 16);
            for (int r = lane; r < kB; r += 32) aug_row_repeated(dst, r, g);
            fence_proxy_async_smem();
            mbar_arrive(&aug_full[st]);
        }
    } else {
        // ------------------------------------------------------------ P^T, dS^T, column sums; dk/dv epilogue
        const int sw = warp - 3;
        const int wg = sw >> 2;              // which kWGCols queries of each half
        const int qd = warp & 3;
        const int row = qd * 32 + lane;      // key in the tile == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
        const int64_t key = static_cast<int64_t>(n_tile) * kB + row;
        const float s_c = (a.s_kept && key < a.K) ? a.s_kept[key] : 0.0f;
        float ds_acc = 0.0f, cs = 0.0f;  // sum_h g_h colsum_h, and the current head's colsum
        // the current head's column sum into ds, and s_c times it into the warp's dg slot
        auto flush = [&](int hh) {
            const int head = kvh * a.G + hh;
            ds_acc = fmaf(a.gain ? a.gain[head] : 0.0f, cs, ds_acc);
            float d = s_c * cs;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (lane == 0) dgw[sw * kMaxGroup + hh] = d;
            cs = 0.0f;
        };
        bool ok = true;
        for (int u = 0; u < U && ok; ++u) {
            const int t = u >> 1, hf = u & 1;
            const int st = t % S;
            const int hh = t / nq;
            const int i = n_tile + t % nq;
            if (hf == 0 && t > 0 && t % nq == 0) flush(hh - 1);
            if (!(ok = warp_wait(&s_full[hf], static_cast<uint32_t>(t) & 1, abort_flag, a.status))) break;
            tc_fence_after();
            const float* lse2s = reinterpret_cast<const float*>(smem + C::kOffVec + st * 1024);
            const float* dvs = lse2s + kB;
            const bool diag = i == n_tile;
            const int c0 = kWGCols * wg;          // first query of this warpgroup in the half
            const int q0 = hf * kHalf + c0;       // ... and in the tile
            uint32_t sv[32], pv[32];
            tmem_ld32(tmem + lane_off + col_s(hf) + c0, sv);
            tmem_ld32(tmem + lane_off + col_dp(hf) + c0, pv);
            tmem_ld_wait();
            uint32_t p16[16], d16[16];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 L = *reinterpret_cast<const float4*>(lse2s + q0 + e);
                const float4 Dd = *reinterpret_cast<const float4*>(dvs + q0 + e);
                const float lv[4] = {L.x, L.y, L.z, L.w};
                const float dv4[4] = {Dd.x, Dd.y, Dd.z, Dd.w};
                float p[4], ds[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    p[w] = ex2(fmaf(__uint_as_float(sv[e + w]), a.scale_log2, -lv[w]));
                    if (diag && q0 + e + w < row) p[w] = 0.0f;  // query before the key
                    ds[w] = p[w] * (__uint_as_float(pv[e + w]) - dv4[w]);
                    cs += ds[w];
                }
                p16[e >> 1] = pack_bf16x2(p[0], p[1]);
                p16[(e >> 1) + 1] = pack_bf16x2(p[2], p[3]);
                d16[e >> 1] = pack_bf16x2(ds[0], ds[1]);
                d16[(e >> 1) + 1] = pack_bf16x2(ds[2], ds[3]);
            }
            tmem_st16(tmem + lane_off + col_s(hf) + c0, p16);
            tmem_st16(tmem + lane_off + col_dp(hf) + c0, d16);
            tmem_st_wait();
            fence_proxy_async_smem();  // the lse2 / D reads come before the stage is refilled by TMA
            tc_fence_before();
            mbar_arrive(&p_full[hf]);
        }
        if (ok) {
            flush(a.G - 1);
            dsw[wg * kB + row] = ds_acc;
        }
        if (ok && warp_wait(o_full, 0, abort_flag, a.status)) {
            tc_fence_after();
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
                const uint32_t col0 = pass == 0 ? C::kColDV : C::kColDK;
                const float f = pass == 0 ? 1.0f : a.scale;
                __nv_bfloat16* dst_row = (pass == 0 ? a.dv : a.dk) + (key * a.Hkv + kvh) * D;
#pragma unroll
                for (int c0 = wg * (D / kWG); c0 < (wg + 1) * (D / kWG); c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem + lane_off + col0 + c0, v);
                    tmem_ld_wait();
                    if (key < a.K) {
                        uint32_t o[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            o[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * f, __uint_as_float(v[2 * e + 1]) * f);
                        uint4* dst = reinterpret_cast<uint4*>(dst_row + c0);
                        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x < kB) {
        float t = 0.0f;
        for (int w = 0; w < kWG; ++w) t += dsw[w * kB + threadIdx.x];
        a.ds_part[kvh * a.Kp + static_cast<int64_t>(n_tile) * kB + threadIdx.x] = t;
    }
    if (threadIdx.x < a.G) {
        float t = 0.0f;
        for (int w = 0; w < kSoftWarps; ++w) t += dgw[w * kMaxGroup + threadIdx.x];
        a.dg_part[static_cast<int64_t>(kvh * a.G + threadIdx.x) * a.num_k_tiles + n_tile] = t;
    }
}

// ============================================================== finish: fixed-order reductions
__global__ void __launch_bounds__(256) bwd_finish_kernel(const float* __restrict__ ds_part,
                                                         const float* __restrict__ dg_part,
                                                         const float* __restrict__ dtau_part, int64_t K, int64_t Kp,
                                                         int Hq, int Hkv, int num_k_tiles, int n_dq_ctas,
                                                         float inv_sqrt_d, float* ds, float* dg, float* dtau) {
    __shared__ float red[256];
    if (ds) {
        for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < K;
             c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
            float t = 0.0f;
            for (int h = 0; h < Hkv; ++h) t += ds_part[h * Kp + c];
            ds[c] = t;
        }
    }
    if (blockIdx.x == 0) {
        if (dg)
            for (int h = threadIdx.x; h < Hq; h += blockDim.x) {
                float t = 0.0f;
                for (int n = 0; n < num_k_tiles; ++n) t += dg_part[static_cast<int64_t>(h) * num_k_tiles + n];
                dg[h] = t;
            }
        // dtau: strided partial sums, then a fixed tree (the same order on every run)
        float t = 0.0f;
        for (int i = threadIdx.x; i < n_dq_ctas; i += blockDim.x) t += dtau_part[i];
        red[threadIdx.x] = t;
        __syncthreads();
        for (int w = blockDim.x / 2; w > 0; w >>= 1) {
            if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
            __syncthreads();
        }
        if (dtau && threadIdx.x == 0) *dtau = red[0] * inv_sqrt_d;
    }
}

}  // namespace bwd

// Workspace layout of the backward (after the 256-byte status header), every region 256-byte aligned.
struct BwdLayout {
    int64_t Kp;
    int nqt;
    size_t lse2, dvec, ds_part, dg_part, dtau_part, total;
};
static BwdLayout bwd_layout(int64_t K, int Hq, int Hkv) {
    BwdLayout L;
    L.Kp = ((K + bwd::kB - 1) / bwd::kB) * bwd::kB;
    L.nqt = static_cast<int>(L.Kp / bwd::kB);
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    size_t off = kWsHeader;
    L.lse2 = off;
    off += up(sizeof(float) * static_cast<size_t>(Hq) * L.Kp);
    L.dvec = off;
    off += up(sizeof(float) * static_cast<size_t>(Hq) * L.Kp);
    L.ds_part = off;
    off += up(sizeof(float) * static_cast<size_t>(Hkv) * L.Kp);
    L.dg_part = off;
    off += up(sizeof(float) * static_cast<size_t>(Hq) * L.nqt);
    L.dtau_part = off;
    off += up(sizeof(float) * static_cast<size_t>(Hq) * L.nqt);
    L.total = off;
    return L;
}

size_t ws_attn_bwd_bytes(int64_t K, int32_t Hq, int32_t Hkv) {
    if (K < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0) return 0;
    return bwd_layout(K, Hq, Hkv).total;
}

}  // namespace tg

using namespace tg;

namespace {
template <int D>
tg_status launch_bwd(const CUtensorMap& mq, const CUtensorMap& mdo, const CUtensorMap& mk, const CUtensorMap& mv,
                     const bwd::ArgsQ& aq, const bwd::ArgsKV& akv, cudaStream_t st) {
    {
        auto kern = bwd::bwd_dq_kernel<D>;
        static std::atomic<int> smem_set[64];
        if (!set_max_dynamic_smem(kern, bwd::CfgQ<D>::kSmem, smem_set)) return TG_ERR_CUDA;
        const int64_t grid = static_cast<int64_t>(aq.num_q_tiles) * aq.Hq;
        if (grid > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
        kern<<<static_cast<unsigned>(grid), bwd::kThreads, bwd::CfgQ<D>::kSmem, st>>>(mq, mdo, mk, mv, aq);
        if (launch_status() != TG_OK) return TG_ERR_CUDA;
    }
    {
        auto kern = bwd::bwd_dkdv_kernel<D>;
        static std::atomic<int> smem_set[64];
        if (!set_max_dynamic_smem(kern, bwd::CfgKV<D>::kSmem, smem_set)) return TG_ERR_CUDA;
        const int64_t grid = static_cast<int64_t>(akv.num_k_tiles) * akv.Hkv;
        if (grid > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
        kern<<<static_cast<unsigned>(grid), bwd::kThreads, bwd::CfgKV<D>::kSmem, st>>>(mq, mdo, mk, mv, akv);
        if (launch_status() != TG_OK) return TG_ERR_CUDA;
    }
    return TG_OK;
}
}  // namespace

extern "C" tg_status tg_gated_attention_backward(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                                 const tg_bf16* v, int64_t ld_v, int64_t K, int32_t Hq, int32_t Hkv,
                                                 int32_t d_h, const float* s_kept, const float* gain, float tau,
                                                 const tg_bf16* out, const tg_bf16* dout, const float* lse,
                                                 tg_bf16* dq, tg_bf16* dk, tg_bf16* dv, float* ds, float* dg,
                                                 float* dtau, void* workspace, size_t workspace_bytes, void* stream) {
    if (K < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || !std::isfinite(tau) || !(tau > 0.0f))
        return TG_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return TG_ERR_UNSUPPORTED;
    if (Hq / Hkv > bwd::kMaxGroup) return TG_ERR_UNSUPPORTED;
    if (K > 0x7fffffffLL - bwd::kB) return TG_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    if (K == 0) {
        if (dg && cudaMemsetAsync(dg, 0, sizeof(float) * Hq, st) != cudaSuccess) return TG_ERR_CUDA;
        if (dtau && cudaMemsetAsync(dtau, 0, sizeof(float), st) != cudaSuccess) return TG_ERR_CUDA;
        return TG_OK;
    }
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !workspace) return TG_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return TG_ERR_INVALID_ARG;
    if (ld_q < static_cast<int64_t>(Hq) * d_h || ld_k < static_cast<int64_t>(Hkv) * d_h ||
        ld_v < static_cast<int64_t>(Hkv) * d_h || (ld_q % 8) || (ld_k % 8) || (ld_v % 8))
        return TG_ERR_INVALID_ARG;
    const BwdLayout L = bwd_layout(K, Hq, Hkv);
    if (workspace_bytes < L.total) return TG_ERR_INVALID_ARG;
    char* ws = static_cast<char*>(workspace);
    float* lse2 = reinterpret_cast<float*>(ws + L.lse2);
    float* dvec = reinterpret_cast<float*>(ws + L.dvec);
    float* ds_part = reinterpret_cast<float*>(ws + L.ds_part);
    float* dg_part = reinterpret_cast<float*>(ws + L.dg_part);
    float* dtau_part = reinterpret_cast<float*>(ws + L.dtau_part);
    {
        const int64_t items = L.Kp * Hq;
        const int64_t blocks = std::min<int64_t>((items + 255) / 256, static_cast<int64_t>(num_sms()) * 64);
        const auto* o16 = reinterpret_cast<const __nv_bfloat16*>(out);
        const auto* g16 = reinterpret_cast<const __nv_bfloat16*>(dout);
        if (d_h == 128)
            bwd::bwd_prep_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(o16, g16, lse, K, L.Kp, Hq, lse2,
                                                                                     dvec);
        else
            bwd::bwd_prep_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(o16, g16, lse, K, L.Kp, Hq, lse2,
                                                                                    dvec);
        if (launch_status() != TG_OK) return TG_ERR_CUDA;
    }
    CUtensorMap mq, mdo, mk, mv;
    const uint32_t box[3] = {64, 1, static_cast<uint32_t>(bwd::kB)};
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(d_h), static_cast<uint64_t>(Hq), static_cast<uint64_t>(K)};
        const uint64_t sq[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_q) * 2};
        const uint64_t so[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(Hq) * d_h * 2};
        if (!make_tmap_bf16(&mq, q, 3, dims, sq, box) || !make_tmap_bf16(&mdo, dout, 3, dims, so, box))
            return TG_ERR_CUDA;
    }
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(d_h), static_cast<uint64_t>(Hkv), static_cast<uint64_t>(K)};
        const uint64_t sk[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_k) * 2};
        const uint64_t sv[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_v) * 2};
        if (!make_tmap_bf16(&mk, k, 3, dims, sk, box) || !make_tmap_bf16(&mv, v, 3, dims, sv, box))
            return TG_ERR_CUDA;
    }
    const float scale = tau / std::sqrt(static_cast<float>(d_h));
    bwd::ArgsQ aq;
    aq.K = K;
    aq.Kp = L.Kp;
    aq.Hq = Hq;
    aq.G = Hq / Hkv;
    aq.num_q_tiles = L.nqt;
    aq.scale_log2 = scale * bwd::kLog2e;
    aq.scale = scale;
    aq.s_kept = s_kept;
    aq.gain = gain;
    aq.lse2 = lse2;
    aq.dvec = dvec;
    aq.q = reinterpret_cast<const __nv_bfloat16*>(q);
    aq.ld_q = ld_q;
    aq.dq = reinterpret_cast<__nv_bfloat16*>(dq);
    aq.dtau_part = dtau_part;
    aq.status = status_word(workspace);
    bwd::ArgsKV akv;
    akv.K = K;
    akv.Kp = L.Kp;
    akv.Hq = Hq;
    akv.Hkv = Hkv;
    akv.G = Hq / Hkv;
    akv.num_q_tiles = L.nqt;
    akv.num_k_tiles = L.nqt;
    akv.scale_log2 = aq.scale_log2;
    akv.scale = scale;
    akv.s_kept = s_kept;
    akv.gain = gain;
    akv.lse2 = lse2;
    akv.dvec = dvec;
    akv.dk = reinterpret_cast<__nv_bfloat16*>(dk);
    akv.dv = reinterpret_cast<__nv_bfloat16*>(dv);
    akv.ds_part = ds_part;
    akv.dg_part = dg_part;
    akv.status = aq.status;
    const tg_status r = d_h == 128 ? launch_bwd<128>(mq, mdo, mk, mv, aq, akv, st)
                                   : launch_bwd<64>(mq, mdo, mk, mv, aq, akv, st);
    if (r != TG_OK) return r;
    const int64_t fb = std::min<int64_t>((K + 255) / 256, static_cast<int64_t>(num_sms()) * 4);
    bwd::bwd_finish_kernel<<<static_cast<unsigned>(fb), 256, 0, st>>>(
        ds_part, dg_part, dtau_part, K, L.Kp, Hq, Hkv, L.nqt, L.nqt * Hq, 1.0f / std::sqrt(static_cast<float>(d_h)),
        ds, dg, dtau);
    return launch_status();
}
