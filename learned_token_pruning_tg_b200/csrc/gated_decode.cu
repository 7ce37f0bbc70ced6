// gated_decode.cu -- one decoding step of token-gated attention over a KV cache.
//
// After a pruned prefill, the layers above the gate layer keep only the kept
// tokens' keys and values, and each kept key keeps its gate score as a logit
// bias (TokenGate: aiproducthub.cn article, paragraph 事件详情; chathome.org
// article, section トークンゲート付きアテンションとは).  A decoding step's query
// attends to every key in the cache (its own included, so no causal mask):
//   l_c = tau * (q_h . k_{c,kv(h)}) / sqrt(d_h) + g_h * s_c,   c < T
//   out_h = sum_c softmax_c(l_c) v_{c,kv(h)}
// The step reads the whole cache once, so it is bound by HBM bandwidth:
// T * Hkv * d_h * 2 bytes of K and as many of V (+ 4T of scores).
//
// Kernel: grid (Hkv, splits), 16 warps per CTA.  A CTA owns one KV head (and
// the G = Hq / Hkv query heads that read it) and one contiguous range of keys.
// Its key range (a multiple of 64 keys long) streams through a 4-stage ring in
// shared memory (64 keys' K and V rows and scores a stage, one TMA box per
// matrix (d_h x 1 head x 64 keys, no swizzle, keys past T read as zeros) and
// one for the scores, issued by one thread and completing on the stage's
// mbarrier: 128 KB in flight per CTA for d_h = 128, as HBM latency needs; one
// wave of CTAs).  A key is handled by a group of LPK lanes (8 for
// G <= 2, 16 for G = 4, 32 for G = 8, which keeps the registers per lane
// about the same): each lane holds d_h / LPK elements of every query head
// (scaled by tau / sqrt(d_h) log2(e)) and of the output, as 16-byte units
// j LPK + sub of the row (8-byte units when it holds only 4 elements), so a
// quarter-warp -- one lane group or half of one -- reads 128 contiguous bytes of
// one row from shared memory (no bank conflicts); the group reduces the G
// partial dot products with log2(LPK) xor shuffles.  Every lane group keeps its own fp32
// online softmax (running max, sum, output piece) over the keys it sees; the
// groups of a warp merge by shuffles at the end, then the warps' states
// are merged in shared memory, the CTA writes (m, l, o) to the workspace, and
// the last CTA of the KV head (a counter in the workspace, reset by that CTA)
// merges all splits and writes out (bf16) and the log-sum-exp.  Waits on the
// copies are bounded (TG_STATUS_DECODE_TIMEOUT); no thread waits on another.
#include <cmath>

#include "tg_host.cuh"

namespace tg {
namespace dec {

constexpr int kWarps = 16;
constexpr int kStageKeys = 64;
constexpr int kUnroll = kStageKeys / kWarps;  // keys per warp per stage
constexpr int kRing = 4;                    // stages in flight
constexpr int kMaxSplits = 64;
constexpr int kMaxD = 128;
constexpr float kLog2e = 1.4426950408889634f;

struct Args {
    const __nv_bfloat16* q;   // [Hq, d_h]
    const __nv_bfloat16* k;   // [T, Hkv, d_h], token stride ld_k
    const __nv_bfloat16* v;
    int64_t ld_k, ld_v, T;
    int Hkv;
    int split_len;            // keys per split
    float scale_log2;         // tau / sqrt(d_h) * log2(e)
    const float* s;           // [T] or NULL
    const float* gain;        // [Hq] or NULL
    __nv_bfloat16* out;       // [Hq, d_h]
    float* lse;               // [Hq] or NULL
    float* part;              // [Hq][kMaxSplits][2 + d_h]: m, l (log2 units), o
    unsigned int* counter;    // [Hkv]
    unsigned int* status;     // the workspace's status word
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One-dimensional tiled TMA load (coordinate c0 in elements) completing on `bar`.
__device__ __forceinline__ void tma_load_1d(void* dst, const void* tmap, uint64_t* bar, int c0, uint64_t cache_hint) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2}], [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(c0), "r"(smem_u32(bar)), "l"(cache_hint)
        : "memory");
}

// EW consecutive bf16 elements (4 or 8: one 8- or 16-byte load) widened to fp32.
template <int EW>
__device__ __forceinline__ void load_unit(const __nv_bfloat16* p, float (&f)[EW]) {
    if constexpr (EW == 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        f[0] = __uint_as_float(u.x << 16);
        f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16);
        f[3] = __uint_as_float(u.y & 0xffff0000u);
    }
}

// Lanes that share one key: fewer lanes (fewer shuffles per key) when few query
// heads read the KV head, at most d_h / 4 so that a lane holds whole 8-byte pieces.
template <int D, int G>
struct Lanes {
    static constexpr int kByG = G <= 2 ? 8 : (G == 4 ? 16 : 32);
    static constexpr int kPerKey = kByG < D / 4 ? kByG : D / 4;
};

template <int D, int G>
__global__ void __launch_bounds__(kWarps * 32)
gated_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_s, const Args a) {
    constexpr int LPK = Lanes<D, G>::kPerKey;
    constexpr int ED = D / LPK;          // elements per lane (multiple of 4)
    static_assert(ED % 4 == 0, "a lane holds whole 8-byte pieces");
    constexpr int EW = ED >= 8 ? 8 : 4;  // elements per unit: a 16-byte (or 8-byte) load
    constexpr int NU = ED / EW;          // units per lane; unit j of lane `sub` is unit j LPK + sub of the row
    constexpr int KPS = 32 / LPK;        // keys a warp handles at once
    __shared__ float s_m[kWarps][G], s_l[kWarps][G];
    __shared__ bool s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = lane / LPK, sub = lane % LPK;
    const int kvh = blockIdx.x, split = blockIdx.y;
    const int64_t c_begin = static_cast<int64_t>(split) * a.split_len;
    const int64_t c_end = min(c_begin + a.split_len, a.T);

    float qr[G][ED], gl2[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int head = kvh * G + g;
#pragma unroll
        for (int j = 0; j < NU; ++j) {
            float f[EW];
            load_unit<EW>(a.q + static_cast<int64_t>(head) * D + (j * LPK + sub) * EW, f);
#pragma unroll
            for (int i = 0; i < EW; ++i) qr[g][j * EW + i] = f[i] * a.scale_log2;
        }
        gl2[g] = a.gain ? a.gain[head] * kLog2e : 0.0f;
    }
    float m[G], l[G], o[G][ED];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.0f;
#pragma unroll
        for (int e = 0; e < ED; ++e) o[g][e] = 0.0f;
    }

    constexpr int kRow = D * 2;                        // bytes of one key's row (one head)
    constexpr int kScoreOff = kStageKeys * kRow * 2;    // K rows, then V rows, then the 64 scores
    constexpr int kStageBytes = kScoreOff + kStageKeys * 4;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t full[kRing];
    __shared__ int abort_flag;
    const int n_keys = static_cast<int>(c_end - c_begin);
    const int n_stages = (n_keys + kStageKeys - 1) / kStageKeys;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRing; ++i) mbar_init(&full[i], 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
        if (a.s) tma_prefetch_desc(&tmap_s);
    }
    __syncthreads();
    // one thread: stage t's K and V boxes into slot t mod kRing
    auto issue = [&](int t) {
        if (lane != 0) return;
        uint8_t* slot = ring + (t % kRing) * kStageBytes;
        uint64_t* bar = &full[t % kRing];
        const int c_first = static_cast<int>(c_begin) + t * kStageKeys;
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(a.s ? kStageBytes : kScoreOff));
        tma_load_3d(slot, &tmap_k, bar, 0, kvh, c_first, kEvictFirst);
        tma_load_3d(slot + kStageKeys * kRow, &tmap_v, bar, 0, kvh, c_first, kEvictFirst);
        if (a.s) tma_load_1d(slot + kScoreOff, &tmap_s, bar, c_first, kEvictFirst);
    };
    if (warp == 0)
        for (int t = 0; t < kRing - 1 && t < n_stages; ++t) issue(t);
    bool ok = true;
    int t = 0;
    for (; t < n_stages; ++t) {
        if (warp == 0 && t + kRing - 1 < n_stages) issue(t + kRing - 1);
        ok = mbar_wait(&full[t % kRing], static_cast<uint32_t>(t / kRing) & 1, &abort_flag, a.status,
                       TG_STATUS_DECODE_TIMEOUT);
        if (!__syncthreads_and(ok)) break;  // every thread leaves together
        const uint8_t* slot = ring + (t % kRing) * kStageBytes;
#pragma unroll
        for (int step = 0; step < kUnroll / KPS; ++step) {
            // this lane group's key of the step
            const int r = warp * kUnroll + step * KPS + grp;
            const int64_t c = c_begin + static_cast<int64_t>(t) * kStageKeys + r;
            const bool valid = c < c_end;
            float kf[ED], vf[ED];
#pragma unroll
            for (int j = 0; j < NU; ++j) {
                const int off = (j * LPK + sub) * EW * 2;
                if (valid) {
                    load_unit<EW>(reinterpret_cast<const __nv_bfloat16*>(slot + r * kRow + off),
                                  *reinterpret_cast<float(*)[EW]>(kf + j * EW));
                    load_unit<EW>(reinterpret_cast<const __nv_bfloat16*>(slot + kStageKeys * kRow + r * kRow + off),
                                  *reinterpret_cast<float(*)[EW]>(vf + j * EW));
                } else {  // past the range: the slot holds another key or zeros here (weight 0)
#pragma unroll
                    for (int i = 0; i < EW; ++i) kf[j * EW + i] = vf[j * EW + i] = 0.0f;
                }
            }
            const float sb = (valid && a.s) ? reinterpret_cast<const float*>(slot + kScoreOff)[r] : 0.0f;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float d = 0.0f;
#pragma unroll
                for (int e = 0; e < ED; ++e) d = fmaf(qr[g][e], kf[e], d);
#pragma unroll
                for (int off = LPK / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
                if (!valid) continue;  // uniform over the lane group
                const float x = d + gl2[g] * sb;
                if (x > m[g]) {        // new running max for this group (rescale its state)
                    const float alpha = ex2(m[g] - x);
                    m[g] = x;
                    l[g] *= alpha;
#pragma unroll
                    for (int e = 0; e < ED; ++e) o[g][e] *= alpha;
                }
                const float p = ex2(x - m[g]);
                l[g] += p;
#pragma unroll
                for (int e = 0; e < ED; ++e) o[g][e] = fmaf(p, vf[e], o[g][e]);
            }
        }
        // these generic-proxy reads of the slot come before the bulk copies (async proxy) that
        // refill it once every thread is past the barrier
        fence_proxy_async_smem();
        __syncthreads();
    }
    if (t < n_stages) {
        // gave up: let the copies already issued land before the CTA's shared memory goes away
        if (threadIdx.x == 0) {
            volatile int no_abort = 0;
            for (int u = t; u < n_stages && u < t + kRing; ++u)
                mbar_wait(&full[u % kRing], static_cast<uint32_t>(u / kRing) & 1, &no_abort, a.status,
                          TG_STATUS_DECODE_TIMEOUT);
        }
        __syncthreads();
        return;
    }

    // merge the lane groups of each warp (lanes sub, sub + LPK, ... hold the same output piece)
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int off = LPK; off < 32; off <<= 1) {
            const float mo = __shfl_xor_sync(0xffffffffu, m[g], off);
            const float lo = __shfl_xor_sync(0xffffffffu, l[g], off);
            const float mx = fmaxf(m[g], mo);
            const float fa = m[g] == -INFINITY ? 0.0f : ex2(m[g] - mx);
            const float fb = mo == -INFINITY ? 0.0f : ex2(mo - mx);
            l[g] = l[g] * fa + lo * fb;
#pragma unroll
            for (int e = 0; e < ED; ++e) {
                const float oo = __shfl_xor_sync(0xffffffffu, o[g][e], off);
                o[g][e] = o[g][e] * fa + oo * fb;
            }
            m[g] = mx;
        }
    }
    // merge the warps' states (through the ring, idle now: every stage has landed and been read)
    float (*s_o)[G][D] = reinterpret_cast<float (*)[G][D]>(ring);
    static_assert(kWarps * G * D * 4 <= kRing * (kStageKeys * D * 2 * 2), "the merge fits in the ring");
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (lane == 0) {
            s_m[warp][g] = m[g];
            s_l[warp][g] = l[g];
        }
        if (grp == 0) {
#pragma unroll
            for (int j = 0; j < NU; ++j)
#pragma unroll
                for (int i = 0; i < EW; ++i) s_o[warp][g][(j * LPK + sub) * EW + i] = o[g][j * EW + i];
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += kWarps * 32) {
        const int g = i / D, col = i % D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, s_m[w][g]);
        float ls = 0.0f, os = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float f = s_m[w][g] == -INFINITY ? 0.0f : ex2(s_m[w][g] - mx);
            ls += s_l[w][g] * f;
            os += s_o[w][g][col] * f;
        }
        float* pr = a.part + (static_cast<int64_t>(kvh * G + g) * kMaxSplits + split) * (2 + D);
        if (col == 0) {
            pr[0] = mx;
            pr[1] = ls;
        }
        pr[2 + col] = os;
    }

    // the last CTA of this KV head merges every split
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(&a.counter[kvh], 1u);
        s_last = prev == gridDim.y - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int nsplit = static_cast<int>(gridDim.y);
    for (int i = threadIdx.x; i < G * D; i += kWarps * 32) {
        const int g = i / D, col = i % D;
        const int head = kvh * G + g;
        const float* pr = a.part + static_cast<int64_t>(head) * kMaxSplits * (2 + D);
        float mx = -INFINITY;
        for (int sp = 0; sp < nsplit; ++sp) mx = fmaxf(mx, __ldcg(pr + sp * (2 + D)));
        float ls = 0.0f, os = 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) {
            const float ms = __ldcg(pr + sp * (2 + D));
            if (ms == -INFINITY) continue;
            const float f = ex2(ms - mx);
            ls += __ldcg(pr + sp * (2 + D) + 1) * f;
            os += __ldcg(pr + sp * (2 + D) + 2 + col) * f;
        }
        a.out[static_cast<int64_t>(head) * D + col] = __float2bfloat16_rn(os / ls);
        if (col == 0 && a.lse) a.lse[head] = (mx + log2f(ls)) / kLog2e;
    }
    if (threadIdx.x == 0) a.counter[kvh] = 0;  // ready for the next call on this workspace
}

// Splits of the key range: one wave of CTAs over the GPU (resident CTAs per SM
// from the occupancy calculator, cached per kernel and device), at least 64
// keys per split.
template <int D, int G>
static tg_status launch(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& ms, Args a, int64_t T,
                        cudaStream_t st) {
    static std::atomic<int> occ_cache[64];
    static std::atomic<int> smem_set0[64];
    const int dev = current_device();
    int occ = dev >= 0 ? occ_cache[dev].load(std::memory_order_relaxed) : 0;
    if (occ <= 0) {
        if (!set_max_dynamic_smem(gated_decode_kernel<D, G>, kRing * (kStageKeys * D * 2 * 2 + kStageKeys * 4), smem_set0) ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gated_decode_kernel<D, G>, kWarps * 32,
                                                          kRing * (kStageKeys * D * 2 * 2 + kStageKeys * 4)) !=
                cudaSuccess ||
            occ <= 0)
            occ = 1;
        if (dev >= 0) occ_cache[dev].store(occ, std::memory_order_relaxed);
    }
    int64_t nsplit = static_cast<int64_t>(num_sms()) * occ / a.Hkv;
    if (nsplit > (T + 63) / 64) nsplit = (T + 63) / 64;
    if (nsplit > kMaxSplits) nsplit = kMaxSplits;
    if (nsplit < 1) nsplit = 1;
    // split lengths are multiples of the 64-key stage (the scores' TMA coordinate must be a multiple of 4)
    a.split_len = static_cast<int>(((T + nsplit - 1) / nsplit + kStageKeys - 1) / kStageKeys * kStageKeys);
    nsplit = (T + a.split_len - 1) / a.split_len;
    constexpr int kSmem = kRing * (kStageKeys * D * 2 * 2 + kStageKeys * 4);  // the ring
    static std::atomic<int> smem_set[64];
    if (!set_max_dynamic_smem(gated_decode_kernel<D, G>, kSmem, smem_set)) return TG_ERR_CUDA;
    gated_decode_kernel<D, G><<<dim3(static_cast<unsigned>(a.Hkv), static_cast<unsigned>(nsplit)), kWarps * 32,
                                kSmem, st>>>(mk, mv, ms, a);
    return launch_status();
}

template <int D>
static tg_status launch_g(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& ms, const Args& a, int G,
                          int64_t T, cudaStream_t st) {
    switch (G) {
        case 1: return launch<D, 1>(mk, mv, ms, a, T, st);
        case 2: return launch<D, 2>(mk, mv, ms, a, T, st);
        case 4: return launch<D, 4>(mk, mv, ms, a, T, st);
        case 8: return launch<D, 8>(mk, mv, ms, a, T, st);
    }
    return TG_ERR_UNSUPPORTED;
}

}  // namespace dec

size_t ws_decode_bytes(int32_t Hq) {
    // status header, Hkv <= Hq counters (one 256-byte line), then the per-split partials
    return kWsHeader + 256 + static_cast<size_t>(Hq) * dec::kMaxSplits * (2 + dec::kMaxD) * sizeof(float);
}

}  // namespace tg

using namespace tg;

extern "C" tg_status tg_gated_decode(const tg_bf16* q, const tg_bf16* k_cache, int64_t ld_k, const tg_bf16* v_cache,
                                     int64_t ld_v, int64_t T, int32_t Hq, int32_t Hkv, int32_t d_h,
                                     const float* s_cache, const float* gain, float tau, tg_bf16* out, float* lse,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    if (T <= 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0 || !std::isfinite(tau)) return TG_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !out || !workspace) return TG_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return TG_ERR_UNSUPPORTED;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return TG_ERR_UNSUPPORTED;
    if (Hkv > 64 || T > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    if (!aligned16(workspace) || workspace_bytes < ws_decode_bytes(Hq)) return TG_ERR_INVALID_ARG;
    // TMA boxes of cache rows (16-byte aligned bases and strides); q read in 16-byte units
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || (ld_k % 8) != 0 || (ld_v % 8) != 0)
        return TG_ERR_INVALID_ARG;
    if (ld_k < static_cast<int64_t>(Hkv) * d_h || ld_v < static_cast<int64_t>(Hkv) * d_h) return TG_ERR_INVALID_ARG;

    dec::Args a;
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.k = reinterpret_cast<const __nv_bfloat16*>(k_cache);
    a.v = reinterpret_cast<const __nv_bfloat16*>(v_cache);
    a.ld_k = ld_k;
    a.ld_v = ld_v;
    a.T = T;
    a.Hkv = Hkv;
    a.scale_log2 = tau / std::sqrt(static_cast<float>(d_h)) * dec::kLog2e;
    a.s = s_cache;
    a.gain = gain;
    a.out = reinterpret_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.counter = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + kWsHeader);
    a.status = status_word(workspace);
    a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kWsHeader + 256);
    a.split_len = 0;
    // K and V as [T, Hkv, d_h] boxes of d_h x 1 x 64 keys, rows kept in order (no swizzle)
    CUtensorMap mk, mv;
    const uint64_t dims[3] = {static_cast<uint64_t>(d_h), static_cast<uint64_t>(Hkv), static_cast<uint64_t>(T)};
    const uint64_t sk[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_k) * 2};
    const uint64_t sv[2] = {static_cast<uint64_t>(d_h) * 2, static_cast<uint64_t>(ld_v) * 2};
    const uint32_t box[3] = {static_cast<uint32_t>(d_h), 1, static_cast<uint32_t>(dec::kStageKeys)};
    if (!make_tmap_bf16(&mk, k_cache, 3, dims, sk, box, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tmap_bf16(&mv, v_cache, 3, dims, sv, box, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
        return TG_ERR_CUDA;
    // the scores as [T] fp32 boxes of 64 (unused without scores: the K map stands in)
    CUtensorMap ms = mk;
    if (s_cache) {
        if (!aligned16(s_cache)) return TG_ERR_INVALID_ARG;
        const uint64_t sdims[1] = {static_cast<uint64_t>(T)};
        const uint32_t sbox[1] = {static_cast<uint32_t>(dec::kStageKeys)};
        if (!make_tmap_bf16(&ms, s_cache, 1, sdims, nullptr, sbox, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
            return TG_ERR_CUDA;
    }
    cudaStream_t st = as_stream(stream);
    return d_h == 128 ? dec::launch_g<128>(mk, mv, ms, a, G, T, st) : dec::launch_g<64>(mk, mv, ms, a, G, T, st);
}
