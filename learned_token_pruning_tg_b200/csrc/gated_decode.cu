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
// Kernel: grid (Hkv, splits), 8 warps per CTA.  A CTA owns one KV head (and
// the G = Hq / Hkv query heads that read it) and one contiguous range of keys.
// Its key range streams through a 4-stage ring in shared memory (64 keys' K
// and V rows a stage, copied with cp.async by all threads, each thread always
// the same row pieces: 128 KB in flight per CTA for d_h = 128, as HBM latency
// needs; one wave of CTAs).  A key is handled by a group of LPK lanes (8 for
// G <= 2, 16 for G = 4, 32 for G = 8, which keeps the registers per lane
// about the same): each lane holds d_h / LPK elements of every query head
// (scaled by tau / sqrt(d_h) log2(e)) and of the output, reads its piece of the
// K and V rows from shared memory, and the group reduces the G partial dot
// products with log2(LPK) xor shuffles.  Every lane group keeps its own fp32
// online softmax (running max, sum, output piece) over the keys it sees; the
// groups of a warp merge by shuffles at the end, then the warps' states
// are merged in shared memory, the CTA writes (m, l, o) to the workspace, and
// the last CTA of the KV head (a counter in the workspace, reset by that CTA)
// merges all splits and writes out (bf16) and the log-sum-exp.  No thread
// waits on another.
#include <cmath>
#include <type_traits>

#include "tg_host.cuh"

namespace tg {
namespace dec {

constexpr int kWarps = 8;
constexpr int kUnroll = 8;                  // keys per warp per stage
constexpr int kStageKeys = kWarps * kUnroll;  // 64
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
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// E consecutive bf16 elements (E = 2 or 4) widened to fp32.
template <int E>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float (&f)[E]) {
    if constexpr (E == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        f[0] = __uint_as_float(u.x << 16);
        f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16);
        f[3] = __uint_as_float(u.y & 0xffff0000u);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
        f[0] = __uint_as_float(u << 16);
        f[1] = __uint_as_float(u & 0xffff0000u);
    }
}

// Raw row pieces: E bf16 (E = 2 or 4) in one 4- or 8-byte load.
template <int E>
struct Piece {
    using T = typename std::conditional<E == 4, uint2, uint32_t>::type;
};
template <int E>
__device__ __forceinline__ void widen(const typename Piece<E>::T& u, float (&f)[E]) {
    if constexpr (E == 4) {
        f[0] = __uint_as_float(u.x << 16);
        f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16);
        f[3] = __uint_as_float(u.y & 0xffff0000u);
    } else {
        f[0] = __uint_as_float(u << 16);
        f[1] = __uint_as_float(u & 0xffff0000u);
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
__global__ void __launch_bounds__(kWarps * 32) gated_decode_kernel(const Args a) {
    constexpr int LPK = Lanes<D, G>::kPerKey;
    constexpr int ED = D / LPK;          // elements per lane (multiple of 4)
    static_assert(ED % 4 == 0, "a lane holds whole 8-byte pieces");
    constexpr int KPS = 32 / LPK;        // keys a warp handles at once
    __shared__ float s_m[kWarps][G], s_l[kWarps][G];
    __shared__ float s_o[kWarps][G][D];
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
        for (int e = 0; e < ED; e += 4) {
            float f[4];
            load_row<4>(a.q + static_cast<int64_t>(head) * D + sub * ED + e, f);
#pragma unroll
            for (int i = 0; i < 4; ++i) qr[g][e + i] = f[i] * a.scale_log2;
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
    constexpr int kStageBytes = kStageKeys * kRow * 2;  // K rows, then V rows
    constexpr int kPiecesPerRow = kRow / 16;
    constexpr int kRowsPerPass = kWarps * 32 / kPiecesPerRow;
    constexpr int kPasses = kStageKeys / kRowsPerPass;
    extern __shared__ __align__(16) uint8_t ring[];
    const int n_keys = static_cast<int>(c_end - c_begin);
    const int n_stages = (n_keys + kStageKeys - 1) / kStageKeys;
    // this thread always copies piece `cp_piece` of rows cp_row + kRowsPerPass j of K and of V
    const int cp_piece = threadIdx.x % kPiecesPerRow, cp_row = threadIdx.x / kPiecesPerRow;
    const char* kg = reinterpret_cast<const char*>(a.k + static_cast<int64_t>(kvh) * D) + cp_piece * 16;
    const char* vg = reinterpret_cast<const char*>(a.v + static_cast<int64_t>(kvh) * D) + cp_piece * 16;
    const int64_t ldk2 = a.ld_k * 2, ldv2 = a.ld_v * 2;
    auto issue = [&](int t) {
        uint8_t* slot = ring + (t % kRing) * kStageBytes + cp_row * kRow + cp_piece * 16;
#pragma unroll
        for (int j = 0; j < kPasses; ++j) {
            const int r = cp_row + j * kRowsPerPass;
            const int64_t c = c_begin + static_cast<int64_t>(t) * kStageKeys + r;
            if (c < c_end) {
                const uint32_t dk = smem_u32(slot + j * kRowsPerPass * kRow);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dk), "l"(kg + c * ldk2) : "memory");
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dk + kStageKeys * kRow),
                             "l"(vg + c * ldv2)
                             : "memory");
            }
        }
    };
    for (int t = 0; t < kRing - 1; ++t) {
        if (t < n_stages) issue(t);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int t = 0; t < n_stages; ++t) {
        if (t + kRing - 1 < n_stages) issue(t + kRing - 1);
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group %0;" ::"n"(kRing - 1) : "memory");  // stage t has landed (own copies)
        __syncthreads();                                                      // ... and everyone's
        const uint8_t* slot = ring + (t % kRing) * kStageBytes;
#pragma unroll
        for (int step = 0; step < kUnroll / KPS; ++step) {
            // this lane group's key of the step
            const int r = warp * kUnroll + step * KPS + grp;
            const int64_t c = c_begin + static_cast<int64_t>(t) * kStageKeys + r;
            const bool valid = c < c_end;
            float kf[ED], vf[ED];
#pragma unroll
            for (int e = 0; e < ED; e += 4) {
                if (valid) {
                    widen<4>(*reinterpret_cast<const uint2*>(slot + r * kRow + (sub * ED + e) * 2),
                             *reinterpret_cast<float(*)[4]>(kf + e));
                    widen<4>(*reinterpret_cast<const uint2*>(slot + kStageKeys * kRow + r * kRow + (sub * ED + e) * 2),
                             *reinterpret_cast<float(*)[4]>(vf + e));
                } else {  // past the range: no row here (weight 0, and no NaN from stale bits)
#pragma unroll
                    for (int i = 0; i < 4; ++i) kf[e + i] = vf[e + i] = 0.0f;
                }
            }
            const float sb = (valid && a.s) ? __ldg(a.s + c) : 0.0f;
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
        __syncthreads();  // the slot is refilled by the next iteration's copies
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");

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
    // merge the warps' states
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (lane == 0) {
            s_m[warp][g] = m[g];
            s_l[warp][g] = l[g];
        }
        if (grp == 0) {
#pragma unroll
            for (int e = 0; e < ED; ++e) s_o[warp][g][sub * ED + e] = o[g][e];
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
static tg_status launch(Args a, int64_t T, cudaStream_t st) {
    static std::atomic<int> occ_cache[64];
    static std::atomic<int> smem_set0[64];
    const int dev = current_device();
    int occ = dev >= 0 ? occ_cache[dev].load(std::memory_order_relaxed) : 0;
    if (occ <= 0) {
        if (!set_max_dynamic_smem(gated_decode_kernel<D, G>, kRing * kStageKeys * D * 2 * 2, smem_set0) ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gated_decode_kernel<D, G>, kWarps * 32,
                                                          kRing * kStageKeys * D * 2 * 2) !=
                cudaSuccess ||
            occ <= 0)
            occ = 1;
        if (dev >= 0) occ_cache[dev].store(occ, std::memory_order_relaxed);
    }
    int64_t nsplit = static_cast<int64_t>(num_sms()) * occ / a.Hkv;
    if (nsplit > (T + 63) / 64) nsplit = (T + 63) / 64;
    if (nsplit > kMaxSplits) nsplit = kMaxSplits;
    if (nsplit < 1) nsplit = 1;
    a.split_len = static_cast<int>((T + nsplit - 1) / nsplit);
    nsplit = (T + a.split_len - 1) / a.split_len;
    constexpr int kSmem = kRing * kStageKeys * D * 2 * 2;
    static std::atomic<int> smem_set[64];
    if (!set_max_dynamic_smem(gated_decode_kernel<D, G>, kSmem, smem_set)) return TG_ERR_CUDA;
    gated_decode_kernel<D, G><<<dim3(static_cast<unsigned>(a.Hkv), static_cast<unsigned>(nsplit)), kWarps * 32,
                                kSmem, st>>>(a);
    return launch_status();
}

template <int D>
static tg_status launch_g(const Args& a, int G, int64_t T, cudaStream_t st) {
    switch (G) {
        case 1: return launch<D, 1>(a, T, st);
        case 2: return launch<D, 2>(a, T, st);
        case 4: return launch<D, 4>(a, T, st);
        case 8: return launch<D, 8>(a, T, st);
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
    // 16-byte copies of cache rows; q read in 8-byte pieces
    if (!aligned16(k_cache) || !aligned16(v_cache) || (ld_k % 8) != 0 || (ld_v % 8) != 0 ||
        reinterpret_cast<uintptr_t>(q) % 8 != 0)
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
    a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kWsHeader + 256);
    a.split_len = 0;
    cudaStream_t st = as_stream(stream);
    return d_h == 128 ? dec::launch_g<128>(a, G, T, st) : dec::launch_g<64>(a, G, T, st);
}
