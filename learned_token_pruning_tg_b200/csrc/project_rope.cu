// project_rope.cu -- the Q/K/V projection of the kept rows with the rotary
// embedding and V's fp16 copy fused into the GEMM's epilogue.
//
// Layers above the gate see only the kept tokens (aiproducthub.cn article,
// paragraph 事件详情; chathome.org article, section TokenGate の学習可能な
// トークンプルーニングの仕組み); their queries and keys are rotated at the kept
// tokens' original positions (the specification's reading: positions travel
// with the rows).  Unfused, the kept rows' projection is a library GEMM whose
// bf16 output RoPE then reads and rewrites, and the attention converts V to
// fp16 in one more pass; here one kernel does all three:
//   qkv[r, :] = x[r, :] W^T                     (bf16 x bf16 -> fp32 in TMEM)
//   q/k heads: rotate-half pairs (t, t + d_h/2) at pos[r], from the fp32
//              accumulator (one bf16 rounding instead of two)
//   v heads:   bf16 into qkv and, when asked, fp16 into v16
// Angles in the epilogue: pos[r] * base^(-2t / d_h) in fp64 (the frequencies
// formed on the host in fp64), reduced modulo 2 pi in fp64, then cos and sin of
// the reduced angle (|x| <= pi) in fp32 -- within 6e-7 of the fp64 values (the fast
// sine and cosine, 2^-21.4 on [-pi, pi], and the fp32 rounding of the angle), far
// below the bf16 rounding of the result.
//
// Kernel (persistent, one CTA per SM, 8 warps): tiles of 128 rows x 256
// output columns, row-tile-major so the CTAs working at one time share the
// rows of x in L2.
//   warp 0      TMA producer: 128 x 64 tiles of x and 256 x 64 tiles of W into
//               a 4-deep ring (128-byte swizzle)
//   warp 1      TMEM allocation (2 x 256 columns) and the single thread that
//               issues tcgen05.mma (M = 128, N = 256, K = 16)
//   warps 4-7   epilogue, one row per thread, double-buffered with the next
//               tile's main loop
// Every wait is bounded (TG_STATUS_PROJECT_TIMEOUT).
// Where the device offers clusters of 2, the same roles run on CTA pairs with
// 256 x 256 tiles and a 6-deep ring (project_rope_pair_kernel below), which
// halves the W bytes each SM moves per stage.
// With a row index array (tg_project_rope_gather) the producer warp fetches the
// x tiles as rows of h instead: lane l issues one TMA gather4 copy of tile rows
// 4l .. 4l + 3 per 64-column step, and each lane checks its indices.
#include <cuda_fp16.h>

#include <cmath>

#include "tg_host.cuh"

namespace tg {
namespace proj {

constexpr int kBM = 128;       // rows per tile
constexpr int kBN = 256;       // output columns per tile
constexpr int kBK = 64;        // K elements per stage (one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr int kThreads = 256;  // 8 warps
constexpr int kStageA = kBM * kBK * 2;
constexpr int kStageB = kBN * kBK * 2;
constexpr int kStage = kStageA + kStageB;
constexpr int kOffBar = kStages * kStage;
constexpr int kNumBars = 2 * kStages + 5;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffMisc + 16 + 1024;
// 128-byte-swizzled TMA destinations start on 1024-byte boundaries; everything fits in 227 KB.
static_assert(kStageA % 1024 == 0 && kStage % 1024 == 0 && kOffBar % 8 == 0 && kSmem <= 232448,
              "projection shared-memory layout");

struct Args {
    double inv_freq[64];  // base^(-2t / d_h), t < d_h / 2, formed on the host in fp64
    int64_t K;
    int d;
    int Hq, Hkv, D;
    int num_col_tiles;
    int64_t num_tiles;
    const int32_t* pos;   // [K] original positions
    const int32_t* rows;  // [K] rows of h to gather (tg_project_rope_gather), or null: x is dense
    int64_t n_rows;       // rows of h (the valid range of `rows`)
    __nv_bfloat16* qkv;
    int64_t ld_qkv;
    __half* v16;          // [K, Hkv D] or null
    unsigned int* status;
};

// The 4 rows of h that lane `lane` of the producer warp gathers for tile rows [r0, r0 + 4): indices
// outside [0, n_rows) are replaced by row 0 and flagged; rows past K (the last tile's tail, whose
// outputs are not stored) read row 0.
__device__ __forceinline__ void gather_rows4(const Args& a, int64_t r0, int (&g)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int v = 0;
        if (r0 + i < a.K) {
            v = __ldg(a.rows + r0 + i);
            if (v < 0 || static_cast<int64_t>(v) >= a.n_rows) {
                atomicOr(a.status, TG_STATUS_INDEX_RANGE);
                v = 0;
            }
        }
        g[i] = v;
    }
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// cos / sin of pos * inv_freq: the angle and its reduction modulo 2 pi in fp64, the cos and sin of
// the reduced angle in fp32 (|angle| <= pi there).
__device__ __forceinline__ void rope_cos_sin(double p, double inv_freq, float* c, float* s) {
    constexpr double kTwoPi = 6.283185307179586;
    constexpr double kInvTwoPi = 0.15915494309189535;
    const double ang = p * inv_freq;
    const double r = fma(-rint(ang * kInvTwoPi), kTwoPi, ang);
    __sincosf(static_cast<float>(r), s, c);
}

// One output tile's epilogue for the thread that owns TMEM lane `row` (row
// `grow` of qkv): the 128 x 256 fp32 accumulator at `taddr` (this thread's
// lane), column tile `ct`.  Query and key heads are rotated and stored in
// bf16; value heads are stored in bf16 and, when asked, fp16.
__device__ __forceinline__ void epilogue_tile(const Args& a, uint32_t taddr, int64_t grow, int ct, bool& v_range) {
    const bool live = grow < a.K;
    const int D = a.D, half = a.D >> 1;
    __nv_bfloat16* orow = a.qkv + grow * a.ld_qkv + static_cast<int64_t>(ct) * kBN;
    for (int c_head = 0; c_head < kBN; c_head += D) {
        const int head = (ct * kBN + c_head) / D;
        if (head < a.Hq + a.Hkv) {
            // rotate-half pairs (t, t + D/2) of a query or key head, 32 pairs at a time
            for (int t0 = 0; t0 < half; t0 += 32) {
                uint32_t x1[32], x2[32];
                tmem_ld32(taddr + c_head + t0, x1);
                tmem_ld32(taddr + c_head + half + t0, x2);
                tmem_ld_wait();
                if (live) {
                    const double p = static_cast<double>(__ldg(a.pos + grow));
                    uint32_t o1[16], o2[16];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float cc[4], ss[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) rope_cos_sin(p, a.inv_freq[t0 + 4 * i + e], &cc[e], &ss[e]);
                        float r1[4], r2[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float u = __uint_as_float(x1[4 * i + e]);
                            const float w = __uint_as_float(x2[4 * i + e]);
                            r1[e] = u * cc[e] - w * ss[e];
                            r2[e] = w * cc[e] + u * ss[e];
                        }
                        o1[2 * i] = pack_bf16x2(r1[0], r1[1]);
                        o1[2 * i + 1] = pack_bf16x2(r1[2], r1[3]);
                        o2[2 * i] = pack_bf16x2(r2[0], r2[1]);
                        o2[2 * i + 1] = pack_bf16x2(r2[2], r2[3]);
                    }
                    uint4* d1 = reinterpret_cast<uint4*>(orow + c_head + t0);
                    uint4* d2 = reinterpret_cast<uint4*>(orow + c_head + half + t0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        d1[i] = make_uint4(o1[4 * i], o1[4 * i + 1], o1[4 * i + 2], o1[4 * i + 3]);
                        d2[i] = make_uint4(o2[4 * i], o2[4 * i + 1], o2[4 * i + 2], o2[4 * i + 3]);
                    }
                }
            }
        } else {
            // a value head: bf16 into qkv and fp16 into v16
            const int vh = head - a.Hq - a.Hkv;
            for (int t0 = 0; t0 < D; t0 += 32) {
                uint32_t x[32];
                tmem_ld32(taddr + c_head + t0, x);
                tmem_ld_wait();
                if (live) {
                    uint32_t ob[16], oh[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float lo = __uint_as_float(x[2 * i]), hi = __uint_as_float(x[2 * i + 1]);
                        ob[i] = pack_bf16x2(lo, hi);
                        oh[i] = pack_f16x2(lo, hi);
                        v_range |= fabsf(lo) > 65504.0f || fabsf(hi) > 65504.0f;
                    }
                    uint4* db = reinterpret_cast<uint4*>(orow + c_head + t0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) db[i] = make_uint4(ob[4 * i], ob[4 * i + 1], ob[4 * i + 2], ob[4 * i + 3]);
                    if (a.v16) {
                        uint4* dh = reinterpret_cast<uint4*>(a.v16 + grow * (static_cast<int64_t>(a.Hkv) * D) +
                                                             static_cast<int64_t>(vh) * D + t0);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dh[i] = make_uint4(oh[4 * i], oh[4 * i + 1], oh[4 * i + 2], oh[4 * i + 3]);
                    }
                }
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
project_rope_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                    const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;                   // [kStages] TMA -> MMA
    uint64_t* empty = bars + kStages;        // [kStages] MMA commit -> TMA
    uint64_t* acc_full = bars + 2 * kStages; // [2] MMA commit -> epilogue
    uint64_t* acc_empty = acc_full + 2;      // [2] 128 epilogue threads -> MMA
    uint64_t* drain = acc_full + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb_per_tile = a.d / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_w);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * kBN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 && a.rows) {
        // ------------------------------------------------------------ TMA producer, rows gathered from h
        // lane l fetches tile rows 4l .. 4l + 3 with one gather4 copy per 64-column step
        int s = 0;
        uint32_t ph = 0;
        int last_ph[kStages];
        for (int i = 0; i < kStages; ++i) last_ph[i] = -1;
        for (int64_t t = blockIdx.x; t < a.num_tiles; t += gridDim.x) {
            if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
            const int rt = static_cast<int>(t / a.num_col_tiles);
            const int ct = static_cast<int>(t % a.num_col_tiles);
            int g[4];
            gather_rows4(a, static_cast<int64_t>(rt) * kBM + lane * 4, g);
            bool ok = true;
            for (int kb = 0; kb < kb_per_tile; ++kb) {
                if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT);
                if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + s * kStage;
                if (lane == 0) mbar_arrive_expect_tx(&full[s], kStage);
                __syncwarp();
                tma_gather4(sa + lane * 512, &tmap_x, &full[s], kb * kBK, g[0], g[1], g[2], g[3], kEvictLast);
                if (lane == 0) tma_load_2d(sa + kStageA, &tmap_w, &full[s], kb * kBK, ct * kBN, kEvictLast);
                last_ph[s] = static_cast<int>(ph);
                if (++s == kStages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (!ok) break;
        }
        // every issued copy lands before shared memory is released (matters on abort only)
        if (lane == 0) {
            volatile int no_abort = 0;
            for (int i = 0; i < kStages; ++i)
                if (last_ph[i] >= 0)
                    mbar_wait(&full[i], static_cast<uint32_t>(last_ph[i]), &no_abort, a.status,
                              TG_STATUS_PROJECT_TIMEOUT);
        }
    } else if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int last_ph[kStages];
            for (int i = 0; i < kStages; ++i) last_ph[i] = -1;
            for (int64_t t = blockIdx.x; t < a.num_tiles && !*abort_flag; t += gridDim.x) {
                const int rt = static_cast<int>(t / a.num_col_tiles);
                const int ct = static_cast<int>(t % a.num_col_tiles);
                for (int kb = 0; kb < kb_per_tile; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT)) break;
                    uint8_t* sa = smem + s * kStage;
                    mbar_arrive_expect_tx(&full[s], kStage);
                    tma_load_2d(sa, &tmap_x, &full[s], kb * kBK, rt * kBM, kEvictLast);
                    tma_load_2d(sa + kStageA, &tmap_w, &full[s], kb * kBK, ct * kBN, kEvictLast);
                    last_ph[s] = static_cast<int>(ph);
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // every issued copy lands before shared memory is released (matters on abort only)
            volatile int no_abort = 0;
            for (int i = 0; i < kStages; ++i)
                if (last_ph[i] >= 0)
                    mbar_wait(&full[i], static_cast<uint32_t>(last_ph[i]), &no_abort, a.status,
                              TG_STATUS_PROJECT_TIMEOUT);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, false);
            int s = 0;
            uint32_t ph = 0;
            int64_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < a.num_tiles && ok; t += gridDim.x, ++it) {
                const int buf = static_cast<int>(it & 1);
                const uint32_t use = static_cast<uint32_t>(it >> 1);
                if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
                for (int kb = 0; kb < kb_per_tile; ++kb) {
                    if (!mbar_wait(&full[s], ph, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * kStage);
                    const uint64_t da = smem_desc_sw128(sa, 16, 1024);
                    const uint64_t db = smem_desc_sw128(sa + kStageA, 16, 1024);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)  // +32 bytes per K = 16 step inside the swizzle row
                        mma_ss(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
                    mma_commit(&empty[s]);
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (ok) mma_commit(&acc_full[buf]);
            }
            if (!ok) {
                mma_commit(drain);
                volatile int no_abort = 0;
                mbar_wait(drain, 0, &no_abort, a.status, TG_STATUS_PROJECT_TIMEOUT);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int qd = warp & 3;             // TMEM lane quarter of this warp
        const int row = qd * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
        bool v_range = false;  // a value beyond fp16's range went into the fp16 copy of V
        int64_t it = 0;
        for (int64_t t = blockIdx.x; t < a.num_tiles; t += gridDim.x, ++it) {
            const int rt = static_cast<int>(t / a.num_col_tiles);
            const int ct = static_cast<int>(t % a.num_col_tiles);
            const int buf = static_cast<int>(it & 1);
            const uint32_t par = static_cast<uint32_t>(it >> 1) & 1;
            // warp-uniform outcome: tcgen05.ld below is warp-collective
            const bool ok = mbar_wait(&acc_full[buf], par, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int64_t grow = static_cast<int64_t>(rt) * kBM + row;
            epilogue_tile(a, tmem_base + lane_off + static_cast<uint32_t>(buf * kBN), grow, ct, v_range);
            tc_fence_before();
            mbar_arrive(&acc_empty[buf]);
        }
        if (v_range && a.v16) atomicOr(a.status, TG_STATUS_V_RANGE);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 2 * kBN);
    }
}

// The same projection on CTA pairs: the two CTAs of a cluster share 256 x 256
// output tiles through one tcgen05.mma.cta_group::2 (M = 256) per 16 columns of
// x; each CTA holds its own 128 rows of x and 128 of the tile's 256 rows of W
// in its own shared memory and receives its 128 rows of the accumulator in its
// own TMEM.  Per 64-column stage a CTA moves 32 KB instead of 48 KB (half of
// W), which is what bounds the single-CTA kernel.  No multicast: every TMA copy
// lands in the CTA that issues it; only its completion is counted on the even
// CTA's barrier, whose thread issues the pair's MMAs.
constexpr int kPairStageA = kBM * kBK * 2;          // 16 KB: 128 rows of x
constexpr int kPairStageB = (kBN / 2) * kBK * 2;    // 16 KB: 128 rows of W
constexpr int kPairStage = kPairStageA + kPairStageB;
constexpr int kPairStages = 6;
constexpr int kPairOffBar = kPairStages * kPairStage;
constexpr int kPairNumBars = 2 * kPairStages + 5;
constexpr int kPairOffMisc = kPairOffBar + kPairNumBars * 8;
constexpr int kPairSmem = kPairOffMisc + 16 + 1024;
static_assert(kPairStageA % 1024 == 0 && kPairStage % 1024 == 0 && kPairOffBar % 8 == 0 && kPairSmem <= 232448,
              "projection pair kernel shared-memory layout");

__global__ void __launch_bounds__(kThreads, 1)
project_rope_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                         const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairOffBar);
    uint64_t* full = bars;                        // [S] even CTA: both CTAs' copies of the stage landed
    uint64_t* empty = bars + kPairStages;         // [S] pair MMA commit -> each CTA's producer
    uint64_t* acc_full = bars + 2 * kPairStages;  // [2] pair MMA commit -> epilogue (both CTAs)
    uint64_t* acc_empty = acc_full + 2;           // [2] even CTA: 256 epilogue threads of the pair -> MMA
    uint64_t* drain = acc_full + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kPairOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kPairOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank_in();
    const bool leader = rank == 0;
    const int64_t pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int kb_per_tile = a.d / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_w);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 2 * kBN);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers are initialised before either touches the other's
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger();
    pdl_wait();  // global memory is shared with the kernels before this one from here on

    if (warp == 0 && a.rows) {
        // ------------------------------------------------------------ TMA producer (both CTAs), rows gathered
        // lane l fetches this CTA's tile rows 4l .. 4l + 3 with one gather4 copy per 64-column step
        int s = 0;
        uint32_t ph = 0;
        int last_ph[kPairStages];
        for (int i = 0; i < kPairStages; ++i) last_ph[i] = -1;
        for (int64_t t = pair; t < a.num_tiles; t += num_pairs) {
            if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
            const int rt = static_cast<int>(t / a.num_col_tiles);
            const int ct = static_cast<int>(t % a.num_col_tiles);
            int g[4];
            gather_rows4(a, static_cast<int64_t>(rt) * 2 * kBM + static_cast<int64_t>(rank) * kBM + lane * 4, g);
            bool ok = true;
            for (int kb = 0; kb < kb_per_tile; ++kb) {
                if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT);
                if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                    ok = false;
                    break;
                }
                uint8_t* sa = smem + s * kPairStage;
                if (leader && lane == 0) mbar_arrive_expect_tx(&full[s], 2 * kPairStage);
                __syncwarp();
                const uint32_t fb = cluster_addr(&full[s], 0);
                tma_gather4_pair(sa + lane * 512, &tmap_x, fb, kb * kBK, g[0], g[1], g[2], g[3], kEvictLast);
                if (lane == 0)
                    tma_load_2d_pair(sa + kPairStageA, &tmap_w, fb, kb * kBK,
                                     ct * kBN + static_cast<int>(rank) * (kBN / 2), kEvictLast);
                last_ph[s] = static_cast<int>(ph);
                if (++s == kPairStages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (!ok) break;
        }
        if (lane == 0 && *abort_flag && leader) {
            volatile int no_abort = 0;
            for (int i = 0; i < kPairStages; ++i)
                if (last_ph[i] >= 0)
                    mbar_wait_cluster(&full[i], static_cast<uint32_t>(last_ph[i]), &no_abort, a.status,
                                      TG_STATUS_PROJECT_TIMEOUT);
        }
    } else if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int last_ph[kPairStages];
            for (int i = 0; i < kPairStages; ++i) last_ph[i] = -1;
            for (int64_t t = pair; t < a.num_tiles && !*abort_flag; t += num_pairs) {
                const int rt = static_cast<int>(t / a.num_col_tiles);
                const int ct = static_cast<int>(t % a.num_col_tiles);
                for (int kb = 0; kb < kb_per_tile; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT)) break;
                    uint8_t* sa = smem + s * kPairStage;
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * kPairStage);
                    const uint32_t fb = cluster_addr(&full[s], 0);
                    tma_load_2d_pair(sa, &tmap_x, fb, kb * kBK, rt * 2 * kBM + static_cast<int>(rank) * kBM,
                                     kEvictLast);
                    tma_load_2d_pair(sa + kPairStageA, &tmap_w, fb, kb * kBK,
                                     ct * kBN + static_cast<int>(rank) * (kBN / 2), kEvictLast);
                    last_ph[s] = static_cast<int>(ph);
                    if (++s == kPairStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            if (*abort_flag && leader) {
                volatile int no_abort = 0;
                for (int i = 0; i < kPairStages; ++i)
                    if (last_ph[i] >= 0)
                        mbar_wait_cluster(&full[i], static_cast<uint32_t>(last_ph[i]), &no_abort, a.status,
                                          TG_STATUS_PROJECT_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, kBN, false);
            int s = 0;
            uint32_t ph = 0;
            int64_t it = 0;
            bool ok = true;
            for (int64_t t = pair; t < a.num_tiles && ok; t += num_pairs, ++it) {
                const int buf = static_cast<int>(it & 1);
                const uint32_t use = static_cast<uint32_t>(it >> 1);
                if (!mbar_wait_cluster(&acc_empty[buf], (use & 1) ^ 1, abort_flag, a.status,
                                       TG_STATUS_PROJECT_TIMEOUT)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
                for (int kb = 0; kb < kb_per_tile; ++kb) {
                    if (!mbar_wait_cluster(&full[s], ph, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * kPairStage);
                    const uint64_t da = smem_desc_sw128(sa, 16, 1024);
                    const uint64_t db = smem_desc_sw128(sa + kPairStageA, 16, 1024);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        mma_ss_pair(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
                    mma_commit_pair_mc(&empty[s], 0x3);
                    if (++s == kPairStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (ok) mma_commit_pair_mc(&acc_full[buf], 0x3);
            }
            if (!ok) {
                mma_commit_pair(drain);
                volatile int no_abort = 0;
                mbar_wait(drain, 0, &no_abort, a.status, TG_STATUS_PROJECT_TIMEOUT);
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue (own 128 rows)
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
        const uint32_t acc_empty_leader[2] = {cluster_addr(&acc_empty[0], 0), cluster_addr(&acc_empty[1], 0)};
        bool v_range = false;
        int64_t it = 0;
        for (int64_t t = pair; t < a.num_tiles; t += num_pairs, ++it) {
            const int rt = static_cast<int>(t / a.num_col_tiles);
            const int ct = static_cast<int>(t % a.num_col_tiles);
            const int buf = static_cast<int>(it & 1);
            const uint32_t par = static_cast<uint32_t>(it >> 1) & 1;
            const bool ok = mbar_wait_cluster(&acc_full[buf], par, abort_flag, a.status, TG_STATUS_PROJECT_TIMEOUT);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int64_t grow = static_cast<int64_t>(rt) * 2 * kBM + static_cast<int64_t>(rank) * kBM + row;
            epilogue_tile(a, tmem_base + lane_off + static_cast<uint32_t>(buf * kBN), grow, ct, v_range);
            tc_fence_before();
            mbar_arrive_cluster(acc_empty_leader[buf]);
        }
        if (v_range && a.v16) atomicOr(a.status, TG_STATUS_V_RANGE);
    }

    tc_fence_before();
    cluster_sync_all();  // neither CTA leaves while the other may still read its barriers or shared memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 2 * kBN);
    }
}

// Whether this device runs the pair kernel (clusters of 2 with its shared memory), once per device.
static bool pair_kernel_available() {
    static std::atomic<int> cache[64];
    const int dev = current_device();
    if (dev >= 0 && cache[dev].load() != 0) return cache[dev].load() == 2;
    static std::atomic<int> smem_set[64];
    bool ok = set_max_dynamic_smem(project_rope_pair_kernel, kPairSmem, smem_set);
    if (ok) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kPairSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        ok = cudaOccupancyMaxActiveClusters(&n, project_rope_pair_kernel, &cfg) == cudaSuccess && n >= 1;
        cudaGetLastError();
    }
    if (dev >= 0) cache[dev].store(ok ? 2 : 1);
    return ok;
}

}  // namespace proj

size_t ws_project_bytes(int64_t K, int32_t d_h) {
    if (K < 0 || (d_h != 64 && d_h != 128)) return 0;
    return kWsHeader;  // the status word
}

}  // namespace tg

using namespace tg;

// x: [K, d] dense rows (rows == null), or h: [n_rows, d] with x[r] = h[rows[r]].
static tg_status project_impl(const tg_bf16* x, int64_t n_rows, const int32_t* rows, int64_t K, int32_t d,
                              int64_t ld_x, const tg_bf16* W, int32_t Hq, int32_t Hkv, int32_t d_h,
                              const int32_t* pos, double base, tg_bf16* qkv, int64_t ld_qkv, uint16_t* v16,
                              void* workspace, size_t workspace_bytes, void* stream) {
    if (K < 0 || d <= 0 || Hq <= 0 || Hkv <= 0 || ld_x < d || !(base > 0.0)) return TG_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return TG_ERR_UNSUPPORTED;
    const int64_t cols = static_cast<int64_t>(Hq + 2 * Hkv) * d_h;
    if ((d % 64) != 0 || (cols % proj::kBN) != 0 || cols > (1 << 20)) return TG_ERR_UNSUPPORTED;
    if (K > 0x7fffffffLL - proj::kBM) return TG_ERR_UNSUPPORTED;
    if (K == 0) return TG_OK;
    if (!x || !W || !pos || !qkv || !workspace) return TG_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W) || !aligned16(qkv) || (v16 && !aligned16(v16)) || !aligned16(workspace) ||
        (ld_x % 8) != 0 || (ld_qkv % 8) != 0 || ld_qkv < cols)
        return TG_ERR_INVALID_ARG;
    if (workspace_bytes < ws_project_bytes(K, d_h)) return TG_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    CUtensorMap mx, mw;
    const uint64_t xd[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(rows ? n_rows : K)};
    const uint64_t xs[1] = {static_cast<uint64_t>(ld_x) * 2};
    const uint32_t xb[2] = {proj::kBK, rows ? 1u : static_cast<uint32_t>(proj::kBM)};  // gather4: one-row boxes
    const uint64_t wd[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(cols)};
    const uint64_t wsd[1] = {static_cast<uint64_t>(d) * 2};
    const uint32_t wb[2] = {proj::kBK, proj::kBN};
    if (!make_tmap_bf16(&mx, x, 2, xd, xs, xb) || !make_tmap_bf16(&mw, W, 2, wd, wsd, wb)) return TG_ERR_CUDA;

    proj::Args a;
    a.K = K;
    a.d = d;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.D = d_h;
    a.num_col_tiles = static_cast<int>(cols / proj::kBN);
    a.num_tiles = ((K + proj::kBM - 1) / proj::kBM) * a.num_col_tiles;
    a.pos = pos;
    a.rows = rows;
    a.n_rows = n_rows;
    for (int t = 0; t < d_h / 2; ++t)
        a.inv_freq[t] = std::pow(base, -2.0 * static_cast<double>(t) / static_cast<double>(d_h));
    a.qkv = reinterpret_cast<__nv_bfloat16*>(qkv);
    a.ld_qkv = ld_qkv;
    a.v16 = reinterpret_cast<__half*>(v16);
    a.status = status_word(workspace);
    if (cta_pairs_enabled().load() && proj::pair_kernel_available()) {
        // 256 x 256 tiles over CTA pairs; W's box is half a tile (128 rows)
        CUtensorMap mw2;
        const uint32_t wb2[2] = {proj::kBK, proj::kBN / 2};
        if (!make_tmap_bf16(&mw2, W, 2, wd, wsd, wb2)) return TG_ERR_CUDA;
        a.num_tiles = ((K + 2 * proj::kBM - 1) / (2 * proj::kBM)) * a.num_col_tiles;
        const int pairs = static_cast<int>(std::min<int64_t>(a.num_tiles, num_sms() / 2));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * pairs);
        cfg.blockDim = dim3(proj::kThreads);
        cfg.dynamicSmemBytes = proj::kPairSmem;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1] = pdl_attr();
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return cudaLaunchKernelEx(&cfg, proj::project_rope_pair_kernel, mx, mw2, a) == cudaSuccess ? TG_OK
                                                                                                  : TG_ERR_CUDA;
    }
    auto kern = proj::project_rope_kernel;
    static std::atomic<int> smem_set[64];
    if (!set_max_dynamic_smem(kern, proj::kSmem, smem_set)) return TG_ERR_CUDA;
    const int grid = static_cast<int>(std::min<int64_t>(a.num_tiles, num_sms()));
    kern<<<grid, proj::kThreads, proj::kSmem, st>>>(mx, mw, a);
    return launch_status();
}

extern "C" tg_status tg_project_rope(const tg_bf16* x, int64_t K, int32_t d, int64_t ld_x, const tg_bf16* W,
                                     int32_t Hq, int32_t Hkv, int32_t d_h, const int32_t* pos, double base,
                                     tg_bf16* qkv, int64_t ld_qkv, uint16_t* v16, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    return project_impl(x, K, nullptr, K, d, ld_x, W, Hq, Hkv, d_h, pos, base, qkv, ld_qkv, v16, workspace,
                        workspace_bytes, stream);
}

extern "C" tg_status tg_project_rope_gather(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h,
                                            const int32_t* rows, int64_t K, const tg_bf16* W, int32_t Hq,
                                            int32_t Hkv, int32_t d_h, const int32_t* pos, double base,
                                            tg_bf16* qkv, int64_t ld_qkv, uint16_t* v16, void* workspace,
                                            size_t workspace_bytes, void* stream) {
    if (N < 0 || N > 0x7fffffffLL) return N < 0 ? TG_ERR_INVALID_ARG : TG_ERR_UNSUPPORTED;
    if (K > 0 && (N == 0 || !rows)) return TG_ERR_INVALID_ARG;
    return project_impl(h, N, rows, K, d, ld_h, W, Hq, Hkv, d_h, pos, base, qkv, ld_qkv, v16, workspace,
                        workspace_bytes, stream);
}
