// gate_score.cu -- the gate MLP that scores every token's post-attention
// residual at the gate layer (TokenGate: a small MLP gives each token a score,
// aiproducthub.cn article, paragraph 事件详情; chathome.org article, section
// TokenGate の学習可能なトークンプルーニングの仕組み).  Shape from the
// specification: RMSNorm -> Linear(d -> d_g) -> SiLU -> Linear(d_g -> 1).
//
//   s_i = sum_j SiLU(r_i * (h_i . W_j) + b1_j) * w2_j + b2,
//   r_i = (mean_c h_ic^2 + eps)^(-1/2)
//
// The RMS factor is a per-row scale, so it commutes with the GEMM: the tensor
// cores multiply the raw bf16 rows of h with W (no rounding of normalised
// activations) and r_i is applied in the epilogue.  The pass over h that the
// GEMM makes anyway also feeds the row sums of squares, so h is read from HBM
// exactly once.
//
// Kernel (persistent, one CTA per SM, 12 warps):
//   warp 0      TMA producer: 128x64 tiles of h (evict-first) and d_g x 64
//               tiles of W (evict-last, L2-resident) into a STAGES-deep ring
//   warp 1      allocates TMEM and issues tcgen05.mma (M=128, N=d_g, K=16)
//               into one of two fp32 accumulators (2 x d_g TMEM columns)
//   warps 4-7   epilogue: tcgen05.ld of the accumulator row, r_i, +b1, SiLU,
//               dot with w2, +b2, one fp32 score per row
//   warps 8-11  sum of squares of each row straight from the swizzled smem
//               tiles (one thread per row), handed to the epilogue
// The accumulators are double-buffered, so the epilogue of tile t overlaps the
// main loop of tile t+1.  Every wait is bounded (TG_STATUS_GATE_TIMEOUT).
// For d_g = 256 the same roles run on CTA pairs (gate_score_pair_kernel below),
// which halves the W bytes each SM moves per stage.
#include "tg_host.cuh"

namespace tg {
namespace gate {

constexpr int kBM = 128;       // rows per tile
constexpr int kBK = 64;        // K elements per stage (one 128-byte swizzle row)
constexpr int kThreads = 384;  // 12 warps
constexpr int kHistBins = 2048;  // bins of the select's first radix pass (top 11 bits of the key)

template <int DG>
struct Cfg {
    static constexpr int kStageA = kBM * kBK * 2;
    static constexpr int kStageB = DG * kBK * 2;
    static constexpr int kStage = kStageA + kStageB;
    static constexpr int kStages = (DG == 256) ? 4 : (DG == 128 ? 6 : 8);
    static constexpr int kTmemCols = (2 * DG < 32) ? 32 : 2 * DG;
    // shared memory: stages | ss[2][128] | w2[DG] | b1[DG] | barriers | tmem slot, abort flag
    static constexpr int kOffSS = kStages * kStage;
    static constexpr int kOffW2 = kOffSS + 2 * kBM * 4;
    static constexpr int kOffB1 = kOffW2 + DG * 4;
    static constexpr int kOffBar = kOffB1 + DG * 4;
    static constexpr int kNumBars = 2 * kStages + 7;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kOffHist = kOffMisc + 16;
    static constexpr int kSmem = kOffHist + kHistBins * 4 + 1024;  // + alignment slack
    static_assert(kStage % 1024 == 0 && kOffBar % 8 == 0 && kSmem <= 232448, "gate shared-memory layout");
};

struct Args {
    int64_t N;
    int d;
    float eps;
    const float* b1;
    const float* w2;
    float b2;
    float* scores;
    unsigned int* status;
    // when non-null: histogram of the top 11 bits of the radix keys of the scores of rows in [D0, D1)
    // (the select's first pass), added into these 2048 global counters
    unsigned int* hist0;
    int64_t D0, D1;
};


// The select's first-pass histogram of one warp's 32 scores: rows in the document span count; lanes
// that share a digit are folded into one shared-memory increment.
__device__ __forceinline__ void hist0_add(unsigned int* s_hist, const Args& a, int64_t grow, float score) {
    const bool in = grow < a.N && grow >= a.D0 && grow < a.D1;
    const unsigned active = __ballot_sync(0xffffffffu, in);
    if (in) {
        const uint32_t digit = radix_key(score) >> kSelectDigit0Shift;
        const unsigned peers = __match_any_sync(active, digit);
        if ((threadIdx.x & 31) == static_cast<unsigned>(__ffs(peers) - 1))
            atomicAdd(&s_hist[digit], static_cast<unsigned>(__popc(peers)));
    }
}

// Adds a CTA's histogram into the global one (nonzero bins only).
__device__ __forceinline__ void hist0_flush(const unsigned int* s_hist, unsigned int* hist0) {
    for (int b = threadIdx.x; b < kHistBins; b += blockDim.x) {
        const unsigned c = s_hist[b];
        if (c) atomicAdd(&hist0[b], c);
    }
}

template <int DG>
__global__ void __launch_bounds__(kThreads, 1)
gate_score_kernel(const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_w,
                  const Args a) {
    using C = Cfg<DG>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* ss_s = reinterpret_cast<float*>(smem + C::kOffSS);
    float* w2_s = reinterpret_cast<float*>(smem + C::kOffW2);
    float* b1_s = reinterpret_cast<float*>(smem + C::kOffB1);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;                      // [kStages]  TMA -> MMA, sum-of-squares
    uint64_t* empty = bars + C::kStages;        // [kStages]  MMA commit + 128 sum-of-squares threads
    uint64_t* acc_full = bars + 2 * C::kStages; // [2]        MMA commit -> epilogue
    uint64_t* acc_empty = acc_full + 2;         // [2]        128 epilogue threads -> MMA, sum-of-squares
    uint64_t* ss_full = acc_full + 4;           // [2]        128 sum-of-squares threads -> epilogue
    uint64_t* drain = acc_full + 6;             // [1]        MMA completion on the abort path
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    unsigned int* s_hist = reinterpret_cast<unsigned int*>(smem + C::kOffHist);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t num_tiles = (a.N + kBM - 1) / kBM;
    if (a.hist0)
        for (int bb = threadIdx.x; bb < kHistBins; bb += kThreads) s_hist[bb] = 0u;
    const int kb_per_tile = a.d / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + 128);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
            mbar_init(&ss_full[b], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_h);
        tma_prefetch_desc(&tmap_w);
    }
    for (int j = threadIdx.x; j < DG; j += kThreads) {
        w2_s[j] = a.w2[j];
        b1_s[j] = a.b1 ? a.b1[j] : 0.0f;
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int last_ph[C::kStages];  // parity of the last phase loaded into each stage, -1 if none
            for (int i = 0; i < C::kStages; ++i) last_ph[i] = -1;
            for (int64_t t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
                for (int kb = 0; kb < kb_per_tile; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) break;
                    uint8_t* sa = smem + s * C::kStage;
                    mbar_arrive_expect_tx(&full[s], C::kStage);
                    tma_load_2d(sa, &tmap_h, &full[s], kb * kBK, static_cast<int>(t * kBM), kEvictFirst);
                    tma_load_2d(sa + C::kStageA, &tmap_w, &full[s], kb * kBK, 0, kEvictLast);
                    last_ph[s] = static_cast<int>(ph);
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            if (*abort_flag) {
                // Let every issued copy land before the CTA's shared memory is released.
                volatile int no_abort = 0;
                for (int i = 0; i < C::kStages; ++i)
                    if (last_ph[i] >= 0)
                        mbar_wait(&full[i], static_cast<uint32_t>(last_ph[i]), &no_abort, a.status,
                                  TG_STATUS_GATE_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, DG, false);
            int s = 0;
            uint32_t ph = 0;
            int64_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++it) {
                const int buf = static_cast<int>(it & 1);
                const uint32_t use = static_cast<uint32_t>(it >> 1);
                if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * DG);
                for (int kb = 0; kb < kb_per_tile; ++kb) {
                    if (!mbar_wait(&full[s], ph, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::kStage);
                    const uint64_t da = smem_desc_sw128(sa, 16, 1024);
                    const uint64_t db = smem_desc_sw128(sa + C::kStageA, 16, 1024);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)  // +32 bytes per K=16 step inside the swizzle row
                        mma_ss(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
                    mma_commit(&empty[s]);
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (ok) mma_commit(&acc_full[buf]);
            }
            if (!ok) {
                // Drain: wait (bounded) for the MMAs already issued before TMEM is freed.
                mma_commit(drain);
                volatile int no_abort = 0;
                mbar_wait(drain, 0, &no_abort, a.status, TG_STATUS_GATE_TIMEOUT);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;              // TMEM lane quarter of this warp
        const int row = q * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const float inv_d = 1.0f / static_cast<float>(a.d);
        int64_t it = 0;
        for (int64_t t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
            const int buf = static_cast<int>(it & 1);
            const uint32_t par = static_cast<uint32_t>(it >> 1) & 1;
            // warp-uniform outcome: tcgen05.ld below is warp-collective
            bool ok = mbar_wait(&acc_full[buf], par, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT) &&
                      mbar_wait(&ss_full[buf], par, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const float r = rsqrtf(ss_s[buf * kBM + row] * inv_d + a.eps);
            float acc = 0.0f;
            const uint32_t taddr = tmem_base + lane_off + static_cast<uint32_t>(buf * DG);
#pragma unroll 1
            for (int c0 = 0; c0 < DG; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float u = fmaf(r, __uint_as_float(v[j]), b1_s[c0 + j]);
                    const float e = __expf(fminf(-u, 80.0f));
                    acc = fmaf(__fdividef(u, 1.0f + e), w2_s[c0 + j], acc);
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[buf]);
            const int64_t grow = t * kBM + row;
            if (grow < a.N) a.scores[grow] = acc + a.b2;
            if (a.hist0) hist0_add(s_hist, a, grow, acc + a.b2);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ row sums of squares
        const int row = (warp - 8) * 32 + lane;
        const int sw = row & 7;  // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
        int s = 0;
        uint32_t ph = 0;
        int64_t it = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++it) {
            float ss0 = 0.0f, ss1 = 0.0f;
            for (int kb = 0; kb < kb_per_tile; ++kb) {
                if (!mbar_wait(&full[s], ph, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) {
                    ok = false;
                    break;
                }
                const uint8_t* rp = smem + s * C::kStage + row * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 x = *reinterpret_cast<const uint4*>(rp + ((c ^ sw) << 4));
                    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(w[e] << 16);
                        const float hi = __uint_as_float(w[e] & 0xffff0000u);
                        ss0 = fmaf(lo, lo, ss0);
                        ss1 = fmaf(hi, hi, ss1);
                    }
                }
                // These generic-proxy reads must be ordered before the TMA (async proxy) that
                // refills this stage once it is released; the mbarrier alone does not order them.
                fence_proxy_async_smem();
                mbar_arrive(&empty[s]);
                if (++s == C::kStages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (!ok) break;
            const int buf = static_cast<int>(it & 1);
            const uint32_t use = static_cast<uint32_t>(it >> 1);
            if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) break;
            ss_s[buf * kBM + row] = ss0 + ss1;
            mbar_arrive(&ss_full[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (a.hist0) hist0_flush(s_hist, a.hist0);
}

// ---------------------------------------------------------------- CTA-pair kernel (d_g = 256)
// The same gate on 256-row tiles shared by the two CTAs of a cluster: one
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16) per 16 columns of h, with
// each CTA holding its own 128 rows of h and HALF of W (128 of its 256 rows) in
// its own shared memory.  Per 64-column stage a CTA then moves 16 KB of W
// instead of 32 KB, and its shared memory supplies (and receives) half as many
// W bytes -- the single-CTA kernel is bound by shared-memory traffic, W's share
// of which this halves.  No multicast: every TMA copy lands in the CTA that
// issues it; only completion is counted on the even CTA's barrier.
//   both CTAs   warp 0 TMA (own rows of h, own half of W), warps 4-7 epilogue
//               of own rows, warps 8-11 own rows' sums of squares, warp 1 the
//               pair's TMEM allocation
//   even CTA    warp 1 lane 0 issues the pair's MMAs; their completion is
//               committed to both CTAs' barriers
constexpr int kPairBN = 128;  // rows of W per CTA
struct PairCfg {
    static constexpr int kDG = 256;
    static constexpr int kStageA = kBM * kBK * 2;       // 16 KB
    static constexpr int kStageB = kPairBN * kBK * 2;   // 16 KB
    static constexpr int kStage = kStageA + kStageB;
    static constexpr int kStages = 6;
    static constexpr int kTmemCols = 2 * kDG;           // two 256-column accumulators
    static constexpr int kOffSS = kStages * kStage;
    static constexpr int kOffW2 = kOffSS + 2 * kBM * 4;
    static constexpr int kOffB1 = kOffW2 + kDG * 4;
    static constexpr int kOffBar = kOffB1 + kDG * 4;
    // full, empty, a_full per stage; acc_full, acc_empty, ss_full, ss_empty per buffer; drain
    static constexpr int kNumBars = 3 * kStages + 9;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kOffHist = kOffMisc + 16;
    static constexpr int kSmem = kOffHist + kHistBins * 4 + 1024;
};
static_assert(PairCfg::kStageA % 1024 == 0 && PairCfg::kStage % 1024 == 0 && PairCfg::kOffBar % 8 == 0 &&
                  PairCfg::kSmem <= 232448,
              "gate pair kernel shared-memory layout");

__global__ void __launch_bounds__(kThreads, 1)
gate_score_pair_kernel(const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_w,
                       const Args a) {
    using C = PairCfg;
    constexpr int DG = C::kDG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* ss_s = reinterpret_cast<float*>(smem + C::kOffSS);
    float* w2_s = reinterpret_cast<float*>(smem + C::kOffW2);
    float* b1_s = reinterpret_cast<float*>(smem + C::kOffB1);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;                      // [S] even CTA: both CTAs' copies of the stage landed
    uint64_t* empty = bars + C::kStages;        // [S] pair MMA commit + 128 sum-of-squares threads
    uint64_t* a_full = bars + 2 * C::kStages;   // [S] pair MMA commit: the stage was consumed (odd CTA's row sums)
    uint64_t* acc_full = bars + 3 * C::kStages; // [2] pair MMA commit -> epilogue (both CTAs)
    uint64_t* acc_empty = acc_full + 2;         // [2] even CTA: 256 epilogue threads of the pair -> MMA
    uint64_t* ss_full = acc_full + 4;           // [2] 128 sum-of-squares threads -> epilogue
    uint64_t* ss_empty = acc_full + 6;          // [2] 128 epilogue threads -> sum-of-squares
    uint64_t* drain = acc_full + 8;             // [1] MMA completion on the abort path
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    unsigned int* s_hist = reinterpret_cast<unsigned int*>(smem + C::kOffHist);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank_in();   // 0: issues the MMAs
    if (a.hist0)
        for (int bb = threadIdx.x; bb < kHistBins; bb += kThreads) s_hist[bb] = 0u;
    const bool leader = rank == 0;
    const int64_t pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int64_t num_tiles = (a.N + 2 * kBM - 1) / (2 * kBM);  // 256-row tiles of the pair
    const int kb_per_tile = a.d / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + 128);
            mbar_init(&a_full[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * 128);
            mbar_init(&ss_full[b], 128);
            mbar_init(&ss_empty[b], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_h);
        tma_prefetch_desc(&tmap_w);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers are initialised before either touches the other's
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // set-up done: from here on global memory is shared with the kernels before this one
    pdl_trigger();
    pdl_wait();
    for (int j = threadIdx.x; j < DG; j += kThreads) {
        w2_s[j] = a.w2[j];
        b1_s[j] = a.b1 ? a.b1[j] : 0.0f;
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int last_ph[C::kStages];
            for (int i = 0; i < C::kStages; ++i) last_ph[i] = -1;
            for (int64_t t = pair; t < num_tiles && !*abort_flag; t += num_pairs) {
                const int row0 = static_cast<int>(t * 2 * kBM + rank * kBM);
                for (int kb = 0; kb < kb_per_tile; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) break;
                    uint8_t* sa = smem + s * C::kStage;
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::kStage);
                    const uint32_t fb = cluster_addr(&full[s], 0);
                    tma_load_2d_pair(sa, &tmap_h, fb, kb * kBK, row0, kEvictFirst);
                    tma_load_2d_pair(sa + C::kStageA, &tmap_w, fb, kb * kBK, static_cast<int>(rank) * kPairBN,
                                     kEvictLast);
                    last_ph[s] = static_cast<int>(ph);
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            if (*abort_flag && leader) {
                // Let every issued copy land before the CTA's shared memory is released.
                volatile int no_abort = 0;
                for (int i = 0; i < C::kStages; ++i)
                    if (last_ph[i] >= 0)
                        mbar_wait_cluster(&full[i], static_cast<uint32_t>(last_ph[i]), &no_abort, a.status,
                                          TG_STATUS_GATE_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, DG, false);
            int s = 0;
            uint32_t ph = 0;
            int64_t it = 0;
            bool ok = true;
            for (int64_t t = pair; t < num_tiles && ok; t += num_pairs, ++it) {
                const int buf = static_cast<int>(it & 1);
                const uint32_t use = static_cast<uint32_t>(it >> 1);
                if (!mbar_wait_cluster(&acc_empty[buf], (use & 1) ^ 1, abort_flag, a.status,
                                       TG_STATUS_GATE_TIMEOUT)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * DG);
                for (int kb = 0; kb < kb_per_tile; ++kb) {
                    if (!mbar_wait_cluster(&full[s], ph, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::kStage);
                    const uint64_t da = smem_desc_sw128(sa, 16, 1024);
                    const uint64_t db = smem_desc_sw128(sa + C::kStageA, 16, 1024);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        mma_ss_pair(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
                    // the stage's MMAs done: the odd CTA's rows of h had landed, its row sums may read
                    // them (they are released only after that); then the stage's MMA share of `empty`
                    mma_commit_pair_mc(&a_full[s], 0x3);
                    mma_commit_pair_mc(&empty[s], 0x3);
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (ok) mma_commit_pair_mc(&acc_full[buf], 0x3);
            }
            if (!ok) {
                mma_commit_pair(drain);
                volatile int no_abort = 0;
                mbar_wait(drain, 0, &no_abort, a.status, TG_STATUS_GATE_TIMEOUT);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ epilogue (own rows)
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const float inv_d = 1.0f / static_cast<float>(a.d);
        const uint32_t acc_empty_leader[2] = {cluster_addr(&acc_empty[0], 0), cluster_addr(&acc_empty[1], 0)};
        int64_t it = 0;
        for (int64_t t = pair; t < num_tiles; t += num_pairs, ++it) {
            const int buf = static_cast<int>(it & 1);
            const uint32_t par = static_cast<uint32_t>(it >> 1) & 1;
            bool ok = mbar_wait_cluster(&acc_full[buf], par, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT) &&
                      mbar_wait(&ss_full[buf], par, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const float r = rsqrtf(ss_s[buf * kBM + row] * inv_d + a.eps);
            mbar_arrive(&ss_empty[buf]);
            float acc = 0.0f;
            const uint32_t taddr = tmem_base + lane_off + static_cast<uint32_t>(buf * DG);
#pragma unroll 1
            for (int c0 = 0; c0 < DG; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float u = fmaf(r, __uint_as_float(v[j]), b1_s[c0 + j]);
                    const float e = __expf(fminf(-u, 80.0f));
                    acc = fmaf(__fdividef(u, 1.0f + e), w2_s[c0 + j], acc);
                }
            }
            tc_fence_before();
            mbar_arrive_cluster(acc_empty_leader[buf]);
            const int64_t grow = t * 2 * kBM + static_cast<int64_t>(rank) * kBM + row;
            if (grow < a.N) a.scores[grow] = acc + a.b2;
            if (a.hist0) hist0_add(s_hist, a, grow, acc + a.b2);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ row sums of squares (own rows)
        const int row = (warp - 8) * 32 + lane;
        const int sw = row & 7;
        uint64_t* landed = leader ? full : a_full;
        int s = 0;
        uint32_t ph = 0;
        int64_t it = 0;
        bool ok = true;
        for (int64_t t = pair; t < num_tiles && ok; t += num_pairs, ++it) {
            float ss0 = 0.0f, ss1 = 0.0f;
            for (int kb = 0; kb < kb_per_tile; ++kb) {
                if (!mbar_wait_cluster(&landed[s], ph, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) {
                    ok = false;
                    break;
                }
                const uint8_t* rp = smem + s * C::kStage + row * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 x = *reinterpret_cast<const uint4*>(rp + ((c ^ sw) << 4));
                    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(w[e] << 16);
                        const float hi = __uint_as_float(w[e] & 0xffff0000u);
                        ss0 = fmaf(lo, lo, ss0);
                        ss1 = fmaf(hi, hi, ss1);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&empty[s]);
                if (++s == C::kStages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (!ok) break;
            const int buf = static_cast<int>(it & 1);
            const uint32_t use = static_cast<uint32_t>(it >> 1);
            if (!mbar_wait(&ss_empty[buf], (use & 1) ^ 1, abort_flag, a.status, TG_STATUS_GATE_TIMEOUT)) break;
            ss_s[buf * kBM + row] = ss0 + ss1;
            mbar_arrive(&ss_full[buf]);
        }
    }

    tc_fence_before();
    cluster_sync_all();  // neither CTA leaves while the other may still read its barriers or shared memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
    if (a.hist0) hist0_flush(s_hist, a.hist0);
}

// W'_jc = bf16(gamma_c * W1_jc): the RMSNorm weight folded into the first layer.
__global__ void fold_gamma_kernel(const __nv_bfloat16* __restrict__ W1, const __nv_bfloat16* __restrict__ gamma,
                                  __nv_bfloat16* __restrict__ out, int d, int64_t total) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride)
        out[i] = __float2bfloat16_rn(__bfloat162float(W1[i]) * __bfloat162float(gamma[i % d]));
}

// Whether this device runs the pair kernel (clusters of 2 with its shared memory), queried once per device.
static bool pair_kernel_available() {
    static std::atomic<int> cache[64];
    const int dev = current_device();
    if (dev >= 0 && cache[dev].load() != 0) return cache[dev].load() == 2;
    static std::atomic<int> smem_set[64];
    bool ok = set_max_dynamic_smem(gate_score_pair_kernel, PairCfg::kSmem, smem_set);
    if (ok) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = PairCfg::kSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        ok = cudaOccupancyMaxActiveClusters(&n, gate_score_pair_kernel, &cfg) == cudaSuccess && n >= 1;
        cudaGetLastError();
    }
    if (dev >= 0) cache[dev].store(ok ? 2 : 1);
    return ok;
}

static tg_status launch_pair(const CUtensorMap& mh, const CUtensorMap& mw, const Args& a, cudaStream_t st) {
    const int64_t pair_tiles = (a.N + 2 * kBM - 1) / (2 * kBM);
    const int pairs = static_cast<int>(std::min<int64_t>(pair_tiles, num_sms() / 2));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = PairCfg::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, gate_score_pair_kernel, mh, mw, a) == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

template <int DG>
static tg_status launch(const CUtensorMap& mh, const CUtensorMap& mw, const Args& a, int64_t num_tiles,
                        cudaStream_t st) {
    using C = Cfg<DG>;
    auto kern = gate_score_kernel<DG>;
    static std::atomic<int> smem_set[64];  // zero before first use (static storage)
    if (!set_max_dynamic_smem(kern, C::kSmem, smem_set))
        return TG_ERR_CUDA;
    const int grid = static_cast<int>(std::min<int64_t>(num_tiles, num_sms()));
    kern<<<grid, kThreads, C::kSmem, st>>>(mh, mw, a);
    return launch_status();
}

}  // namespace gate
}  // namespace tg

using namespace tg;

static tg_status gate_impl(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h, const tg_bf16* rms_weight, float eps,
                           const tg_bf16* W1, const float* b1, const float* w2, float b2, int32_t d_g, float* scores,
                           void* workspace, size_t workspace_bytes, unsigned int* hist0, int64_t D0, int64_t D1,
                           void* stream) {
    if (N < 0 || d <= 0 || d_g <= 0 || ld_h < d || !(eps >= 0.0f)) return TG_ERR_INVALID_ARG;
    if ((d % 64) != 0 || d > 16384) return TG_ERR_UNSUPPORTED;
    if (d_g != 64 && d_g != 128 && d_g != 256) return TG_ERR_UNSUPPORTED;
    if (N > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    if (N == 0) return TG_OK;
    if (!h || !W1 || !w2 || !scores || !workspace) return TG_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(W1) || !aligned16(workspace) || (ld_h % 8) != 0) return TG_ERR_INVALID_ARG;
    if (workspace_bytes < tg_workspace_bytes(TG_OP_GATE, N, d, d_g)) return TG_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);

    const void* wsrc = W1;
    if (rms_weight) {
        __nv_bfloat16* folded = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(workspace) + ws_gate_offset());
        const int64_t total = static_cast<int64_t>(d) * d_g;
        gate::fold_gamma_kernel<<<static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, 1184)), 256, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(W1), reinterpret_cast<const __nv_bfloat16*>(rms_weight), folded, d,
            total);
        if (launch_status() != TG_OK) return TG_ERR_CUDA;
        wsrc = folded;
    }

    CUtensorMap mh, mw;
    const uint64_t hd[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(N)};
    const uint64_t hs[1] = {static_cast<uint64_t>(ld_h) * 2};
    const uint32_t hb[2] = {gate::kBK, gate::kBM};
    const uint64_t wd[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(d_g)};
    const uint64_t wsd[1] = {static_cast<uint64_t>(d) * 2};
    const uint32_t wb[2] = {gate::kBK, static_cast<uint32_t>(d_g)};
    if (!make_tmap_bf16(&mh, h, 2, hd, hs, hb) || !make_tmap_bf16(&mw, wsrc, 2, wd, wsd, wb)) return TG_ERR_CUDA;

    gate::Args a;
    a.N = N;
    a.d = d;
    a.eps = eps;
    a.b1 = b1;
    a.w2 = w2;
    a.b2 = b2;
    a.scores = scores;
    a.status = status_word(workspace);
    a.hist0 = hist0;
    a.D0 = D0;
    a.D1 = D1;
    const int64_t num_tiles = (N + gate::kBM - 1) / gate::kBM;
    if (d_g == 256 && cta_pairs_enabled().load() && gate::pair_kernel_available()) {
        // W's half tile: 128 rows per CTA
        CUtensorMap mw2;
        const uint32_t wb2[2] = {gate::kBK, static_cast<uint32_t>(gate::kPairBN)};
        if (!make_tmap_bf16(&mw2, wsrc, 2, wd, wsd, wb2)) return TG_ERR_CUDA;
        return gate::launch_pair(mh, mw2, a, st);
    }
    switch (d_g) {
        case 64: return gate::launch<64>(mh, mw, a, num_tiles, st);
        case 128: return gate::launch<128>(mh, mw, a, num_tiles, st);
        default: return gate::launch<256>(mh, mw, a, num_tiles, st);
    }
}

extern "C" tg_status tg_gate_score(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h, const tg_bf16* rms_weight,
                                   float eps, const tg_bf16* W1, const float* b1, const float* w2, float b2,
                                   int32_t d_g, float* scores, void* workspace, size_t workspace_bytes,
                                   void* stream) {
    return gate_impl(h, N, d, ld_h, rms_weight, eps, W1, b1, w2, b2, d_g, scores, workspace, workspace_bytes, nullptr,
                     0, 0, stream);
}

extern "C" tg_status tg_gate_score_for_select(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h,
                                              const tg_bf16* rms_weight, float eps, const tg_bf16* W1, const float* b1,
                                              const float* w2, float b2, int32_t d_g, float* scores,
                                              int64_t doc_begin, int64_t doc_end, void* workspace,
                                              size_t workspace_bytes, void* stream) {
    if (doc_begin < 0 || doc_end < doc_begin || doc_end > N) return TG_ERR_INVALID_ARG;
    if (!workspace) return TG_ERR_INVALID_ARG;
    SelectScratch* sc = reinterpret_cast<SelectScratch*>(static_cast<char*>(workspace) + kWsHeader);
    return gate_impl(h, N, d, ld_h, rms_weight, eps, W1, b1, w2, b2, d_g, scores, workspace, workspace_bytes,
                     &sc->hist[0][0], doc_begin, doc_end, stream);
}
