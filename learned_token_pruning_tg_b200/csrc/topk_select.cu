// topk_select.cu -- top-K over the prunable document span (TokenGate: a top-K
// selector keeps the best-scored tokens and only the document part of the
// prompt is prunable, the question never is; aiproducthub.cn article,
// paragraph 事件详情; chathome.org article, section TokenGate の学習可能な
// トークンプルーニングの仕組み).  Tie rule (lower index first) and ascending
// output order are the specification's; NaN ranks below every number and
// -0 equals +0.
//
// Two launch shapes, one algorithm.  Spans of up to 16 x 1024 x 16 keys (the
// 16k-128k workloads) run in ONE thread-block cluster of 16 CTAs (8 where the
// device does not offer 16), one per SM: the CTAs' histograms are merged
// through distributed shared memory (each CTA sums one slice of the bins over
// the cluster, then every CTA reads the slice totals and the one slice that
// holds the target), and the hardware cluster barrier replaces the global
// memory barrier; nothing is written to global memory but the result, so this
// shape needs no scratch and has no software wait.  Each thread holds a run of
// consecutive keys, so the ordered compaction takes one block scan.
// Longer spans use one cooperative launch, G <= #SM blocks of 1024 threads:
//   * every score is mapped to an order-preserving 32-bit key and kept in
//     registers for the whole kernel (block b owns a contiguous chunk of the
//     span, thread t the elements t, t+1024, ... of it);
//   * three radix passes over 11/11/10-bit digits find the exact key T of the
//     k-th document token: per pass, a shared-memory histogram built with
//     warp-aggregated increments (__match_any_sync groups the lanes that share
//     a digit, so skewed digit distributions do not serialise on one bank),
//     merged into a global histogram, a grid barrier, then every block scans
//     the global histogram redundantly and identically;
//   * a compaction pass writes kept document indices in ascending order:
//     position = #(keys > T before i) + min(#(keys == T before i), r), where r
//     is the number of T-keys to keep; block prefixes come from per-block
//     counts after one more grid barrier, in-block prefixes from ballots.
// The grid barrier is a sense-reversing counter in the workspace that resets
// itself; each wait is bounded and reports TG_STATUS_SELECT_TIMEOUT.
//
// The same kernel is the random-K selector (the pages' budget-matched random
// baseline) when it is given no scores: token i's key is then the top 32 bits
// of the (i + 1)-th output of a SplitMix64 stream started at `seed` (Steele,
// Lea and Flood; the state advances by 0x9E3779B97F4A7C15 and each output is
// the state through the published finalizer), drawn in registers.
#include <mutex>

#include "tg_host.cuh"

namespace tg {

// Token i's random key: the top 32 bits of SplitMix64 output i + 1 from `seed`
// (the state after i + 1 steps is seed + (i + 1) * 0x9E3779B97F4A7C15 mod 2^64).
__device__ __forceinline__ uint32_t random_key(uint64_t seed, int64_t i) {
    uint64_t z = seed + static_cast<uint64_t>(i + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return static_cast<uint32_t>((z ^ (z >> 31)) >> 32);
}


// Time limit of the grid barrier's wait (ns of %globaltimer), per device.
// tg_debug_set_select_wait_limit shrinks it so that tests can make the barrier
// give up (fault injection without a fault); no other wait reads it.
__device__ unsigned long long g_select_wait_limit_ns = kWaitLimitNs;

// Grid-wide barrier.  Returns false (block-uniformly) if the wait timed out.
__device__ __forceinline__ bool grid_sync(SelectScratch* sc, unsigned nblocks, unsigned int* status, int* s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        volatile unsigned int* vgen = &sc->bar_gen;
        const unsigned int g = *vgen;
        __threadfence();
        const unsigned int arrived = atomicAdd(&sc->bar_count, 1u);
        if (arrived == nblocks - 1) {
            atomicExch(&sc->bar_count, 0u);
            __threadfence();
            atomicAdd(&sc->bar_gen, 1u);
        } else {
            const unsigned long long t0 = globaltimer_ns();
            while (*vgen == g) {
                if (globaltimer_ns() - t0 > g_select_wait_limit_ns) {
                    atomicOr(status, TG_STATUS_SELECT_TIMEOUT);
                    ok = 0;
                    break;
                }
                __nanosleep(32);
            }
        }
        __threadfence();
        *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

// Exclusive prefix of v over the 1024 threads of the block, in thread order;
// *total receives the block sum.  s_warp: 32 words of shared memory.
__device__ __forceinline__ unsigned block_excl_scan(unsigned v, unsigned* s_warp, unsigned* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        unsigned w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const unsigned res = (warp ? s_warp[warp - 1] : 0u) + x - v;
    *total = s_warp[31];
    __syncthreads();
    return res;
}

struct SelectArgs {
    const float* scores;   // NULL: random keys from `seed`
    uint64_t seed;
    int64_t N, D0, D1;
    unsigned int kd;   // document tokens kept, 0 < kd < n_doc
    int32_t* out;
    float* s_out;      // when non-null: the kept tokens' scores, in the order of `out`
    SelectScratch* sc;
    unsigned int* status;
    int ept;           // keys per thread actually used (<= EPT)
    int hist_given;    // the first pass's histogram is already in sc->hist[0] (written with the scores)
};

// Token i goes to slot p of the kept list (and its score beside it when asked).
__device__ __forceinline__ void keep_at(const SelectArgs& a, int64_t p, int64_t i) {
    a.out[p] = static_cast<int32_t>(i);
    if (a.s_out) a.s_out[p] = __ldg(a.scores + i);
}

template <int EPT>
__global__ void __launch_bounds__(kSelectThreads, 1) topk_select_kernel(const SelectArgs a) {
    __shared__ unsigned int s_hist[2048];
    __shared__ unsigned int s_warp[32];
    __shared__ unsigned int s_pick[2];
    __shared__ int s_ok;
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t chunk = static_cast<int64_t>(a.ept) * kSelectThreads;
    const int64_t base = a.D0 + static_cast<int64_t>(blockIdx.x) * chunk;
    const int64_t end = min(base + chunk, a.D1);
    const unsigned nblocks = gridDim.x;

    uint32_t key[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        const int64_t i = base + static_cast<int64_t>(j) * kSelectThreads + tid;
        key[j] = (j < a.ept && i < end) ? (a.scores ? radix_key(__ldg(a.scores + i)) : random_key(a.seed, i)) : 0u;
    }

    uint32_t prefix = 0, pmask = 0;
    unsigned int krem = a.kd;  // 1-based rank of the target among keys matching `prefix`
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
        const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
        const int nb = p == 2 ? 1024 : 2048;
        const uint32_t dmask = static_cast<uint32_t>(nb - 1);
        if (!(p == 0 && a.hist_given)) {
        for (int b = tid; b < 2048; b += kSelectThreads) s_hist[b] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            if (j < a.ept) {
                const int64_t i = base + static_cast<int64_t>(j) * kSelectThreads + tid;
                const bool match = i < end && (key[j] & pmask) == prefix;
                const unsigned active = __ballot_sync(0xffffffffu, match);
                if (match) {
                    const uint32_t digit = (key[j] >> shift) & dmask;
                    const unsigned peers = __match_any_sync(active, digit);
                    if (lane == __ffs(peers) - 1) atomicAdd(&s_hist[digit], static_cast<unsigned>(__popc(peers)));
                }
            }
        }
        __syncthreads();
        for (int b = tid; b < nb; b += kSelectThreads) {
            const unsigned c = s_hist[b];
            if (c) atomicAdd(&a.sc->hist[p][b], c);
        }
        if (!grid_sync(a.sc, nblocks, a.status, &s_ok)) return;
        }

        // Locate the bin holding the krem-th largest key: scan bins from the top digit down.
        const int d0 = nb - 1 - 2 * tid, d1 = d0 - 1;
        const unsigned c0 = d0 >= 0 ? __ldcg(&a.sc->hist[p][d0]) : 0u;
        const unsigned c1 = d1 >= 0 ? __ldcg(&a.sc->hist[p][d1]) : 0u;
        unsigned tot;
        const unsigned e = block_excl_scan(c0 + c1, s_warp, &tot);
        if (e < krem && krem <= e + c0) {
            s_pick[0] = static_cast<unsigned>(d0);
            s_pick[1] = e;
        } else if (e + c0 < krem && krem <= e + c0 + c1) {
            s_pick[0] = static_cast<unsigned>(d1);
            s_pick[1] = e + c0;
        }
        __syncthreads();
        prefix |= s_pick[0] << shift;
        pmask |= dmask << shift;
        krem -= s_pick[1];
        __syncthreads();
    }
    const uint32_t T = prefix;

    // Per-block counts of keys above T and equal to T (each < 2^16 per block).
    unsigned cnt = 0;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        const int64_t i = base + static_cast<int64_t>(j) * kSelectThreads + tid;
        if (j < a.ept && i < end) cnt += (key[j] > T ? 1u : 0u) + (key[j] == T ? 0x10000u : 0u);
    }
    unsigned btot;
    block_excl_scan(cnt, s_warp, &btot);
    if (tid == 0) {
        a.sc->blk_gt[blockIdx.x] = btot & 0xffffu;
        a.sc->blk_eq[blockIdx.x] = btot >> 16;
    }
    if (!grid_sync(a.sc, nblocks, a.status, &s_ok)) return;

    if (tid < 32) {
        unsigned g = 0, q = 0;
        for (unsigned b = lane; b < blockIdx.x; b += 32) {
            g += __ldcg(&a.sc->blk_gt[b]);
            q += __ldcg(&a.sc->blk_eq[b]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            q += __shfl_xor_sync(0xffffffffu, q, o);
        }
        if (lane == 0) {
            s_pick[0] = g;
            s_pick[1] = q;
        }
    }
    __syncthreads();
    unsigned run_g = s_pick[0], run_e = s_pick[1];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        if (j < a.ept) {
            const int64_t i = base + static_cast<int64_t>(j) * kSelectThreads + tid;
            const bool valid = i < end;
            const bool fg = valid && key[j] > T;
            const bool fe = valid && key[j] == T;
            unsigned t2;
            const unsigned ex = block_excl_scan((fg ? 1u : 0u) | (fe ? 0x10000u : 0u), s_warp, &t2);
            const unsigned g_before = run_g + (ex & 0xffffu);
            const unsigned e_before = run_e + (ex >> 16);
            if (fg)
                keep_at(a, a.D0 + g_before + min(e_before, krem), i);
            else if (fe && e_before < krem)
                keep_at(a, a.D0 + g_before + e_before, i);
            run_g += t2 & 0xffffu;
            run_e += t2 >> 16;
        }
    }

    // Tokens outside the span are always kept: [0, D0) first, [D1, N) after the kept document tokens.
    const int64_t gstride = static_cast<int64_t>(nblocks) * kSelectThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kSelectThreads + tid; i < a.D0; i += gstride)
        keep_at(a, i, i);
    for (int64_t i = a.D1 + static_cast<int64_t>(blockIdx.x) * kSelectThreads + tid; i < a.N; i += gstride)
        keep_at(a, a.D0 + a.kd + (i - a.D1), i);

    // Every block has read the global histograms; block 0 clears them for the next call.
    if (blockIdx.x == 0)
        for (int b = tid; b < 3 * 2048; b += kSelectThreads) (&a.sc->hist[0][0])[b] = 0u;
}

// ---------------------------------------------------------------- one-cluster shape
// Cluster rank and size, barrier and distributed-shared-memory access.
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// All threads of every CTA of the cluster; shared-memory writes before it are
// visible cluster-wide after it (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_map(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ uint32_t dsmem_ld(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

constexpr int kSelectClusterMax = 16;

// Keys per thread: a run of `a.ept` consecutive span elements (tb, tb + 1, ...).
// Per radix pass: each CTA's histogram of the keys that match the prefix found
// so far; CTA c then sums bins [c sl, (c + 1) sl) over the cluster (sl = bins /
// cluster size) and their total; warp 0 of every CTA walks the slice totals
// from the top digit down to the slice that holds the target, then that
// slice's bins to the target bin.  Every CTA computes the same result.
template <int EPT>
__global__ void __launch_bounds__(kSelectThreads, 1) topk_select_cluster_kernel(const SelectArgs a) {
    __shared__ unsigned int s_hist[2048];
    __shared__ unsigned int s_slice[2048 / 8];   // this CTA's merged slice (at most 2048 / 8 bins)
    __shared__ unsigned int s_tot;               // its total
    __shared__ unsigned int s_cnt[2];            // this CTA's keys above / equal to the threshold
    __shared__ unsigned int s_warp[32];
    __shared__ unsigned int s_pick[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_ctarank(), ncta = cluster_nctarank();
    const int64_t chunk = static_cast<int64_t>(a.ept) * kSelectThreads;
    const int64_t base = a.D0 + static_cast<int64_t>(rank) * chunk;
    const int64_t end = min(base + chunk, a.D1);
    const int64_t tb = base + static_cast<int64_t>(tid) * a.ept;
    // global memory is shared with the kernels before this one from here on
    pdl_trigger();
    pdl_wait();

    uint32_t key[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        const int64_t i = tb + j;
        key[j] = (j < a.ept && i < end) ? (a.scores ? radix_key(__ldg(a.scores + i)) : random_key(a.seed, i)) : 0u;
    }

    uint32_t prefix = 0, pmask = 0;
    unsigned int krem = a.kd;  // 1-based rank of the target among keys matching `prefix`
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
        const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
        const int nb = p == 2 ? 1024 : 2048;
        const uint32_t dmask = static_cast<uint32_t>(nb - 1);
        if (p == 0 && a.hist_given) {
            // the first pass's histogram was built with the scores: every CTA finds the bin from the
            // 2048 global counts (two per thread, from the top digit down)
            const int d0 = nb - 1 - 2 * tid, d1 = d0 - 1;
            const unsigned c0 = __ldcg(&a.sc->hist[0][d0]), c1 = __ldcg(&a.sc->hist[0][d1]);
            unsigned tot;
            const unsigned e = block_excl_scan(c0 + c1, s_warp, &tot);
            if (e < krem && krem <= e + c0) {
                s_pick[0] = static_cast<unsigned>(d0);
                s_pick[1] = e;
            } else if (e + c0 < krem && krem <= e + c0 + c1) {
                s_pick[0] = static_cast<unsigned>(d1);
                s_pick[1] = e + c0;
            }
            __syncthreads();
            prefix |= s_pick[0] << shift;
            pmask |= dmask << shift;
            krem -= s_pick[1];
            __syncthreads();
            continue;
        }
        for (int b = tid; b < nb; b += kSelectThreads) s_hist[b] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            if (j < a.ept) {
                const bool match = tb + j < end && (key[j] & pmask) == prefix;
                const unsigned active = __ballot_sync(0xffffffffu, match);
                if (match) {
                    const uint32_t digit = (key[j] >> shift) & dmask;
                    const unsigned peers = __match_any_sync(active, digit);
                    if (lane == __ffs(peers) - 1) atomicAdd(&s_hist[digit], static_cast<unsigned>(__popc(peers)));
                }
            }
        }
        cluster_barrier();  // every CTA's histogram of this pass is complete

        // this CTA's slice of the bins, summed over the cluster
        const int sl = nb / static_cast<int>(ncta);
        unsigned part = 0;
        if (tid < sl) {
            const int b = static_cast<int>(rank) * sl + tid;
            // every CTA's count of bin b, all loads in flight at once (up to 16 CTAs)
            uint32_t c[kSelectClusterMax];
#pragma unroll
            for (int r = 0; r < kSelectClusterMax; ++r)
                c[r] = static_cast<uint32_t>(r) < ncta ? dsmem_ld(dsmem_map(&s_hist[b], static_cast<uint32_t>(r))) : 0u;
#pragma unroll
            for (int r = 0; r < kSelectClusterMax; ++r) part += c[r];
            s_slice[tid] = part;
        }
        if (warp < 8) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == 0) s_warp[warp] = part;
        }
        __syncthreads();
        if (tid == 0) {
            unsigned t = 0;
            for (int w = 0; w < 8; ++w) t += s_warp[w];
            s_tot = t;
        }
        cluster_barrier();  // every slice and slice total is ready

        if (warp == 0) {
            // slices from the top digit down: lane l takes slice ncta - 1 - l
            const uint32_t sli = ncta - 1 - static_cast<uint32_t>(lane);
            const unsigned t = static_cast<uint32_t>(lane) < ncta ? dsmem_ld(dsmem_map(&s_tot, sli)) : 0u;
            unsigned incl = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned hit = __ballot_sync(0xffffffffu, incl - t < krem && krem <= incl);
            const int L = hit ? __ffs(hit) - 1 : 0;  // a lane always hits: krem <= the keys matching `prefix`
            const uint32_t slice = ncta - 1 - static_cast<uint32_t>(L);
            const unsigned before = __shfl_sync(0xffffffffu, incl - t, L);
            // that slice's bins from the top down: lane l takes bins top - l per .. top - l per - per + 1
            const int per = sl / 32;
            const int top = sl - 1 - lane * per;  // index inside the slice
            unsigned c[8];
            unsigned lsum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = i < per ? dsmem_ld(dsmem_map(&s_slice[top - i], slice)) : 0u;
                lsum += c[i];
            }
            unsigned lincl = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_up_sync(0xffffffffu, lincl, o);
                if (lane >= o) lincl += y;
            }
            const unsigned lex = before + lincl - lsum;
            if (lane == 0) {
                s_pick[0] = slice * static_cast<uint32_t>(sl);  // overwritten below by the lane that holds the target
                s_pick[1] = before;
            }
            __syncwarp();
            if (lex < krem && krem <= lex + lsum) {
                unsigned acc = lex;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i < per && acc < krem && krem <= acc + c[i]) {
                        s_pick[0] = slice * static_cast<uint32_t>(sl) + static_cast<uint32_t>(top - i);
                        s_pick[1] = acc;
                    }
                    acc += c[i];
                }
            }
        }
        __syncthreads();
        prefix |= s_pick[0] << shift;
        pmask |= dmask << shift;
        krem -= s_pick[1];
        __syncthreads();
    }
    const uint32_t T = prefix;

    // counts of keys above T and equal to T: per thread, per CTA (< 2^16 each), per cluster prefix
    unsigned cnt = 0;
#pragma unroll
    for (int j = 0; j < EPT; ++j)
        if (j < a.ept && tb + j < end) cnt += (key[j] > T ? 1u : 0u) + (key[j] == T ? 0x10000u : 0u);
    unsigned btot;
    const unsigned ex = block_excl_scan(cnt, s_warp, &btot);
    if (tid == 0) {
        s_cnt[0] = btot & 0xffffu;
        s_cnt[1] = btot >> 16;
    }
    cluster_barrier();
    if (warp == 0) {
        unsigned g = 0, q = 0;
        if (static_cast<uint32_t>(lane) < rank) {
            g = dsmem_ld(dsmem_map(&s_cnt[0], lane));
            q = dsmem_ld(dsmem_map(&s_cnt[1], lane));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            q += __shfl_xor_sync(0xffffffffu, q, o);
        }
        if (lane == 0) {
            s_pick[0] = g;
            s_pick[1] = q;
        }
    }
    __syncthreads();
    unsigned g_before = s_pick[0] + (ex & 0xffffu), e_before = s_pick[1] + (ex >> 16);
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        if (j < a.ept && tb + j < end) {
            const int32_t i = static_cast<int32_t>(tb + j);
            if (key[j] > T) {
                keep_at(a, a.D0 + g_before + min(e_before, krem), i);
                ++g_before;
            } else if (key[j] == T) {
                if (e_before < krem) keep_at(a, a.D0 + g_before + e_before, i);
                ++e_before;
            }
        }
    }
    // Tokens outside the span are always kept: [0, D0) first, [D1, N) after the kept document tokens.
    const int64_t gstride = static_cast<int64_t>(ncta) * kSelectThreads;
    for (int64_t i = static_cast<int64_t>(rank) * kSelectThreads + tid; i < a.D0; i += gstride)
        keep_at(a, i, i);
    for (int64_t i = a.D1 + static_cast<int64_t>(rank) * kSelectThreads + tid; i < a.N; i += gstride)
        keep_at(a, a.D0 + a.kd + (i - a.D1), i);
    cluster_barrier();  // this CTA's shared memory stays alive until every CTA has read it
    // every CTA read the given first-pass histogram in pass 0: leave it zero for the next gate
    if (a.hist_given && rank == 0)
        for (int b = tid; b < 2048; b += kSelectThreads) a.sc->hist[0][b] = 0u;
}

// K_doc == 0 (only tokens outside the span) or K_doc >= N_doc (every token).
__global__ void select_trivial_kernel(int64_t N, int64_t D0, int64_t D1, int keep_doc, int32_t* out,
                                      const float* scores, float* s_out) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < N; i += stride) {
        int64_t p = -1;
        if (keep_doc || i < D0)
            p = i;
        else if (i >= D1)
            p = D0 + (i - D1);
        if (p >= 0) {
            out[p] = static_cast<int32_t>(i);
            if (s_out) s_out[p] = __ldg(scores + i);
        }
    }
}

template <int EPT>
static cudaError_t launch_select(const SelectArgs& a, int grid, cudaStream_t st) {
    void* args[] = {const_cast<SelectArgs*>(&a)};
    return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(topk_select_kernel<EPT>), dim3(grid),
                                       dim3(kSelectThreads), args, 0, st);
}

// Largest cluster (16, else 8, else 0 = none) this device runs the cluster
// kernel with, queried once per device.
static int select_cluster_size() {
    static std::atomic<int> cache[64];
    const int dev = current_device();
    if (dev >= 0 && cache[dev].load() != 0) return cache[dev].load() - 1;
    int best = 0;
    auto kern = topk_select_cluster_kernel<16>;
    const bool nonportable =
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    for (int cl : {16, 8}) {
        if (cl > 8 && !nonportable) continue;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cl);
        cfg.blockDim = dim3(kSelectThreads);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cl;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 1) {
            best = cl;
            break;
        }
        cudaGetLastError();
    }
    if (dev >= 0) cache[dev].store(best + 1);
    return best;
}

template <int EPT>
static cudaError_t launch_select_cluster(const SelectArgs& a, int cl, cudaStream_t st) {
    auto kern = topk_select_cluster_kernel<EPT>;
    if (cl > 8) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl);
    cfg.blockDim = dim3(kSelectThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr();
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

// The one-cluster shape when the span fits it (keys per thread <= 16);
// returns false when the span is too long or the device offers no cluster.
static bool try_select_cluster(SelectArgs a, int64_t n_doc, cudaStream_t st, cudaError_t* err) {
    const int cl = select_cluster_size();
    if (cl == 0) return false;
    const int64_t per_cta = static_cast<int64_t>(cl) * kSelectThreads;
    const int64_t ept = (n_doc + per_cta - 1) / per_cta;
    if (ept > kSelectMaxEpt) return false;
    a.ept = static_cast<int>(ept < 1 ? 1 : ept);
    if (a.ept <= 1)
        *err = launch_select_cluster<1>(a, cl, st);
    else if (a.ept <= 2)
        *err = launch_select_cluster<2>(a, cl, st);
    else if (a.ept <= 4)
        *err = launch_select_cluster<4>(a, cl, st);
    else if (a.ept <= 8)
        *err = launch_select_cluster<8>(a, cl, st);
    else
        *err = launch_select_cluster<16>(a, cl, st);
    return true;
}

}  // namespace tg

using namespace tg;

// The select with keys from `scores`, or random keys from `seed` when scores is NULL.
static tg_status select_impl(const float* scores, uint64_t seed, int64_t N, int64_t doc_begin, int64_t doc_end,
                             int64_t k_doc, int32_t* kept_idx, void* workspace, size_t workspace_bytes,
                             void* stream, bool hist_given = false, float* s_kept = nullptr) {
    const int64_t K = tg_kept_count(N, doc_begin, doc_end, k_doc);
    if (K < 0) return TG_ERR_INVALID_ARG;
    if (N > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    const int64_t n_doc = doc_end - doc_begin;
    const int64_t kd = k_doc < n_doc ? k_doc : n_doc;
    cudaStream_t st = as_stream(stream);
    if (hist_given && (K == 0 || kd == 0 || kd == n_doc)) {
        // no radix pass reads the gate's histogram: clear it here for the next gate
        if (!workspace || workspace_bytes < tg_workspace_bytes(TG_OP_SELECT, N, 0, 0)) return TG_ERR_INVALID_ARG;
        SelectScratch* sc = reinterpret_cast<SelectScratch*>(static_cast<char*>(workspace) + kWsHeader);
        if (cudaMemsetAsync(&sc->hist[0][0], 0, sizeof(sc->hist[0]), st) != cudaSuccess) return TG_ERR_CUDA;
    }
    if (K == 0) return TG_OK;
    if (!kept_idx || (s_kept && !scores)) return TG_ERR_INVALID_ARG;
    if (kd == 0 || kd == n_doc) {
        const int64_t blocks = std::min<int64_t>((N + 255) / 256, static_cast<int64_t>(num_sms()) * 8);
        select_trivial_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(N, doc_begin, doc_end,
                                                                             kd == n_doc ? 1 : 0, kept_idx,
                                                                             scores, s_kept);
        return launch_status();
    }
    if (!workspace || workspace_bytes < tg_workspace_bytes(TG_OP_SELECT, N, 0, 0)) return TG_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return TG_ERR_INVALID_ARG;

    SelectArgs a;
    a.scores = scores;
    a.seed = seed;
    a.N = N;
    a.D0 = doc_begin;
    a.D1 = doc_end;
    a.kd = static_cast<unsigned int>(kd);
    a.out = kept_idx;
    a.s_out = s_kept;
    a.sc = reinterpret_cast<SelectScratch*>(static_cast<char*>(workspace) + kWsHeader);
    a.status = status_word(workspace);
    a.hist_given = hist_given ? 1 : 0;
    cudaError_t e;
    if (try_select_cluster(a, n_doc, st, &e)) return e == cudaSuccess ? TG_OK : TG_ERR_CUDA;

    const int sms = num_sms();
    const int64_t per_block_min = kSelectThreads;
    int64_t ept = (n_doc + static_cast<int64_t>(sms) * per_block_min - 1) / (static_cast<int64_t>(sms) * per_block_min);
    if (ept < 1) ept = 1;
    if (ept > kSelectMaxEpt) return TG_ERR_UNSUPPORTED;
    const int64_t chunk = ept * kSelectThreads;
    const int grid = static_cast<int>((n_doc + chunk - 1) / chunk);
    if (grid > kSelectMaxBlocks) return TG_ERR_UNSUPPORTED;
    a.ept = static_cast<int>(ept);
    if (ept <= 1)
        e = launch_select<1>(a, grid, st);
    else if (ept <= 2)
        e = launch_select<2>(a, grid, st);
    else if (ept <= 4)
        e = launch_select<4>(a, grid, st);
    else if (ept <= 8)
        e = launch_select<8>(a, grid, st);
    else
        e = launch_select<16>(a, grid, st);
    return e == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

extern "C" tg_status tg_topk_select(const float* scores, int64_t N, int64_t doc_begin, int64_t doc_end,
                                    int64_t k_doc, int32_t* kept_idx, void* workspace, size_t workspace_bytes,
                                    void* stream) {
    if (!scores && tg_kept_count(N, doc_begin, doc_end, k_doc) > 0) return TG_ERR_INVALID_ARG;
    return select_impl(scores, 0, N, doc_begin, doc_end, k_doc, kept_idx, workspace, workspace_bytes, stream);
}

extern "C" tg_status tg_topk_select_after_gate(const float* scores, int64_t N, int64_t doc_begin, int64_t doc_end,
                                               int64_t k_doc, int32_t* kept_idx, void* workspace,
                                               size_t workspace_bytes, void* stream) {
    if (!scores && tg_kept_count(N, doc_begin, doc_end, k_doc) > 0) return TG_ERR_INVALID_ARG;
    return select_impl(scores, 0, N, doc_begin, doc_end, k_doc, kept_idx, workspace, workspace_bytes, stream, true);
}

extern "C" tg_status tg_topk_select_after_gate_kept_scores(const float* scores, int64_t N, int64_t doc_begin,
                                                           int64_t doc_end, int64_t k_doc, int32_t* kept_idx,
                                                           float* s_kept, void* workspace, size_t workspace_bytes,
                                                           void* stream) {
    const int64_t K = tg_kept_count(N, doc_begin, doc_end, k_doc);
    if (K > 0 && (!scores || !s_kept)) return TG_ERR_INVALID_ARG;
    return select_impl(scores, 0, N, doc_begin, doc_end, k_doc, kept_idx, workspace, workspace_bytes, stream, true,
                       s_kept);
}

extern "C" tg_status tg_debug_set_select_wait_limit(uint64_t ns) {
    const unsigned long long v = ns ? static_cast<unsigned long long>(ns) : kWaitLimitNs;
    return cudaMemcpyToSymbol(g_select_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

extern "C" tg_status tg_random_select(int64_t N, int64_t doc_begin, int64_t doc_end, int64_t k_doc, uint64_t seed,
                                      int32_t* kept_idx, void* workspace, size_t workspace_bytes, void* stream) {
    return select_impl(nullptr, seed, N, doc_begin, doc_end, k_doc, kept_idx, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- allocation-free entry point
// Some callers cannot allocate device memory at the point where they select
// tokens: code that runs inside an allocator or memory-pool callback, a serving
// process whose device memory is fully reserved up front and handed out by its
// own pool, or a host environment that only hands the library pointers to
// buffers it owns.  tg_topk_select_noalloc serves them: it needs no workspace
// argument, because its scratch lives in the static device array below, which
// every GPU that loads this library keeps for the lifetime of the process.
namespace tg {
namespace noalloc {

// status word (first 256 bytes) + the select scratch: 34,560 bytes in all.
constexpr size_t kScratchBytes = kWsHeader + ((sizeof(SelectScratch) + 255) / 256) * 256;
static_assert(kScratchBytes == 34560, "the documented size of the static scratch");
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch per device.  In host code the symbol name is only
// a host-side stand-in, so the address has to be queried with the device current.
constexpr int kMaxDevices = 64;
static void* g_addr[kMaxDevices] = {nullptr};
static std::mutex g_mu;

static tg_status scratch_for_current_device(unsigned char** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TG_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return TG_ERR_CUDA;
        }
        g_addr[dev] = p;
    }
    *out = static_cast<unsigned char*>(g_addr[dev]);
    return TG_OK;
}

}  // namespace noalloc
}  // namespace tg

extern "C" tg_status tg_topk_select_noalloc(const float* scores, int64_t N, int64_t doc_begin, int64_t doc_end,
                                            int64_t k_doc, int32_t* kept_idx, void* stream) {
    const int64_t K = tg_kept_count(N, doc_begin, doc_end, k_doc);
    if (K < 0) return TG_ERR_INVALID_ARG;
    if (N > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    if (K == 0) return TG_OK;
    if (!scores || !kept_idx) return TG_ERR_INVALID_ARG;
    const int64_t n_doc = doc_end - doc_begin;
    const int64_t kd = k_doc < n_doc ? k_doc : n_doc;
    cudaStream_t st = as_stream(stream);
    if (kd == 0 || kd == n_doc) {
        const int64_t blocks = std::min<int64_t>((N + 255) / 256, static_cast<int64_t>(num_sms()) * 8);
        select_trivial_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(N, doc_begin, doc_end,
                                                                             kd == n_doc ? 1 : 0, kept_idx, nullptr, nullptr);
        return launch_status();
    }
    // the same launch shape as tg_topk_select; spans beyond its largest grid are rejected
    const int sms = num_sms();
    int64_t ept = (n_doc + static_cast<int64_t>(sms) * kSelectThreads - 1) / (static_cast<int64_t>(sms) * kSelectThreads);
    if (ept < 1) ept = 1;
    if (ept > kSelectMaxEpt) return TG_ERR_UNSUPPORTED;
    const int64_t chunk = ept * kSelectThreads;
    const int grid = static_cast<int>((n_doc + chunk - 1) / chunk);
    if (grid > kSelectMaxBlocks) return TG_ERR_UNSUPPORTED;

    unsigned char* scratch = nullptr;
    if (noalloc::scratch_for_current_device(&scratch) != TG_OK) return TG_ERR_CUDA;
    // The array keeps whatever the previous call left; the barrier counters, the
    // histograms and the status word must start at zero, so clear them first.
    if (cudaMemsetAsync(scratch, 0, noalloc::kScratchBytes, st) != cudaSuccess) return TG_ERR_CUDA;

    SelectArgs a;
    a.scores = scores;
    a.seed = 0;
    a.N = N;
    a.D0 = doc_begin;
    a.D1 = doc_end;
    a.kd = static_cast<unsigned int>(kd);
    a.out = kept_idx;
    a.s_out = nullptr;
    a.sc = reinterpret_cast<SelectScratch*>(scratch + kWsHeader);
    a.status = reinterpret_cast<unsigned int*>(scratch);
    a.ept = static_cast<int>(ept);
    a.hist_given = 0;
    cudaError_t e;
    if (ept <= 1)
        e = launch_select<1>(a, grid, st);
    else if (ept <= 2)
        e = launch_select<2>(a, grid, st);
    else if (ept <= 4)
        e = launch_select<4>(a, grid, st);
    else if (ept <= 8)
        e = launch_select<8>(a, grid, st);
    else
        e = launch_select<16>(a, grid, st);
    return e == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

extern "C" tg_status tg_topk_select_noalloc_status(uint32_t* status_word_out, void* stream) {
    unsigned char* scratch = nullptr;
    if (noalloc::scratch_for_current_device(&scratch) != TG_OK) return TG_ERR_CUDA;
    uint32_t w = 0;
    cudaStream_t st = as_stream(stream);
    if (cudaMemcpyAsync(&w, scratch, sizeof(w), cudaMemcpyDeviceToHost, st) != cudaSuccess) return TG_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return TG_ERR_CUDA;
    if (status_word_out) *status_word_out = w;
    return (w & TG_STATUS_TIMEOUT_BITS) ? TG_ERR_TIMEOUT : TG_OK;
}
