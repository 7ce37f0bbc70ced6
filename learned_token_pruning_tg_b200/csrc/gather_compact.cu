// gather_compact.cu -- compaction of the kept rows (TokenGate: the layers above
// the gate process only the K kept tokens and write no KV entries for the
// pruned ones; chathome.org article, section TokenGate の学習可能なトークン
// プルーニングの仕組み).  The kept rows, their original positions (which RoPE
// needs) and their gate scores are copied bit-exactly.
//
// Design: HBM-bound row copy by the bulk-copy engine.  One warp per block, one
// kept row per lane: the lane issues one bulk copy of its row from h into its
// slot of shared memory (4 KB at d = 2048), waits for it on its own mbarrier,
// and issues one bulk copy from the slot to h_out; 32 rows per SM are in flight
// at once, and the whole 128k workload's kept set (4,608 rows) is one wave.
// Rows wider than a slot allows use a plain copy (one warp per row, 16-byte
// vectors, every load of a row issued before its stores).
// An index outside [0, N) is not read: its output row is zero-filled, its
// position set to -1 and its score to NaN (the caller's check: any pos_out < 0).
#include "tg_host.cuh"

namespace tg {

constexpr int kGatherWarps = 8;           // warps per block
constexpr int kGatherMaxVecPerLane = 8;   // d <= 32 * 8 * 8 = 2048 in the unrolled path

constexpr int kBulkRowsPerBlock = 32;      // one row per lane of the block's single warp
constexpr int kBulkSmemBudget = 160 * 1024;

// One block = one warp; lane l copies rows r0 + l of each block-stride step.
__global__ void __launch_bounds__(32)
gather_rows_bulk_kernel(const uint8_t* __restrict__ h, int64_t ld_bytes, uint32_t row_bytes,
                        const int32_t* __restrict__ idx, int64_t K, int64_t N, int rows_per_block,
                        const int32_t* __restrict__ pos_in, const float* __restrict__ scores,
                        uint8_t* __restrict__ h_out, int32_t* __restrict__ pos_out, float* __restrict__ s_out) {
    extern __shared__ __align__(128) uint8_t g_smem[];
    const int lane = threadIdx.x;
    uint64_t* bar = reinterpret_cast<uint64_t*>(g_smem + static_cast<size_t>(rows_per_block) * row_bytes) + lane;
    if (lane < rows_per_block) mbar_init(bar, 1);
    fence_mbar_init();
    __syncwarp();
    pdl_trigger();
    pdl_wait();  // global memory is shared with the kernels before this one from here on
    uint8_t* slot = g_smem + static_cast<size_t>(lane) * row_bytes;
    uint32_t ph = 0;
    for (int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per_block; r0 < K;
         r0 += static_cast<int64_t>(gridDim.x) * rows_per_block) {
        const int64_t r = r0 + lane;
        const bool live = lane < rows_per_block && r < K;
        const int32_t src = live ? __ldg(idx + r) : 0;
        const bool ok = live && src >= 0 && static_cast<int64_t>(src) < N;
        if (ok) {
            mbar_arrive_expect_tx(bar, row_bytes);
            bulk_load(slot, h + static_cast<int64_t>(src) * ld_bytes, row_bytes, bar);
        }
        if (live) {
            pos_out[r] = ok ? (pos_in ? __ldg(pos_in + src) : src) : -1;
            if (s_out && !ok) s_out[r] = __int_as_float(0x7fc00000);
            if (s_out && ok && scores) s_out[r] = __ldg(scores + src);
        }
        if (ok) {
            // the copy of a valid row always completes; the wait is bounded all the same, and a
            // row whose copy has not landed in time is reported like a bad index
            bool landed = mbar_try_wait(bar, ph);
            if (!landed) {
                const unsigned long long t0 = globaltimer_ns();
                while (!(landed = mbar_try_wait(bar, ph)) && globaltimer_ns() - t0 <= kWaitLimitNs) {
                }
            }
            ph ^= 1u;
            if (landed) {
                bulk_store(h_out + r * static_cast<int64_t>(row_bytes), slot, row_bytes);
                bulk_commit();
            } else {
                pos_out[r] = -2;
            }
        } else if (live) {
            uint4* d = reinterpret_cast<uint4*>(h_out + r * static_cast<int64_t>(row_bytes));
            for (uint32_t c = 0; c < row_bytes / 16; ++c) d[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        bulk_wait_read_all();  // the slot is read out before the next row lands in it
    }
    bulk_wait_all();
}

template <int VPL>
__global__ void __launch_bounds__(kGatherWarps * 32)
gather_rows_kernel(const uint4* __restrict__ h, int64_t ld_vec, int vec_per_row, const int32_t* __restrict__ idx,
                   int64_t K, int64_t N, const int32_t* __restrict__ pos_in, const float* __restrict__ scores,
                   uint4* __restrict__ h_out, int32_t* __restrict__ pos_out, float* __restrict__ s_out) {
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = static_cast<int64_t>(blockIdx.x) * kGatherWarps + (threadIdx.x >> 5);
    const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * kGatherWarps;
    for (int64_t r = warp_global; r < K; r += warp_stride) {
        const int32_t src = __ldg(idx + r);
        uint4* d = h_out + r * static_cast<int64_t>(vec_per_row);
        if (src < 0 || static_cast<int64_t>(src) >= N) {  // not read: zero row, position -1, score NaN
            for (int c = lane; c < vec_per_row; c += 32) d[c] = make_uint4(0u, 0u, 0u, 0u);
            if (lane == 0) {
                pos_out[r] = -1;
                if (s_out) s_out[r] = __int_as_float(0x7fc00000);
            }
            continue;
        }
        const uint4* s = h + static_cast<int64_t>(src) * ld_vec;
        if constexpr (VPL > 0) {
            uint4 v[VPL];
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int c = j * 32 + lane;
                if (c < vec_per_row) v[j] = __ldcs(s + c);
            }
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const int c = j * 32 + lane;
                if (c < vec_per_row) d[c] = v[j];
            }
        } else {
            for (int c = lane; c < vec_per_row; c += 32) d[c] = __ldcs(s + c);
        }
        if (lane == 0) {
            pos_out[r] = pos_in ? __ldg(pos_in + src) : src;
            if (scores && s_out) s_out[r] = __ldg(scores + src);
        }
    }
}

}  // namespace tg

using namespace tg;

extern "C" tg_status tg_gather_compact(const tg_bf16* h, int64_t N, int32_t d, int64_t ld_h,
                                       const int32_t* kept_idx, int64_t K, const int32_t* pos_in,
                                       const float* scores, tg_bf16* h_out, int32_t* pos_out, float* s_out,
                                       void* stream) {
    if (N < 0 || K < 0 || d <= 0 || ld_h < d) return TG_ERR_INVALID_ARG;
    if (K == 0) return TG_OK;
    if (!h || !kept_idx || !h_out || !pos_out) return TG_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(h_out)) return TG_ERR_INVALID_ARG;
    if ((d % 8) != 0 || (ld_h % 8) != 0) return TG_ERR_UNSUPPORTED;
    const int vec_per_row = d / 8;
    const int64_t ld_vec = ld_h / 8;
    const int sms = num_sms();
    cudaStream_t st = as_stream(stream);
    const uint32_t row_bytes = static_cast<uint32_t>(d) * 2u;
    const int rows_per_block =
        static_cast<int>(std::min<int64_t>(kBulkRowsPerBlock, kBulkSmemBudget / static_cast<int64_t>(row_bytes)));
    if (rows_per_block >= 8) {
        const int smem = rows_per_block * static_cast<int>(row_bytes) + kBulkRowsPerBlock * 8;
        static std::atomic<int> smem_set[64];
        if (!set_max_dynamic_smem(gather_rows_bulk_kernel, smem, smem_set)) return TG_ERR_CUDA;
        const int64_t blocks = std::min<int64_t>((K + rows_per_block - 1) / rows_per_block, static_cast<int64_t>(sms));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(blocks));
        cfg.blockDim = dim3(32);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1] = {pdl_attr()};
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, gather_rows_bulk_kernel, reinterpret_cast<const uint8_t*>(h), ld_h * 2,
                                  row_bytes, kept_idx, K, N, rows_per_block, pos_in, scores,
                                  reinterpret_cast<uint8_t*>(h_out), pos_out, s_out) == cudaSuccess
                   ? TG_OK
                   : TG_ERR_CUDA;
    }
    int64_t blocks = (K + kGatherWarps - 1) / kGatherWarps;
    const int64_t max_blocks = static_cast<int64_t>(sms) * 8;  // 8 resident blocks of 256 threads per SM
    if (blocks > max_blocks) blocks = max_blocks;
    const uint4* src = reinterpret_cast<const uint4*>(h);
    uint4* dst = reinterpret_cast<uint4*>(h_out);
    const int vpl = (vec_per_row + 31) / 32;
    if (vpl <= 1)
        gather_rows_kernel<1><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, N, pos_in, scores, dst, pos_out, s_out);
    else if (vpl <= 2)
        gather_rows_kernel<2><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, N, pos_in, scores, dst, pos_out, s_out);
    else if (vpl <= 4)
        gather_rows_kernel<4><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, N, pos_in, scores, dst, pos_out, s_out);
    else if (vpl <= kGatherMaxVecPerLane)
        gather_rows_kernel<kGatherMaxVecPerLane><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, N, pos_in, scores, dst, pos_out, s_out);
    else
        gather_rows_kernel<0><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, N, pos_in, scores, dst, pos_out, s_out);
    return launch_status();
}
