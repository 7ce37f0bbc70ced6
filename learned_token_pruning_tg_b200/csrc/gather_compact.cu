// gather_compact.cu -- compaction of the kept rows (TokenGate: the layers above
// the gate process only the K kept tokens and write no KV entries for the
// pruned ones; chathome.org article, section TokenGate の学習可能なトークン
// プルーニングの仕組み).  The kept rows, their original positions (which RoPE
// needs) and their gate scores are copied bit-exactly.
//
// Design: HBM-bound row copy.  One warp per kept row; each lane moves 16-byte
// vectors, all loads of a row are issued before its stores so that every warp
// keeps a whole row (4 KB at d = 2048) in flight.  Source rows are read with
// the no-allocate/streaming hint (each is read once); destination rows are
// stored normally because the next layer's projection reads them right away.
#include "tg_host.cuh"

namespace tg {

constexpr int kGatherWarps = 8;           // warps per block
constexpr int kGatherMaxVecPerLane = 8;   // d <= 32 * 8 * 8 = 2048 in the unrolled path

template <int VPL>
__global__ void __launch_bounds__(kGatherWarps * 32)
gather_rows_kernel(const uint4* __restrict__ h, int64_t ld_vec, int vec_per_row, const int32_t* __restrict__ idx,
                   int64_t K, const int32_t* __restrict__ pos_in, const float* __restrict__ scores,
                   uint4* __restrict__ h_out, int32_t* __restrict__ pos_out, float* __restrict__ s_out) {
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = static_cast<int64_t>(blockIdx.x) * kGatherWarps + (threadIdx.x >> 5);
    const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * kGatherWarps;
    for (int64_t r = warp_global; r < K; r += warp_stride) {
        const int32_t src = __ldg(idx + r);
        const uint4* s = h + static_cast<int64_t>(src) * ld_vec;
        uint4* d = h_out + r * static_cast<int64_t>(vec_per_row);
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
    int64_t blocks = (K + kGatherWarps - 1) / kGatherWarps;
    const int64_t max_blocks = static_cast<int64_t>(sms) * 8;  // 8 resident blocks of 256 threads per SM
    if (blocks > max_blocks) blocks = max_blocks;
    cudaStream_t st = as_stream(stream);
    const uint4* src = reinterpret_cast<const uint4*>(h);
    uint4* dst = reinterpret_cast<uint4*>(h_out);
    const int vpl = (vec_per_row + 31) / 32;
    if (vpl <= 1)
        gather_rows_kernel<1><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, pos_in, scores, dst, pos_out, s_out);
    else if (vpl <= 2)
        gather_rows_kernel<2><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, pos_in, scores, dst, pos_out, s_out);
    else if (vpl <= 4)
        gather_rows_kernel<4><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, pos_in, scores, dst, pos_out, s_out);
    else if (vpl <= kGatherMaxVecPerLane)
        gather_rows_kernel<kGatherMaxVecPerLane><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, pos_in, scores, dst, pos_out, s_out);
    else
        gather_rows_kernel<0><<<static_cast<unsigned>(blocks), kGatherWarps * 32, 0, st>>>(
            src, ld_vec, vec_per_row, kept_idx, K, pos_in, scores, dst, pos_out, s_out);
    return launch_status();
}
