// rope_apply.cu -- rotary embedding of q and k at the kept tokens' ORIGINAL
// positions.  The TokenGate pages do not discuss positions; the specification
// carries the original position ids through compaction so that RoPE (and a
// later decode at position N) stays correct.  Pairing is rotate-half (t with
// t + d_h/2), Qwen3's convention; rotary base 1e6 for Qwen3.
//
// Angles are formed in fp64 (pos up to ~1.3e5 times an fp32 frequency would
// lose ~1e-2 rad), cos/sin are rounded to fp32, the rotation runs in fp32 and
// the result is rounded to bf16.  One block per token: the block computes the
// token's d_h/2 cos/sin pairs into shared memory, then every (head, 8-pair
// chunk) is rotated with 16-byte loads and stores.
#include <cmath>

#include "tg_host.cuh"

namespace tg {

__global__ void __launch_bounds__(128)
rope_kernel(__nv_bfloat16* __restrict__ q, int64_t ld_q, __nv_bfloat16* __restrict__ k, int64_t ld_k,
            const int32_t* __restrict__ pos, int Hq, int Hkv, int d_h, double base) {
    __shared__ float cs[64];
    __shared__ float sn[64];
    const int64_t r = blockIdx.x;
    const int half = d_h >> 1;
    const double p = static_cast<double>(__ldg(pos + r));
    for (int t = threadIdx.x; t < half; t += blockDim.x) {
        const double inv_freq = pow(base, -2.0 * static_cast<double>(t) / static_cast<double>(d_h));
        double s, c;
        sincos(p * inv_freq, &s, &c);
        cs[t] = static_cast<float>(c);
        sn[t] = static_cast<float>(s);
    }
    __syncthreads();
    const int chunks = half / 8;                 // 8 pairs per work item
    const int items = (Hq + Hkv) * chunks;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int head = it / chunks;
        const int t0 = (it % chunks) * 8;
        __nv_bfloat16* x = head < Hq ? q + r * ld_q + static_cast<int64_t>(head) * d_h
                                     : k + r * ld_k + static_cast<int64_t>(head - Hq) * d_h;
        uint4 a = *reinterpret_cast<const uint4*>(x + t0);
        uint4 b = *reinterpret_cast<const uint4*>(x + t0 + half);
        __nv_bfloat16* av = reinterpret_cast<__nv_bfloat16*>(&a);
        __nv_bfloat16* bv = reinterpret_cast<__nv_bfloat16*>(&b);
        uint4 oa, ob;
        __nv_bfloat16* oav = reinterpret_cast<__nv_bfloat16*>(&oa);
        __nv_bfloat16* obv = reinterpret_cast<__nv_bfloat16*>(&ob);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float x1 = __bfloat162float(av[j]);
            const float x2 = __bfloat162float(bv[j]);
            const float c = cs[t0 + j], s = sn[t0 + j];
            oav[j] = __float2bfloat16_rn(x1 * c - x2 * s);
            obv[j] = __float2bfloat16_rn(x2 * c + x1 * s);
        }
        *reinterpret_cast<uint4*>(x + t0) = oa;
        *reinterpret_cast<uint4*>(x + t0 + half) = ob;
    }
}

}  // namespace tg

using namespace tg;

extern "C" tg_status tg_rope_apply(tg_bf16* q, int64_t ld_q, tg_bf16* k, int64_t ld_k, const int32_t* pos,
                                   int64_t K, int32_t Hq, int32_t Hkv, int32_t d_h, double base, void* stream) {
    if (K < 0 || Hq < 0 || Hkv < 0 || !(base > 0.0)) return TG_ERR_INVALID_ARG;
    if (K == 0 || Hq + Hkv == 0) return TG_OK;
    if (!pos || (Hq > 0 && !q) || (Hkv > 0 && !k)) return TG_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return TG_ERR_UNSUPPORTED;
    if ((Hq > 0 && (!aligned16(q) || ld_q < static_cast<int64_t>(Hq) * d_h || (ld_q % 8))) ||
        (Hkv > 0 && (!aligned16(k) || ld_k < static_cast<int64_t>(Hkv) * d_h || (ld_k % 8))))
        return TG_ERR_INVALID_ARG;
    if (K > 0x7fffffffLL) return TG_ERR_UNSUPPORTED;
    rope_kernel<<<static_cast<unsigned>(K), 128, 0, as_stream(stream)>>>(
        reinterpret_cast<__nv_bfloat16*>(q), ld_q, reinterpret_cast<__nv_bfloat16*>(k), ld_k, pos, Hq, Hkv, d_h,
        base);
    return launch_status();
}
