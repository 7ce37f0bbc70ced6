// gated_attention.cu -- token-gated causal GQA attention over the kept tokens.
// (Kernel in progress: the entry point validates its arguments and reports
// TG_ERR_UNSUPPORTED until the tcgen05 kernel lands.)
#include "tg_host.cuh"

using namespace tg;

extern "C" tg_status tg_gated_attention(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                        const tg_bf16* v, int64_t ld_v, int64_t K, int32_t Hq, int32_t Hkv,
                                        int32_t d_h, const float* s_kept, const float* gain, float tau,
                                        tg_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    if (K < 0 || Hq <= 0 || Hkv <= 0 || (Hq % Hkv) != 0) return TG_ERR_INVALID_ARG;
    if (d_h != 64 && d_h != 128) return TG_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return TG_ERR_INVALID_ARG;
    (void)ld_q; (void)ld_k; (void)ld_v; (void)s_kept; (void)gain; (void)tau; (void)lse;
    (void)workspace; (void)workspace_bytes; (void)stream;
    return TG_ERR_UNSUPPORTED;
}
