// tg_abi.cu -- the parts of the libtokengate C ABI that belong to no single
// kernel: status strings, version, kept count, workspace sizing and the
// device status read-back.
//
// Workspace layout (one buffer can serve every call on a stream):
//   [0, 256)                 status word (sticky TG_STATUS_* bits) + padding
//   [256, 256 + S)           select scratch: grid-barrier counter, radix
//                            histograms, per-block counts (self-cleaning)
//   [256 + S', ...)          gate: bf16(rms_weight * W1) when rms_weight given;
//                            attention: fp16 copy of V (the two are rebuilt by
//                            every call that uses them, so they may overlap)
#include <cstdio>

#include "tg_host.cuh"

namespace tg {
size_t ws_gate_offset() { return kWsHeader + ((sizeof(SelectScratch) + 255) / 256) * 256; }
size_t ws_decode_bytes(int32_t Hq);  // gated_decode.cu
size_t ws_attn_bwd_bytes(int64_t K, int32_t Hq, int32_t Hkv);  // gated_attention_bwd.cu
size_t ws_project_bytes(int64_t K, int32_t d_h);                 // project_rope.cu
}  // namespace tg

using namespace tg;

extern "C" const char* tg_status_string(tg_status s) {
    switch (s) {
        case TG_OK: return "ok";
        case TG_ERR_INVALID_ARG: return "invalid argument";
        case TG_ERR_UNSUPPORTED: return "unsupported shape";
        case TG_ERR_CUDA: return "CUDA launch or runtime error";
        case TG_ERR_TIMEOUT: return "device wait timed out";
        case TG_ERR_RANGE: return "a value out of range (V beyond fp16's range, or a row index outside [0, N))";
    }
    return "unknown status";
}

extern "C" int32_t tg_version(void) { return 100; /* 0.1.0 */ }

extern "C" int64_t tg_kept_count(int64_t N, int64_t doc_begin, int64_t doc_end, int64_t k_doc) {
    if (N < 0 || doc_begin < 0 || doc_end < doc_begin || doc_end > N || k_doc < 0) return -1;
    const int64_t n_doc = doc_end - doc_begin;
    return (k_doc < n_doc ? k_doc : n_doc) + (N - n_doc);
}

extern "C" size_t tg_workspace_bytes(tg_op op, int64_t N, int32_t d, int32_t d_g) {
    if (N < 0) return 0;
    const size_t gate = (d > 0 && d_g > 0) ? static_cast<size_t>(d) * static_cast<size_t>(d_g) * 2 : 0;
    const size_t attn = d > 0 ? static_cast<size_t>(N) * static_cast<size_t>(d) * 2 : 0;
    switch (op) {
        case TG_OP_SELECT: return kWsHeader + sizeof(SelectScratch);
        case TG_OP_ATTENTION: return d > 0 ? ws_gate_offset() + attn : 0;
        case TG_OP_GATE: return gate ? ws_gate_offset() + gate : 0;
        case TG_OP_ALL: return ws_gate_offset() + (gate > attn ? gate : attn);
        case TG_OP_DECODE: return (d > 0 && d <= 512) ? ws_decode_bytes(d) : 0;
        case TG_OP_ATTENTION_BACKWARD: return ws_attn_bwd_bytes(N, d, d_g);
        case TG_OP_PROJECT: return ws_project_bytes(N, d);
    }
    return 0;
}

extern "C" tg_status tg_device_status(const void* workspace, uint32_t* status_word_out, void* stream) {
    if (!workspace) return TG_ERR_INVALID_ARG;
    uint32_t w = 0;
    cudaStream_t st = as_stream(stream);
    if (cudaMemcpyAsync(&w, workspace, sizeof(w), cudaMemcpyDeviceToHost, st) != cudaSuccess) return TG_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return TG_ERR_CUDA;
    if (status_word_out) *status_word_out = w;
    if (w & TG_STATUS_TIMEOUT_BITS) return TG_ERR_TIMEOUT;
    return (w & (TG_STATUS_V_RANGE | TG_STATUS_INDEX_RANGE)) ? TG_ERR_RANGE : TG_OK;
}

extern "C" tg_status tg_debug_set_cta_pairs(int enabled) {
    tg::cta_pairs_enabled().store(enabled ? 1 : 0);
    return TG_OK;
}
