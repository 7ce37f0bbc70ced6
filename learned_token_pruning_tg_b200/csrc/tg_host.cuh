// tg_host.cuh -- host-side helpers shared by the libtokengate entry points:
// argument checks, the SM count of the current device, and TMA tensor-map
// encoding through the driver entry point (no link-time libcuda dependency).
#pragma once

#include <atomic>
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tokengate.h"
#include "tg_device.cuh"

namespace tg {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Byte offset of the per-op region of a workspace (after the status header and
// the select scratch); defined with the workspace sizing.
size_t ws_gate_offset();

inline int current_device() {
    int dev = 0;
    return (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) ? dev : -1;
}

// Whether the gate (d_g = 256) and the projection may use their CTA-pair kernels (the default);
// tg_debug_set_cta_pairs(0) makes them take their one-CTA kernels, so tests can run both.
inline std::atomic<int>& cta_pairs_enabled() {
    static std::atomic<int> enabled{1};
    return enabled;
}

// Number of SMs of the current device (queried once per device).
inline int num_sms() {
    static int cache[64] = {0};
    const int dev = current_device();
    if (dev < 0) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// A tensor map is a pure function of its arguments, and encoding one costs
// microseconds of host time per call; each host thread keeps its last few.
struct TmapKey {
    const void* base;
    uint64_t dims[5], strides[4];
    uint32_t box[5];
    int32_t rank, promo, swizzle, dtype;
};
struct TmapCache {
    static constexpr int kEntries = 16;
    TmapKey key[kEntries];
    CUtensorMap map[kEntries];
    bool used[kEntries] = {};
    int next = 0;
};

// Tensor map over a bf16 tensor of `rank` dims (dims[0] innermost, in elements;
// strides[i] in bytes for dims 1..rank-1), box `box` (elements), 128-byte swizzle
// unless `swizzle` says otherwise (and bf16 unless `dtype` does).
inline bool make_tmap_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box,
                           CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B,
                           CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    if (rank < 1 || rank > 5) return false;
    TmapKey k;
    std::memset(&k, 0, sizeof(k));  // padding too, so keys compare bytewise
    k.base = base;
    k.rank = rank;
    k.promo = static_cast<int32_t>(promo);
    k.swizzle = static_cast<int32_t>(swizzle);
    k.dtype = static_cast<int32_t>(dtype);
    for (int i = 0; i < rank; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides_bytes[i];
    thread_local TmapCache cache;
    for (int i = 0; i < TmapCache::kEntries; ++i)
        if (cache.used[i] && std::memcmp(&cache.key[i], &k, sizeof(k)) == 0) {
            *m = cache.map[i];
            return true;
        }
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[5];
    cuuint64_t gstride[4];
    cuuint32_t bdim[5];
    cuuint32_t estride[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estride[i] = 1;
    }
    for (int i = 0; i + 1 < rank; ++i) gstride[i] = strides_bytes[i];
    CUresult r = fn(m, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                    gdim, gstride, bdim, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promo,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    const int slot = cache.next;
    cache.next = (slot + 1) % TmapCache::kEntries;
    cache.key[slot] = k;
    cache.map[slot] = *m;
    cache.used[slot] = true;
    return true;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and device;
// `done` is a per-kernel array of 64 flags owned by the caller (a static in the
// kernel's own launch function).
template <typename Kernel>
inline bool set_max_dynamic_smem(Kernel* kern, int bytes, std::atomic<int>* done) {
    const int dev = current_device();
    if (dev >= 0 && done[dev].load(std::memory_order_acquire) == bytes) return true;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    if (dev >= 0) done[dev].store(bytes, std::memory_order_release);
    return true;
}

// Launch attribute letting a kernel start while the previous kernel on the stream finishes (the
// kernel itself calls pdl_wait() before touching memory the previous kernels use).
inline cudaLaunchAttribute pdl_attr() {
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at.val.programmaticStreamSerializationAllowed = 1;
    return at;
}

inline tg_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

inline unsigned int* status_word(void* ws) { return static_cast<unsigned int*>(ws); }

}  // namespace tg
