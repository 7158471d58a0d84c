// noalloc.cu -- dash_decode_noalloc: the decode step with library-owned scratch memory.
//
// dash_decode takes its scratch (scores, thresholds, block lists, split-KV partials) from a
// workspace the caller allocates.  Some callers cannot allocate device memory at the point
// where they decode: code that runs while a CUDA graph is being captured (cudaMalloc is not
// a capturable operation), real-time serving loops that must not pay the device-wide
// synchronisation cudaMalloc / cudaFree can cause, and hosts whose device memory is owned
// by another allocator that this library cannot call.  For them this file keeps one fixed
// scratch array in device memory, declared below, and runs the unchanged decode kernels on
// it.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes (32 MiB); every GPU
// that loads this library holds it until the process exits.  In host code the name
// g_noalloc_scratch is only a host-side stand-in for the symbol, never a device address,
// so the device address is looked up with cudaGetSymbolAddress once per device (with that
// device current) on the first call made on that device, and cached.
#include <mutex>

#include "../../include/dash_attn.h"
#include "common.cuh"
#include "kernels.h"

namespace dash {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace dash

using namespace dash;

extern "C" int dash_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                   const float* ksum, const int* kv_len, void* out, int B, int Hq,
                                   int Hkv, int Tmax, int d, int block, float alpha,
                                   float coarse_scale, dash_stream_t stream) {
    if (!q || !k_cache || !v_cache || !ksum || !kv_len || !out) return DASH_ERR_ARG;
    const auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!al16(q) || !al16(k_cache) || !al16(v_cache) || !al16(ksum) || !al16(out)) return DASH_ERR_ARG;
    if (!(alpha > 1.0f) || !isfinite(alpha) || !isfinite(coarse_scale)) return DASH_ERR_ARG;
    DecodeGeom g;
    if (block != kBlock || !make_decode_geom(B, Hq, Hkv, Tmax, d, &g)) return DASH_ERR_SHAPE;
    if (g.total > kNoAllocScratchBytes) return DASH_ERR_SCRATCH_LIMIT;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return DASH_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // counters and the status word must start at zero; every other region is written
    // before it is read within the call
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), s) != cudaSuccess) return DASH_ERR_CUDA;
    return launch_decode(q, k_cache, v_cache, ksum, kv_len, out, g, static_cast<char*>(ws), alpha,
                         coarse_scale, s, nullptr) == cudaSuccess
               ? DASH_OK : DASH_ERR_CUDA;
}
