// noalloc.cu -- dash_decode_noalloc: the decode step with library-owned scratch memory.
//
// dash_decode takes its scratch (scores, thresholds, block lists, split-KV partials) from a
// workspace the caller allocates.  Some callers cannot allocate device memory at the point
// where they decode: real-time serving loops that must not pay the device-wide
// synchronisation cudaMalloc / cudaFree can cause, hosts whose device memory is owned by
// another allocator that this library cannot call, and plug-in code that is handed only
// the buffers of its inputs and outputs.  For them this file keeps one fixed scratch array
// in device memory, declared below, and runs the unchanged decode kernels on it.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes (32 MiB); every GPU
// that loads this library holds it until the process exits.  In host code the name
// g_noalloc_scratch is only a host-side stand-in for the symbol, never a device address,
// so the device address is looked up with cudaGetSymbolAddress at set-up, once per device
// (with that device current), and cached together with the identity of the device's
// context: a context created anew (after cudaDeviceReset, say) gets the module loaded
// again, possibly at another address, so a changed identity repeats the set-up.
#include <cudaTypedefs.h>

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
struct ScratchSlot {
    unsigned long long ctx_id;   // identity of the context the address belongs to
    void* ptr;                   // device address of g_noalloc_scratch in that context
};
ScratchSlot g_slot[kMaxDevices] = {};

// Identity of the calling thread's current context (driver entry points reached through the
// runtime, so no libcuda link is needed).  False when no context is current or the driver
// lacks the calls.
bool current_ctx_id(unsigned long long* id) {
    static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    if (!get_cur || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device.  The set-up (the symbol
// lookup) runs on the first call on each device, and again after the device's context has
// been replaced; it is refused while `stream` is being captured.
int scratch_address(cudaStream_t stream, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DASH_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return DASH_ERR_CUDA;
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    ScratchSlot& s = g_slot[dev];
    if (s.ptr != nullptr && have_id && s.ctx_id == id) {
        *out = s.ptr;
        return DASH_OK;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return DASH_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return DASH_ERR_SETUP_IN_CAPTURE;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return DASH_ERR_CUDA;
    // the lookup made the device's primary context current if it was not already
    if (!current_ctx_id(&id)) id = 0;
    s.ctx_id = id;
    s.ptr = p;
    *out = p;
    return DASH_OK;
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
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    const int rc = scratch_address(s, &ws);
    if (rc != DASH_OK) return rc;
    // counters and the status word must start at zero; every other region is written
    // before it is read within the call
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), s) != cudaSuccess) return DASH_ERR_CUDA;
    return launch_decode(q, k_cache, v_cache, ksum, kv_len, out, g, static_cast<char*>(ws), alpha,
                         coarse_scale, s, nullptr) == cudaSuccess
               ? DASH_OK : DASH_ERR_CUDA;
}

extern "C" int dash_decode_noalloc_status(dash_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return DASH_ERR_CUDA;
    // the status word is the first int of the workspace header at the start of the array
    int st = 0;
    if (cudaMemcpyFromSymbol(&st, g_noalloc_scratch, sizeof st, 0, cudaMemcpyDeviceToHost) != cudaSuccess)
        return DASH_ERR_CUDA;
    if (st & kStWaitTimeout) return DASH_ERR_DEVICE_TIMEOUT;
    return (st & kStNoConverge) ? DASH_ERR_NO_CONVERGE : DASH_OK;
}
