// api.cu -- the extern "C" entry points declared in include/dash_attn.h.
//
// Argument checks happen here, before any launch; kernels live in summary.cu, coarse.cu,
// coarse_tc.cu, fine_mma.cu, fine_tc.cu, backward.cu, decode.cu, decode_tc.cu and dump.cu.
// Nothing here allocates memory.
#include <algorithm>
#include <math.h>

#include <new>
#include <stdint.h>
#include <string.h>

#include "../../include/dash_attn.h"
#include "common.cuh"
#include "kernels.h"

using namespace dash;

namespace {

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
inline cudaStream_t S(dash_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool good_params(float alpha, float cs) {
    return isfinite(alpha) && alpha > 1.0f && isfinite(cs);
}

int read_stats(const void* ws, size_t ws_bytes, dash_stats* out, dash_stream_t stream) {
    if (!ws || !out || ws_bytes < sizeof(WsHeader)) return DASH_ERR_ARG;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return DASH_ERR_CUDA;
    WsHeader h;
    if (cudaMemcpy(&h, ws, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return DASH_ERR_CUDA;
    out->scored_pairs = (long long)h.scored_pairs;
    out->selected_pairs = (long long)h.selected_pairs;
    out->union_blocks = (long long)h.union_blocks;
    out->tiles = (long long)h.tiles;
    out->status = h.status;
    out->fine_steps = (long long)h.fine_steps;
    return DASH_OK;
}

// Selection-ordered tiles apply on the tensor-core path with at least one complete block and
// per-head priors; DASH_TILES=positions keeps the position tiles (for comparisons).
bool ordered_tiles_enabled(const PrefillGeom& g, int agg) {
    if (!g.tc || !coarse_tc_supported(g) || !fine_tc_supported(g) || agg || g.nbs == 0) return false;
    const char* e = getenv("DASH_TILES");
    return !(e && strcmp(e, "positions") == 0);
}

}  // namespace

extern "C" {

const char* dash_status_string(int status) {
    switch (status) {
        case DASH_OK: return "DASH_OK";
        case DASH_ERR_ARG: return "DASH_ERR_ARG: null or misaligned pointer, or bad alpha / coarse_scale";
        case DASH_ERR_SHAPE: return "DASH_ERR_SHAPE: unsupported B, H, T, d or block";
        case DASH_ERR_DTYPE: return "DASH_ERR_DTYPE";
        case DASH_ERR_UNSUPPORTED: return "DASH_ERR_UNSUPPORTED";
        case DASH_ERR_WORKSPACE: return "DASH_ERR_WORKSPACE: workspace null, misaligned or too small";
        case DASH_ERR_CUDA: return "DASH_ERR_CUDA: a CUDA runtime call failed";
        case DASH_ERR_NO_CONVERGE: return "DASH_ERR_NO_CONVERGE: a threshold solve hit its iteration cap";
        case DASH_ERR_DEVICE_TIMEOUT: return "DASH_ERR_DEVICE_TIMEOUT: a device-side wait gave up; outputs invalid";
        case DASH_ERR_SCRATCH_LIMIT: return "DASH_ERR_SCRATCH_LIMIT: the decode step needs more than the 32 MiB static scratch";
        case DASH_ERR_SETUP_IN_CAPTURE:
            return "DASH_ERR_SETUP_IN_CAPTURE: dash_decode_noalloc's once-per-device set-up fell due while the stream "
                   "was being captured; make one call outside capture first";
        default: return "unknown dash status";
    }
}

int dash_version(void) { return 100; }

int dash_block_summary(const void* k, float* ksum, int B, int Hkv, int T, int d, int block,
                       dash_stream_t stream) {
    if (!k || !ksum || !al16(k) || !al16(ksum)) return DASH_ERR_ARG;
    if (block != kBlock || (d != 64 && d != 128) || B < 1 || Hkv < 1 || T < 1 || T > kMaxT)
        return DASH_ERR_SHAPE;
    return launch_block_summary(k, ksum, B, Hkv, T, d, S(stream)) == cudaSuccess ? DASH_OK : DASH_ERR_CUDA;
}

int dash_block_summary_w(const void* k, const float* w, float* ksum, int B, int Hkv, int T, int d,
                         int block, dash_stream_t stream) {
    if (!k || !w || !ksum || !al16(k) || !al16(w) || !al16(ksum)) return DASH_ERR_ARG;
    if (block != kBlock || (d != 64 && d != 128) || B < 1 || Hkv < 1 || T < 1 || T > kMaxT)
        return DASH_ERR_SHAPE;
    return launch_block_summary(k, ksum, B, Hkv, T, d, S(stream), nullptr, nullptr, w) == cudaSuccess
               ? DASH_OK : DASH_ERR_CUDA;
}

size_t dash_prefill_workspace_size(int B, int Hq, int Hkv, int T, int d, int block) {
    PrefillGeom g;
    if (block != kBlock || !make_prefill_geom(B, Hq, Hkv, T, d, &g)) return 0;
    return g.total;
}

static int prefill_impl(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                        int Hkv, int T, int d, int block, float alpha, float coarse_scale,
                        void* workspace, size_t ws_bytes, dash_stream_t stream, void* const* events,
                        const float* wsum = nullptr, unsigned flags = 0, const FineDump* dump = nullptr,
                        size_t dump_entries = 0) {
    if (!q || !k || !v || !out || !al16(q) || !al16(k) || !al16(v) || !al16(out)) return DASH_ERR_ARG;
    if (wsum && !al16(wsum)) return DASH_ERR_ARG;
    if (!good_params(alpha, coarse_scale)) return DASH_ERR_ARG;
    PrefillGeom g;
    if (block != kBlock || !make_prefill_geom(B, Hq, Hkv, T, d, &g)) return DASH_ERR_SHAPE;
    if (flags & ~(unsigned)DASH_HEAD_AGGREGATION) return DASH_ERR_ARG;
    const int agg = (flags & DASH_HEAD_AGGREGATION) ? 1 : 0;
    // the CUDA-core fine kernel recovers q . kbar from the mean of the block's scores, which
    // only a mean summary satisfies, and keeps per-head priors only
    const bool need_tc = wsum != nullptr || agg || dump != nullptr;
    if (need_tc && !fine_tc_supported(g)) return DASH_ERR_UNSUPPORTED;
    if (!workspace || !al256(workspace) || ws_bytes < g.total) return DASH_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    cudaStream_t s = S(stream);
    auto mark = [&](int i) {
        return !events || cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[i]), s) == cudaSuccess;
    };
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), s) != cudaSuccess) return DASH_ERR_CUDA;
    if (!mark(0)) return DASH_ERR_CUDA;
    if (g.nbs > 0 && launch_block_summary(k, reinterpret_cast<float*>(ws + g.off_ksum), B, Hkv, T, d, s,
                                          ws + g.off_khi, ws + g.off_klo, wsum) != cudaSuccess)
        return DASH_ERR_CUDA;
    if (!mark(1)) return DASH_ERR_CUDA;
    // selection-ordered tiles on the tensor-core path (head aggregation averages over the
    // heads of a position, which position tiles keep together)
    const bool ordered = ordered_tiles_enabled(g, agg);
    const cudaError_t ce = g.tc ? (coarse_tc_supported(g) ? launch_coarse_tc(q, g, ws, alpha, coarse_scale, s, ordered)
                                                          : launch_coarse(q, g, ws, alpha, coarse_scale, s))
                                : launch_coarse(q, g, ws, alpha, coarse_scale, s);
    if (ce != cudaSuccess) return DASH_ERR_CUDA;
    if (ordered && launch_order_tiles(g, ws, s) != cudaSuccess) return DASH_ERR_CUDA;
    if (!mark(2)) return DASH_ERR_CUDA;
    if (dump) {
        if (launch_dump_fill(dump->x, dump->p, dump_entries, s) != cudaSuccess ||
            launch_fine_tc(q, k, v, out, g, ws, alpha, coarse_scale, s, agg, dump, ordered) != cudaSuccess)
            return DASH_ERR_CUDA;
    } else if (ordered) {
        if (launch_fine_tc(q, k, v, out, g, ws, alpha, coarse_scale, s, agg, nullptr, true) != cudaSuccess)
            return DASH_ERR_CUDA;
    } else if (launch_fine(q, k, v, out, g, ws, alpha, coarse_scale, s, agg, need_tc) != cudaSuccess) {
        return DASH_ERR_CUDA;
    }
    if (!mark(3)) return DASH_ERR_CUDA;
    return DASH_OK;
}

int dash_prefill(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv,
                 int T, int d, int block, float alpha, float coarse_scale, void* workspace,
                 size_t ws_bytes, dash_stream_t stream) {
    return prefill_impl(q, k, v, out, B, Hq, Hkv, T, d, block, alpha, coarse_scale, workspace,
                        ws_bytes, stream, nullptr);
}

int dash_prefill_w(const void* q, const void* k, const void* v, const float* w_summary, void* out, int B,
                   int Hq, int Hkv, int T, int d, int block, float alpha, float coarse_scale, void* workspace,
                   size_t ws_bytes, dash_stream_t stream) {
    return prefill_impl(q, k, v, out, B, Hq, Hkv, T, d, block, alpha, coarse_scale, workspace,
                        ws_bytes, stream, nullptr, w_summary);
}

int dash_prefill_ex(const void* q, const void* k, const void* v, const float* w_summary, void* out, int B,
                    int Hq, int Hkv, int T, int d, int block, float alpha, float coarse_scale,
                    unsigned flags, void* workspace, size_t ws_bytes, dash_stream_t stream) {
    return prefill_impl(q, k, v, out, B, Hq, Hkv, T, d, block, alpha, coarse_scale, workspace,
                        ws_bytes, stream, nullptr, w_summary, flags);
}

int dash_prefill_dump(const void* q, const void* k, const void* v, const float* w_summary, void* out, int B,
                      int Hq, int Hkv, int T, int d, int block, float alpha, float coarse_scale, unsigned flags,
                      const int* row_slot, int nslots, float* x_out, float* p_out, void* workspace,
                      size_t ws_bytes, dash_stream_t stream) {
    if (nslots < 0) return DASH_ERR_ARG;
    if (!row_slot || (nslots > 0 && (!x_out || !p_out))) return DASH_ERR_ARG;
    if (block != kBlock || T < 1) return DASH_ERR_SHAPE;
    FineDump dump{row_slot, x_out, p_out};
    return prefill_impl(q, k, v, out, B, Hq, Hkv, T, d, block, alpha, coarse_scale, workspace, ws_bytes,
                        stream, nullptr, w_summary, flags, &dump, (size_t)nslots * (size_t)(T / kBlock));
}

size_t dash_prefill_backward_workspace_size(int B, int Hq, int Hkv, int T, int d, int block) {
    PrefillGeom g;
    if (block != kBlock || !make_prefill_geom(B, Hq, Hkv, T, d, &g)) return 0;
    BwdGeom bw;
    make_bwd_geom(g, &bw);
    return bw.total;
}

int dash_prefill_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                          void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int T, int d, int block,
                          float alpha, float coarse_scale, void* workspace, size_t ws_bytes,
                          dash_stream_t stream) {
    if (!q || !k || !v || !out || !dout || !dq || !dk || !dv) return DASH_ERR_ARG;
    if (!al16(q) || !al16(k) || !al16(v) || !al16(out) || !al16(dout) || !al16(dq) || !al16(dk) || !al16(dv))
        return DASH_ERR_ARG;
    if (!good_params(alpha, coarse_scale)) return DASH_ERR_ARG;
    PrefillGeom g;
    if (block != kBlock || !make_prefill_geom(B, Hq, Hkv, T, d, &g)) return DASH_ERR_SHAPE;
    BwdGeom bw;
    make_bwd_geom(g, &bw);
    if (!workspace || !al256(workspace) || ws_bytes < bw.total) return DASH_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    cudaStream_t s = S(stream);
    // the forward's Stage 0 and Stage 1 again: summaries, thresholds and tile lists
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), s) != cudaSuccess) return DASH_ERR_CUDA;
    if (g.nbs > 0 && launch_block_summary(k, reinterpret_cast<float*>(ws + g.off_ksum), B, Hkv, T, d, s,
                                          ws + g.off_khi, ws + g.off_klo) != cudaSuccess)
        return DASH_ERR_CUDA;
    const cudaError_t ce = (g.tc && coarse_tc_supported(g)) ? launch_coarse_tc(q, g, ws, alpha, coarse_scale, s)
                                                            : launch_coarse(q, g, ws, alpha, coarse_scale, s);
    if (ce != cudaSuccess) return DASH_ERR_CUDA;
    return launch_backward(q, k, v, out, dout, dq, dk, dv, g, bw, ws, alpha, coarse_scale, s) == cudaSuccess
               ? DASH_OK : DASH_ERR_CUDA;
}

int dash_prefill_profiled(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                          int Hkv, int T, int d, int block, float alpha, float coarse_scale,
                          void* workspace, size_t ws_bytes, dash_stream_t stream, void* const* events) {
    if (!events) return DASH_ERR_ARG;
    return prefill_impl(q, k, v, out, B, Hq, Hkv, T, d, block, alpha, coarse_scale, workspace,
                        ws_bytes, stream, events);
}

namespace {
// Adds a finished unit's header (status bits, statistics) into the header of the whole call.
// Units on different streams may finish together: atomics.
__global__ void accumulate_header_kernel(WsHeader* dst, const WsHeader* src) {
    if (threadIdx.x != 0) return;
    if (src->status) atomicOr(&dst->status, src->status);
    atomicAdd(&dst->scored_pairs, src->scored_pairs);
    atomicAdd(&dst->selected_pairs, src->selected_pairs);
    atomicAdd(&dst->union_blocks, src->union_blocks);
    atomicAdd(&dst->tiles, src->tiles);
    atomicAdd(&dst->fine_steps, src->fine_steps);
}
constexpr int kHostComputeStreams = 4;   // units of a host-buffer prefill in flight at once
}  // namespace

int dash_prefill_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                      void* q_dev, void* k_dev, void* v_dev, void* out_dev, int B, int Hq, int Hkv,
                      int T, int d, int block, float alpha, float coarse_scale, void* workspace,
                      size_t ws_bytes, dash_stream_t stream) {
    if (!q_host || !k_host || !v_host || !out_host) return DASH_ERR_ARG;
    PrefillGeom g;
    if (block != kBlock || !make_prefill_geom(B, Hq, Hkv, T, d, &g)) return DASH_ERR_SHAPE;
    if (!q_dev || !k_dev || !v_dev || !out_dev) return DASH_ERR_ARG;
    if (!good_params(alpha, coarse_scale)) return DASH_ERR_ARG;
    if (!workspace || !al256(workspace) || ws_bytes < g.total) return DASH_ERR_WORKSPACE;
    cudaStream_t s = S(stream);
    // The rows of one query head depend only on that head's queries and its KV group's keys and
    // values, so any set of heads of one (b, kv head) group is an independent prefill on
    // contiguous slices of q, k, v and out.  The work is cut into units of one group and a chunk
    // of its heads (about 8 MiB of queries each), so the copies of one unit overlap the kernels
    // of others: copies in on one helper stream (a group's keys and values with its first
    // chunk), copies out on a second.  A unit's kernels take about the same time whatever its
    // head count (the rows at the end of the sequence, with the most blocks, set their
    // length), so up to kHostComputeStreams units run at once, each on its own compute stream
    // with its own slice of the workspace, and their tails overlap.  The workspace's header
    // collects every unit's status bits and statistics; `stream` finally waits for all of it.
    const int ng = B * Hkv, G = Hq / Hkv;
    const size_t hb = (size_t)T * d * 2;                                   // bytes per head
    const size_t qg = (size_t)G * hb, kg = hb;                             // bytes per group
    const int gc = (int)std::min<size_t>((size_t)G, std::max<size_t>(1, ((size_t)8 << 20) / std::max<size_t>(hb, 1)));
    const int nch = (G + gc - 1) / gc;                                     // head chunks per group
    const int nu = ng * nch;                                               // units
    auto cp = [](void* dst, const void* src, size_t n, cudaMemcpyKind kind, cudaStream_t st) {
        return cudaMemcpyAsync(dst, src, n, kind, st) == cudaSuccess;
    };
    auto at = [](const void* p, size_t off) { return static_cast<const char*>(p) + off; };
    auto atw = [](void* p, size_t off) { return static_cast<char*>(p) + off; };
    if (nu == 1) {
        if (!cp(k_dev, k_host, kg, cudaMemcpyHostToDevice, s) || !cp(v_dev, v_host, kg, cudaMemcpyHostToDevice, s) ||
            !cp(q_dev, q_host, qg, cudaMemcpyHostToDevice, s))
            return DASH_ERR_CUDA;
        int rc = dash_prefill(q_dev, k_dev, v_dev, out_dev, B, Hq, Hkv, T, d, block, alpha, coarse_scale,
                              workspace, ws_bytes, stream);
        if (rc != DASH_OK) return rc;
        return cp(out_host, out_dev, qg, cudaMemcpyDeviceToHost, s) ? DASH_OK : DASH_ERR_CUDA;
    }
    // a unit's workspace: the largest unit (gc heads of one group); slices after the header
    PrefillGeom gu;
    if (!make_prefill_geom(1, gc, 1, T, d, &gu)) return DASH_ERR_SHAPE;
    const size_t wsu = align256(gu.total);
    const int ns = (int)std::min<size_t>({(size_t)kHostComputeStreams, (size_t)nu,
                                          (ws_bytes - sizeof(WsHeader)) / wsu});
    if (ns < 1) return DASH_ERR_WORKSPACE;
    char* const ws0 = static_cast<char*>(workspace);
    auto unit_ws = [&](int i) { return ws0 + sizeof(WsHeader) + (size_t)i * wsu; };
    cudaStream_t sin = nullptr, sout = nullptr;
    cudaStream_t sc[kHostComputeStreams] = {};
    cudaEvent_t start = nullptr, fin = nullptr;
    cudaEvent_t* ev = new (std::nothrow) cudaEvent_t[2 * (size_t)nu]();
    int rc = DASH_OK;
    auto mkev = [](cudaEvent_t* e) { return cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess; };
    if (!ev || cudaStreamCreateWithFlags(&sin, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&sout, cudaStreamNonBlocking) != cudaSuccess || !mkev(&start) || !mkev(&fin))
        rc = DASH_ERR_CUDA;
    for (int i = 0; rc == DASH_OK && i < ns; ++i)
        if (cudaStreamCreateWithFlags(&sc[i], cudaStreamNonBlocking) != cudaSuccess) rc = DASH_ERR_CUDA;
    for (int i = 0; rc == DASH_OK && i < 2 * nu; ++i)
        if (!mkev(&ev[i])) rc = DASH_ERR_CUDA;
    // the helper streams start after the work already queued on `stream`, which clears the
    // call's header first
    if (rc == DASH_OK && (cudaMemsetAsync(ws0, 0, sizeof(WsHeader), s) != cudaSuccess ||
                          cudaEventRecord(start, s) != cudaSuccess || cudaStreamWaitEvent(sin, start, 0) != cudaSuccess ||
                          cudaStreamWaitEvent(sout, start, 0) != cudaSuccess))
        rc = DASH_ERR_CUDA;
    for (int i = 0; rc == DASH_OK && i < ns; ++i)
        if (cudaStreamWaitEvent(sc[i], start, 0) != cudaSuccess) rc = DASH_ERR_CUDA;
    for (int u = 0; rc == DASH_OK && u < nu; ++u) {
        const int gi = u / nch, c = u % nch, h0 = c * gc, hc = std::min(gc, G - h0);
        const size_t ok = (size_t)gi * kg, oq = (size_t)gi * qg + (size_t)h0 * hb, nq = (size_t)hc * hb;
        cudaStream_t cs = sc[u % ns];                                 // units on one stream share a slice
        char* const wsi = unit_ws(u % ns);
        // copies in are in order on `sin`: a unit's event also covers its group's keys and values
        if ((c == 0 && (!cp(atw(k_dev, ok), at(k_host, ok), kg, cudaMemcpyHostToDevice, sin) ||
                        !cp(atw(v_dev, ok), at(v_host, ok), kg, cudaMemcpyHostToDevice, sin))) ||
            !cp(atw(q_dev, oq), at(q_host, oq), nq, cudaMemcpyHostToDevice, sin) ||
            cudaEventRecord(ev[2 * u], sin) != cudaSuccess || cudaStreamWaitEvent(cs, ev[2 * u], 0) != cudaSuccess) {
            rc = DASH_ERR_CUDA;
            break;
        }
        rc = dash_prefill(atw(q_dev, oq), atw(k_dev, ok), atw(v_dev, ok), atw(out_dev, oq), 1, hc, 1, T, d, block,
                          alpha, coarse_scale, wsi, wsu, reinterpret_cast<dash_stream_t>(cs));
        if (rc != DASH_OK) break;
        accumulate_header_kernel<<<1, 32, 0, cs>>>(reinterpret_cast<WsHeader*>(ws0), reinterpret_cast<const WsHeader*>(wsi));
        if (cudaGetLastError() != cudaSuccess || cudaEventRecord(ev[2 * u + 1], cs) != cudaSuccess ||
            cudaStreamWaitEvent(sout, ev[2 * u + 1], 0) != cudaSuccess ||
            !cp(atw(out_host, oq), at(out_dev, oq), nq, cudaMemcpyDeviceToHost, sout))
            rc = DASH_ERR_CUDA;
    }
    // `stream` waits for everything issued on the helper streams, also after an error (each
    // compute stream's work precedes a copy out it ordered, or is joined here)
    if (sout && fin && cudaEventRecord(fin, sout) == cudaSuccess) cudaStreamWaitEvent(s, fin, 0);
    if (sin && start && cudaEventRecord(start, sin) == cudaSuccess) cudaStreamWaitEvent(s, start, 0);
    for (int i = 0; i < ns; ++i)
        if (sc[i] && start && cudaEventRecord(start, sc[i]) == cudaSuccess) cudaStreamWaitEvent(s, start, 0);
    // destroying a stream or event with work pending releases it once the work completes
    for (int i = 0; ev && i < 2 * nu; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    delete[] ev;
    if (start) cudaEventDestroy(start);
    if (fin) cudaEventDestroy(fin);
    if (sin) cudaStreamDestroy(sin);
    if (sout) cudaStreamDestroy(sout);
    for (int i = 0; i < ns; ++i)
        if (sc[i]) cudaStreamDestroy(sc[i]);
    return rc;
}

int dash_prefill_stats(const void* workspace, size_t ws_bytes, dash_stats* out, dash_stream_t stream) {
    return read_stats(workspace, ws_bytes, out, stream);
}

int dash_decode_stats(const void* workspace, size_t ws_bytes, dash_stats* out, dash_stream_t stream) {
    return read_stats(workspace, ws_bytes, out, stream);
}

int dash_prefill_tau(const void* workspace, size_t ws_bytes, float* tau_out, int B, int Hq, int Hkv,
                     int T, int d, int block, dash_stream_t stream) {
    if (!workspace || !tau_out) return DASH_ERR_ARG;
    PrefillGeom g;
    if (block != kBlock || !make_prefill_geom(B, Hq, Hkv, T, d, &g)) return DASH_ERR_SHAPE;
    if (ws_bytes < g.total) return DASH_ERR_WORKSPACE;
    const char* ws = static_cast<const char*>(workspace);
    return cudaMemcpyAsync(tau_out, ws + g.off_tau, (size_t)B * Hq * T * sizeof(float),
                           cudaMemcpyDeviceToDevice, S(stream)) == cudaSuccess ? DASH_OK : DASH_ERR_CUDA;
}

int dash_select_dump(const void* q, const float* ksum, const long long* rows, int nrows, int max_sel,
                     int* out_idx, float* out_p, int* out_count, float* out_tau, int B, int Hq, int Hkv,
                     int T, int d, int block, float alpha, float coarse_scale, dash_stream_t stream) {
    if (nrows < 0 || max_sel < 0) return DASH_ERR_ARG;
    if (nrows > 0 && (!q || !ksum || !rows || !out_count || !out_tau || !al16(q))) return DASH_ERR_ARG;
    if (nrows > 0 && max_sel > 0 && (!out_idx || !out_p)) return DASH_ERR_ARG;
    if (!good_params(alpha, coarse_scale)) return DASH_ERR_ARG;
    PrefillGeom g;
    if (block != kBlock || !make_prefill_geom(B, Hq, Hkv, T, d, &g)) return DASH_ERR_SHAPE;
    return launch_select_dump(q, ksum, rows, nrows, max_sel, out_idx, out_p, out_count, out_tau, B, Hq,
                              Hkv, T, d, alpha, coarse_scale, S(stream)) == cudaSuccess
               ? DASH_OK : DASH_ERR_CUDA;
}

size_t dash_decode_workspace_size(int B, int Hq, int Hkv, int Tmax, int d, int block) {
    DecodeGeom g;
    if (block != kBlock || !make_decode_geom(B, Hq, Hkv, Tmax, d, &g)) return 0;
    return g.total;
}

static int decode_impl(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                       const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d, int block,
                       float alpha, float coarse_scale, void* workspace, size_t ws_bytes,
                       dash_stream_t stream, void* const* events, unsigned flags = 0,
                       float* x_dump = nullptr, float* p_dump = nullptr, float* tau_dump = nullptr) {
    if (!q || !k_cache || !v_cache || !ksum || !kv_len || !out) return DASH_ERR_ARG;
    if (!al16(q) || !al16(k_cache) || !al16(v_cache) || !al16(ksum) || !al16(out)) return DASH_ERR_ARG;
    if (!good_params(alpha, coarse_scale)) return DASH_ERR_ARG;
    DecodeGeom g;
    if (block != kBlock || !make_decode_geom(B, Hq, Hkv, Tmax, d, &g)) return DASH_ERR_SHAPE;
    if (flags & ~(unsigned)DASH_HEAD_AGGREGATION) return DASH_ERR_ARG;
    const int agg = (flags & DASH_HEAD_AGGREGATION) ? 1 : 0;
    if ((agg || x_dump) && !decode_tc_supported(g)) return DASH_ERR_UNSUPPORTED;
    if (!workspace || !al256(workspace) || ws_bytes < g.total) return DASH_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    cudaStream_t s = S(stream);
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), s) != cudaSuccess) return DASH_ERR_CUDA;
    if (x_dump && launch_dump_fill(x_dump, p_dump, (size_t)B * Hq * g.nbs, s) != cudaSuccess) return DASH_ERR_CUDA;
    if (launch_decode(q, k_cache, v_cache, ksum, kv_len, out, g, ws, alpha, coarse_scale, s,
                      reinterpret_cast<cudaEvent_t const*>(events), agg, x_dump, p_dump) != cudaSuccess)
        return DASH_ERR_CUDA;
    if (tau_dump && cudaMemcpyAsync(tau_dump, ws + g.off_tau, (size_t)B * Hq * sizeof(float),
                                    cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return DASH_ERR_CUDA;
    return DASH_OK;
}

int dash_decode(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d, int block,
                float alpha, float coarse_scale, void* workspace, size_t ws_bytes, dash_stream_t stream) {
    return decode_impl(q, k_cache, v_cache, ksum, kv_len, out, B, Hq, Hkv, Tmax, d, block, alpha,
                       coarse_scale, workspace, ws_bytes, stream, nullptr);
}

int dash_decode_ex(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                   const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d, int block,
                   float alpha, float coarse_scale, unsigned flags, void* workspace, size_t ws_bytes,
                   dash_stream_t stream) {
    return decode_impl(q, k_cache, v_cache, ksum, kv_len, out, B, Hq, Hkv, Tmax, d, block, alpha,
                       coarse_scale, workspace, ws_bytes, stream, nullptr, flags);
}

int dash_decode_dump(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                     const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d, int block,
                     float alpha, float coarse_scale, unsigned flags, float* x_out, float* p_out, float* tau_out,
                     void* workspace, size_t ws_bytes, dash_stream_t stream) {
    if (!x_out || !p_out || !tau_out) return DASH_ERR_ARG;
    return decode_impl(q, k_cache, v_cache, ksum, kv_len, out, B, Hq, Hkv, Tmax, d, block, alpha,
                       coarse_scale, workspace, ws_bytes, stream, nullptr, flags, x_out, p_out, tau_out);
}

int dash_decode_profiled(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                         const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d, int block,
                         float alpha, float coarse_scale, void* workspace, size_t ws_bytes,
                         dash_stream_t stream, void* const* events) {
    if (!events) return DASH_ERR_ARG;
    return decode_impl(q, k_cache, v_cache, ksum, kv_len, out, B, Hq, Hkv, Tmax, d, block, alpha,
                       coarse_scale, workspace, ws_bytes, stream, events);
}

int dash_get_device_status(const void* workspace, dash_stream_t stream) {
    if (!workspace) return DASH_ERR_ARG;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return DASH_ERR_CUDA;
    int st = 0;
    if (cudaMemcpy(&st, workspace, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess) return DASH_ERR_CUDA;
    if (st & kStWaitTimeout) return DASH_ERR_DEVICE_TIMEOUT;
    return (st & kStNoConverge) ? DASH_ERR_NO_CONVERGE : DASH_OK;
}

}  // extern "C"
