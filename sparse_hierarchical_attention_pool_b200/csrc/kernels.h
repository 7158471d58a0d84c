// kernels.h -- host-side launchers of the DashAttention kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace dash {

// kbar in fp32, and optionally split into bf16 hi + lo parts for the tensor-core scores;
// w (fp32 [Hkv, d], device) selects the learned attention-pooling head, nullptr the mean
cudaError_t launch_block_summary(const void* k, float* ksum, int B, int Hkv, int T, int d,
                                 cudaStream_t stream, void* khi = nullptr, void* klo = nullptr,
                                 const float* w = nullptr);

// Stage 1 for prefill: scores of every work tile against the block summaries, per-row
// thresholds and the per-tile union of selected blocks.
cudaError_t launch_coarse(const void* q, const PrefillGeom& g, char* ws, float alpha,
                          float coarse_scale, cudaStream_t stream);

// tcgen05 variant of launch_coarse (needs P >= 8 and at least one complete block);
// write_rowbits: also store every row's selection bitmap (for the selection-ordered tiles)
bool coarse_tc_supported(const PrefillGeom& g);
cudaError_t launch_coarse_tc(const void* q, const PrefillGeom& g, char* ws, float alpha,
                             float coarse_scale, cudaStream_t stream, bool write_rowbits = false);

// Selection-ordered tiles from the per-row bitmaps of the coarse stage: sorts the rows of
// every window of a KV group by their signature and writes each ordered tile's rows, block
// list (selected and own blocks, ascending) and count; adds the tiles' unions to the header.
cudaError_t launch_order_tiles(const PrefillGeom& g, char* ws, cudaStream_t stream);

// Parity dump of the tensor-core fine kernel: rows with slot[row] >= 0 (row = (b Hq + h) T + t)
// get x_j and the applied weight p_j of every listed past block j at x[slot nbs + j],
// p[slot nbs + j].
struct FineDump {
    const int* slot;
    float* x;
    float* p;
};

// Stage 2 for prefill: prior-weighted softmax attention over each tile's listed blocks.
// agg: head-aggregated prior; need_tc: the tensor-core kernel is required (head aggregation
// or a learned summary head), whatever DASH_FINE_KERNEL says.
cudaError_t launch_fine(const void* q, const void* k, const void* v, void* out,
                        const PrefillGeom& g, char* ws, float alpha, float coarse_scale,
                        cudaStream_t stream, int agg = 0, bool need_tc = false);

// tcgen05 variant of launch_fine (needs P >= 8, i.e. at most 16 query heads per KV head);
// dump != nullptr selects the dump variant; ordered: run the selection-ordered tiles of
// launch_order_tiles instead of the position tiles (not with head aggregation)
bool fine_tc_supported(const PrefillGeom& g);
cudaError_t launch_fine_tc(const void* q, const void* k, const void* v, void* out,
                           const PrefillGeom& g, char* ws, float alpha, float coarse_scale,
                           cudaStream_t stream, int agg = 0, const FineDump* dump = nullptr,
                           bool ordered = false);

// x = NaN and p = 0 for n entries (the "not listed" marks of the parity dumps)
cudaError_t launch_dump_fill(float* x, float* p, size_t n, cudaStream_t stream);

// Gradients of the prefill (dq, dk, dv) after the coarse stage has filled the workspace
cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out,
                            const void* dout, void* dq, void* dk, void* dv, const PrefillGeom& g,
                            const BwdGeom& bw, char* ws, float alpha, float coarse_scale,
                            cudaStream_t stream);

// tcgen05 variant of the backward's query-major half (statistics, then dq); needs P >= 8
cudaError_t launch_bwd_dq_tc(const void* q, const void* k, const void* v, const void* dout, void* dq,
                             const PrefillGeom& g, const BwdGeom& bw, char* ws, float alpha, float coarse_scale,
                             cudaStream_t stream);

// tcgen05 variant of the backward's key-major half (dk, dv over pairs of key blocks)
cudaError_t launch_bwd_dkv_tc(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                              const PrefillGeom& g, const BwdGeom& bw, char* ws, float alpha, float coarse_scale,
                              cudaStream_t stream);

cudaError_t launch_select_dump(const void* q, const float* ksum, const long long* rows, int nrows,
                               int max_sel, int* out_idx, float* out_p, int* out_count,
                               float* out_tau, int B, int Hq, int Hkv, int T, int d, float alpha,
                               float coarse_scale, cudaStream_t stream);

// split-KV attention of a decode step on TMA + mma.sync, balanced over the CTAs (at most 8
// heads per group); decode_tc_ctas() is the grid it is launched with
bool decode_tc_supported(const DecodeGeom& g);
int decode_tc_ctas();
// x_dump / p_dump (both or neither, fp32 [B Hq, Tmax / 64]): the parity dump of each head's
// listed blocks
cudaError_t launch_decode_attn_tc(const void* q, const void* kc, const void* vc, const int* kv_len,
                                  void* out, const DecodeGeom& g, char* ws, float e_pow, float sm2,
                                  int nctas, cudaStream_t stream, int agg = 0, float* x_dump = nullptr,
                                  float* p_dump = nullptr);
// agg: head-aggregated prior (needs decode_tc_supported); x_dump / p_dump as above (needs
// decode_tc_supported)
cudaError_t launch_decode(const void* q, const void* kc, const void* vc, const float* ksum,
                          const int* kv_len, void* out, const DecodeGeom& g, char* ws,
                          float alpha, float coarse_scale, cudaStream_t stream,
                          const cudaEvent_t* events, int agg = 0, float* x_dump = nullptr,
                          float* p_dump = nullptr);

}  // namespace dash
