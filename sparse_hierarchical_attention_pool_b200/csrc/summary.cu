// summary.cu -- Stage 0: block summaries (mean pooling of each complete 64-key block).
//
// "DashAttention and the year sparse attention became a field", section "What
// alpha-entmax changes": the chunk summary is a small learned attention head initialised
// at zero, i.e. uniform weights over the chunk's keys -- the arithmetic mean.
//
// One warp per (b, kv head, block): the block is 64 * d * 2 bytes contiguous in k.  Lane
// l reads 16-byte vectors (8 bf16) of column group l % (d/8) from rows l / (d/8), + 32/(d/8),
// ...; partial sums are combined with shuffles; fp32 accumulation throughout.  HBM-bound:
// bytes per block = 64 * d * 2 read + d * 4 written.
//
// The learned head (same section: the summary head is a small attention head, initialised
// at zero so that it starts as the mean) pools the block with one query vector w_g per KV
// head: kbar_j = sum_i softmax_i(w_g . k_i / sqrt(d)) k_i.  Its kernel first scores the
// block's keys (lane l takes keys l and l + 32), takes the softmax across the warp, then
// forms the weighted sum with the mean kernel's layout.
#include "common.cuh"
#include "kernels.h"

namespace dash {

template <int D>
__global__ void __launch_bounds__(256)
block_summary_kernel(const __nv_bfloat16* __restrict__ k, float* __restrict__ ksum,
                     __nv_bfloat16* __restrict__ khi, __nv_bfloat16* __restrict__ klo,
                     long long nblocks_total, int nbs, int T) {
    constexpr int CH = D / 8;          // 16-byte column groups per row
    constexpr int RPS = 32 / CH;       // rows covered by one warp-wide load
    constexpr int STEPS = kBlock / RPS;
    const int lane = threadIdx.x & 31;
    long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (wid >= nblocks_total) return;
    long long bg = wid / nbs;
    int j = (int)(wid % nbs);
    const int cg = lane % CH, r0 = lane / CH;
    const uint4* src = reinterpret_cast<const uint4*>(k + ((size_t)bg * T + (size_t)j * kBlock) * D);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    constexpr int BATCH = 8;           // loads in flight per lane
#pragma unroll
    for (int s0 = 0; s0 < STEPS; s0 += BATCH) {
        uint4 buf[BATCH];
#pragma unroll
        for (int s = 0; s < BATCH; ++s) buf[s] = __ldg(src + (size_t)(r0 + (s0 + s) * RPS) * CH + cg);
#pragma unroll
        for (int s = 0; s < BATCH; ++s) {
            float f[8];
            bf16x8_to_float(buf[s], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += f[i];
        }
    }
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    if (lane < CH) {
        const size_t o = ((size_t)bg * nbs + j) * D + lane * 8;
        float4* dst = reinterpret_cast<float4*>(ksum + o);
        const float s = 1.0f / kBlock;
        float mean[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mean[i] = acc[i] * s;
        dst[0] = make_float4(mean[0], mean[1], mean[2], mean[3]);
        dst[1] = make_float4(mean[4], mean[5], mean[6], mean[7]);
        if (khi) {
            // kbar = hi + lo with hi = bf16(kbar), lo = bf16(kbar - hi): 16 significant bits
            __align__(16) __nv_bfloat16 h[8], l[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                h[i] = __float2bfloat16_rn(mean[i]);
                l[i] = __float2bfloat16_rn(mean[i] - __bfloat162float(h[i]));
            }
            *reinterpret_cast<uint4*>(khi + o) = *reinterpret_cast<const uint4*>(h);
            *reinterpret_cast<uint4*>(klo + o) = *reinterpret_cast<const uint4*>(l);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(256)
block_summary_attn_kernel(const __nv_bfloat16* __restrict__ k, const float* __restrict__ w,
                          float* __restrict__ ksum, __nv_bfloat16* __restrict__ khi,
                          __nv_bfloat16* __restrict__ klo, long long nblocks_total, int nbs, int T, int Hkv) {
    constexpr int CH = D / 8;
    constexpr int RPS = 32 / CH;
    constexpr int STEPS = kBlock / RPS;
    __shared__ float a_sh[8][kBlock];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + wl;
    if (wid >= nblocks_total) return;
    const long long bg = wid / nbs;
    const int j = (int)(wid % nbs);
    const __nv_bfloat16* kb = k + ((size_t)bg * T + (size_t)j * kBlock) * D;
    const float4* wg = reinterpret_cast<const float4*>(w + (size_t)(bg % Hkv) * D);
    // scores of keys lane and lane + 32
    const float isd = 1.0f / sqrtf((float)D);
    float sc[2];
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        const uint4* row = reinterpret_cast<const uint4*>(kb + (size_t)(lane + 32 * kk) * D);
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            float f[8];
            bf16x8_to_float(__ldg(row + c), f);
            const float4 w0 = __ldg(wg + 2 * c), w1 = __ldg(wg + 2 * c + 1);
            acc = fmaf(w0.x, f[0], acc); acc = fmaf(w0.y, f[1], acc);
            acc = fmaf(w0.z, f[2], acc); acc = fmaf(w0.w, f[3], acc);
            acc = fmaf(w1.x, f[4], acc); acc = fmaf(w1.y, f[5], acc);
            acc = fmaf(w1.z, f[6], acc); acc = fmaf(w1.w, f[7], acc);
        }
        sc[kk] = acc * isd;
    }
    const float m = warp_max(fmaxf(sc[0], sc[1]));
    const float e0 = expf(sc[0] - m), e1 = expf(sc[1] - m);
    const float inv = 1.0f / warp_sum(e0 + e1);
    a_sh[wl][lane] = e0 * inv;
    a_sh[wl][lane + 32] = e1 * inv;
    __syncwarp();
    // weighted sum, lanes over 16-byte column groups as in the mean kernel
    const int cg = lane % CH, r0 = lane / CH;
    const uint4* src = reinterpret_cast<const uint4*>(kb);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    constexpr int BATCH = 8;
#pragma unroll
    for (int s0 = 0; s0 < STEPS; s0 += BATCH) {
        uint4 buf[BATCH];
#pragma unroll
        for (int s = 0; s < BATCH; ++s) buf[s] = __ldg(src + (size_t)(r0 + (s0 + s) * RPS) * CH + cg);
#pragma unroll
        for (int s = 0; s < BATCH; ++s) {
            float f[8];
            bf16x8_to_float(buf[s], f);
            const float a = a_sh[wl][r0 + (s0 + s) * RPS];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(a, f[i], acc[i]);
        }
    }
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    if (lane < CH) {
        const size_t o = ((size_t)bg * nbs + j) * D + lane * 8;
        float4* dst = reinterpret_cast<float4*>(ksum + o);
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        if (khi) {
            __align__(16) __nv_bfloat16 h[8], l[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                h[i] = __float2bfloat16_rn(acc[i]);
                l[i] = __float2bfloat16_rn(acc[i] - __bfloat162float(h[i]));
            }
            *reinterpret_cast<uint4*>(khi + o) = *reinterpret_cast<const uint4*>(h);
            *reinterpret_cast<uint4*>(klo + o) = *reinterpret_cast<const uint4*>(l);
        }
    }
}

cudaError_t launch_block_summary(const void* k, float* ksum, int B, int Hkv, int T, int d,
                                 cudaStream_t stream, void* khi, void* klo, const float* w) {
    int nbs = T / kBlock;
    long long total = (long long)B * Hkv * nbs;
    if (total == 0) return cudaSuccess;
    unsigned grid = (unsigned)((total + 7) / 8);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    auto* hi = static_cast<__nv_bfloat16*>(khi);
    auto* lo = static_cast<__nv_bfloat16*>(klo);
    if (w) {
        if (d == 128) block_summary_attn_kernel<128><<<grid, 256, 0, stream>>>(kb, w, ksum, hi, lo, total, nbs, T, Hkv);
        else block_summary_attn_kernel<64><<<grid, 256, 0, stream>>>(kb, w, ksum, hi, lo, total, nbs, T, Hkv);
    } else {
        if (d == 128) block_summary_kernel<128><<<grid, 256, 0, stream>>>(kb, ksum, hi, lo, total, nbs, T);
        else block_summary_kernel<64><<<grid, 256, 0, stream>>>(kb, ksum, hi, lo, total, nbs, T);
    }
    return cudaGetLastError();
}

}  // namespace dash
