// coarse.cu -- Stage 1 for prefill: coarse scores, alpha-entmax thresholds, block lists.
//
// "DashAttention: Making Sparse Attention Fully Differentiable with Adaptive Block
// Selection", section "Core Mechanism" (Stage 1: coarse scores Q * block_summary, then
// alpha-entmax gives sparse block weights).  Per query row (b, h, t) with own block
// bt = t / 64, the scored blocks are j < bt and
//     x_j = (alpha - 1) * coarse_scale * (q . kbar_j) / sqrt(d).
//
// Work tile = P positions inside one key block x the G query heads of one KV head (128
// rows), so every row of a tile has the same bt.  A persistent CTA per tile:
//   1. x = Q_tile . Kbar^T in fp32 on the CUDA cores (register-blocked 8 rows x 4 blocks per
//      thread, operands staged in shared memory), written to a per-CTA scratch slab laid
//      out [block][row] so that a warp reading one block for 32 rows is one 128-byte line;
//   2. one thread per row solves for tau (entmax.cuh) reading its column of the slab;
//   3. every (row, block) with x_j > tau marks the block in a shared bitmap (warp ballots),
//      and warp 0 compacts the bitmap into the tile's ascending block list.
// Outputs: tau[b, h, t] (workspace), list[tile][0..U), count[tile], stats counters.
#include "common.cuh"
#include "entmax.cuh"
#include "kernels.h"

namespace dash {

struct SlabCol {
    const float* p;
    __device__ __forceinline__ float operator()(int j) const { return p[(size_t)j * kTileRows]; }
};

template <int D>
__global__ void __launch_bounds__(256)
coarse_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ ksum,
              float* __restrict__ tau_out, int* __restrict__ list, int* __restrict__ count,
              float* __restrict__ scratch, WsHeader* __restrict__ hdr, PrefillGeom g,
              float alpha, float cx) {
    extern __shared__ float4 smem_f4[];
    float* Qs = reinterpret_cast<float*>(smem_f4);     // [D][128]
    float* Ks = Qs + D * kTileRows;                    // [D][64]
    __shared__ unsigned bitmap[kMaxT / kBlock / 32];
    __shared__ unsigned long long red_sel;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BH = g.B * g.Hkv;
    float* slab = scratch + (size_t)blockIdx.x * kTileRows * g.cap;
    int no_conv = 0;

    for (int w = blockIdx.x; w < g.ntiles; w += gridDim.x) {
        const int it = g.ntile_bg - 1 - w / BH;
        const int bg = w % BH;
        const int b = bg / g.Hkv, kvh = bg % g.Hkv;
        const int t0 = it * g.P;
        const int bt = t0 / kBlock;
        const size_t tile_id = (size_t)bg * g.ntile_bg + it;
        if (bt == 0) {
            // no past blocks: own-block attention only; threshold unused
            for (int r = tid; r < g.M; r += blockDim.x) {
                int hl = r / g.P, t = t0 + r % g.P;
                if (t < g.T) tau_out[((size_t)(b * g.Hq + kvh * g.G + hl)) * g.T + t] = __int_as_float(0x7fc00000);
            }
            if (tid == 0) {
                count[tile_id] = 0;
                atomicAdd(&hdr->fine_steps, 1ull);            // the own block alone
            }
            continue;
        }
        // ---- Q tile -> shared, transposed to [d][row], fp32
        for (int idx = tid; idx < kTileRows * (D / 8); idx += blockDim.x) {
            const int r = idx % kTileRows, c8 = idx / kTileRows;
            const int hl = r / g.P, t = t0 + r % g.P;
            float f[8];
            if (r < g.M && t < g.T) {
                uint4 u = __ldg(reinterpret_cast<const uint4*>(
                    q + ((size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t) * D + c8 * 8));
                bf16x8_to_float(u, f);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) Qs[(c8 * 8 + i) * kTileRows + r] = f[i];
        }
        const int nw = (bt + 31) / 32;
        for (int i = tid; i < nw; i += blockDim.x) bitmap[i] = 0u;
        if (tid == 0) red_sel = 0ull;
        __syncthreads();

        // ---- scores, 64 blocks per chunk
        const int ty = tid / 16, tx = tid % 16;
        const float* kb = ksum + (size_t)bg * g.nbs * D;
        for (int c0 = 0; c0 < bt; c0 += 64) {
            const int nj = min(64, bt - c0);
            for (int idx = tid; idx < 64 * (D / 4); idx += blockDim.x) {
                const int jj = idx % 64, k4 = idx / 64;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (jj < nj) v = __ldg(reinterpret_cast<const float4*>(kb + (size_t)(c0 + jj) * D) + k4);
                Ks[(k4 * 4 + 0) * 64 + jj] = v.x;
                Ks[(k4 * 4 + 1) * 64 + jj] = v.y;
                Ks[(k4 * 4 + 2) * 64 + jj] = v.z;
                Ks[(k4 * 4 + 3) * 64 + jj] = v.w;
            }
            __syncthreads();
            float acc[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) acc[i][jj] = 0.f;
#pragma unroll 4
            for (int kk = 0; kk < D; ++kk) {
                const float4 a0 = *reinterpret_cast<const float4*>(Qs + kk * kTileRows + ty * 8);
                const float4 a1 = *reinterpret_cast<const float4*>(Qs + kk * kTileRows + ty * 8 + 4);
                const float4 bq = *reinterpret_cast<const float4*>(Ks + kk * 64 + tx * 4);
                const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a[i], bb[jj], acc[i][jj]);
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = c0 + tx * 4 + jj;
                if (j < bt) {
                    float4* dst = reinterpret_cast<float4*>(slab + (size_t)j * kTileRows + ty * 8);
                    dst[0] = make_float4(acc[0][jj] * cx, acc[1][jj] * cx, acc[2][jj] * cx, acc[3][jj] * cx);
                    dst[1] = make_float4(acc[4][jj] * cx, acc[5][jj] * cx, acc[6][jj] * cx, acc[7][jj] * cx);
                }
            }
            __syncthreads();
        }

        // ---- thresholds (one thread per row) and block union (warps 0..3)
        if (tid < kTileRows) {
            const int r = tid, hl = r / g.P, t = t0 + r % g.P;
            const bool valid = r < g.M && t < g.T;
            float tau = INFINITY;
            if (valid) tau = entmax_threshold<false>(SlabCol{slab + r}, bt, alpha, &no_conv, g.maxit);
            if (valid) tau_out[((size_t)(b * g.Hq + kvh * g.G + hl)) * g.T + t] = tau;
            unsigned nsel = 0;
            for (int j = 0; j < bt; ++j) {
                const bool f = valid && slab[(size_t)j * kTileRows + r] > tau;
                nsel += f;
                const unsigned bal = __ballot_sync(0xffffffffu, f);
                if (lane == 0 && bal) atomicOr(&bitmap[j >> 5], 1u << (j & 31));
            }
            const float s = warp_sum((float)nsel);
            if (lane == 0) atomicAdd(&red_sel, (unsigned long long)s);
        }
        __syncthreads();
        if (warp == 0) {
            int base = 0;
            int* dst = list + tile_id * g.cap;
            for (int w0 = 0; w0 < nw; w0 += 32) {
                const int wi = w0 + lane;
                unsigned word = wi < nw ? bitmap[wi] : 0u;
                const int pc = __popc(word);
                int incl = pc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    int n = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += n;
                }
                int pos = base + incl - pc;
                while (word) {
                    const int bit = __ffs(word) - 1;
                    dst[pos++] = wi * 32 + bit;
                    word &= word - 1;
                }
                base += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) {
                count[tile_id] = base;
                const int rows_valid = g.G * min(g.P, g.T - t0);
                atomicAdd(&hdr->selected_pairs, red_sel);
                atomicAdd(&hdr->scored_pairs, (unsigned long long)rows_valid * bt);
                atomicAdd(&hdr->union_blocks, (unsigned long long)base);
                atomicAdd(&hdr->tiles, 1ull);
                atomicAdd(&hdr->fine_steps, (unsigned long long)base + 1ull);
            }
        }
        __syncthreads();
    }
    if (no_conv) atomicOr(&hdr->status, kStNoConverge);
}

cudaError_t launch_coarse(const void* q, const PrefillGeom& g, char* ws, float alpha,
                          float coarse_scale, cudaStream_t stream) {
    const float cx = (alpha - 1.0f) * coarse_scale / sqrtf((float)g.d);
    const int grid = g.ntiles < kCoarseCTAs ? g.ntiles : kCoarseCTAs;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    float* ksum = reinterpret_cast<float*>(ws + g.off_ksum);
    float* tau = reinterpret_cast<float*>(ws + g.off_tau);
    int* list = reinterpret_cast<int*>(ws + g.off_list);
    int* count = reinterpret_cast<int*>(ws + g.off_count);
    float* scratch = reinterpret_cast<float*>(ws + g.off_scratch);
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
    if (g.d == 128) {
        const size_t sm = (size_t)(128 * kTileRows + 128 * 64) * sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(coarse_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        coarse_kernel<128><<<grid, 256, sm, stream>>>(qb, ksum, tau, list, count, scratch, hdr, g, alpha, cx);
    } else {
        const size_t sm = (size_t)(64 * kTileRows + 64 * 64) * sizeof(float);
        cudaError_t e = cudaFuncSetAttribute(coarse_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        coarse_kernel<64><<<grid, 256, sm, stream>>>(qb, ksum, tau, list, count, scratch, hdr, g, alpha, cx);
    }
    return cudaGetLastError();
}

}  // namespace dash
