// fine_mma.cu -- Stage 2 for prefill: prior-weighted softmax over each tile's listed blocks.
//
// "DashAttention: Making Sparse Attention Fully Differentiable with Adaptive Block
// Selection", section "Core Mechanism" (Stage 2: for each selected block, fine logits
// Q * K_block plus log(p_coarse), softmax, weighted sum of V) and section "Key Concepts"
// (hierarchical prior).  For row (b, h, t) with own block bt:
//     l_i = (q . k_i) / sqrt(d) + log p_j(i)   over tokens of blocks j < bt with p_j > 0,
//     l_i = (q . k_i) / sqrt(d)                over the own block, tokens i <= t,
//     o   = sum_i softmax(l)_i v_i.
// p_j = [x_j - tau]_+^(1/(alpha-1)) needs x_j = (alpha-1) cs (q . kbar_j)/sqrt(d); since
// q . kbar_j is the mean of q . k_i over the block's 64 keys, x_j is recovered from the row
// sums of the Q K^T tile this kernel computes anyway, and log p_j = log(x_j - tau)/(alpha-1)
// (no underflow for tiny weights).  A row whose x_j <= tau skips the block.
//
// One CTA per work tile (128 rows: P positions x G heads of one KV head), heaviest tiles
// first.  8 warps x 16 rows; bf16 mma.sync m16n8k16 with fp32 accumulators; K/V blocks
// streamed through a two-stage cp.async pipeline into XOR-swizzled shared memory; the
// gathered block serves all G heads of the group.  Online softmax in the log2 domain.
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace dash {

template <int D>
__global__ void __launch_bounds__(256, 1)
fine_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ out,
                const float* __restrict__ tau, const int* __restrict__ list,
                const int* __restrict__ count, PrefillGeom g, float cxm, float e_pow, float sm2) {
    constexpr int CH = D / 8;
    extern __shared__ uint4 smem_u4[];
    __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem_u4);   // [128][D]
    __nv_bfloat16* Ks = Qs + kTileRows * D;                          // [2][64][D]
    __nv_bfloat16* Vs = Ks + 2 * kBlock * D;                         // [2][64][D]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BH = g.B * g.Hkv;
    const int w = blockIdx.x;
    const int it = g.ntile_bg - 1 - w / BH;
    const int bg = w % BH;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int t0 = it * g.P;
    const int bt = t0 / kBlock;
    const size_t tile_id = (size_t)bg * g.ntile_bg + it;
    const int U = bt > 0 ? count[tile_id] : 0;
    const int nsteps = U + 1;                        // listed past blocks, then the own block
    const int* lst = list + tile_id * g.cap;
    const size_t kv_row0 = (size_t)bg * g.T;         // row of (b, kvh, token 0) in [B*Hkv*T, D]

    // ---- Q tile
    for (int idx = tid; idx < kTileRows * CH; idx += blockDim.x) {
        const int r = idx / CH, c = idx % CH;
        const int hl = r / g.P, t = t0 + r % g.P;
        const bool ok = r < g.M && t < g.T;
        const __nv_bfloat16* src = ok ? q + ((size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t) * D + c * 8 : q;
        cp_async16(Qs + swz<D>(r, c), src, ok ? 16 : 0);
    }
    auto load_kv = [&](int s, int stage) {
        const int j = s < U ? lst[s] : bt;
        for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
            const int r = idx / CH, c = idx % CH;
            const int tok = j * kBlock + r;
            const bool ok = tok < g.T;
            const size_t off = (kv_row0 + (ok ? tok : 0)) * D + c * 8;
            cp_async16(Ks + stage * kBlock * D + swz<D>(r, c), k + off, ok ? 16 : 0);
            cp_async16(Vs + stage * kBlock * D + swz<D>(r, c), v + off, ok ? 16 : 0);
        }
    };
    load_kv(0, 0);
    cp_async_commit();

    // ---- per-thread rows: g4 and g4 + 8 of this warp's 16
    const int g4 = lane >> 2, t4 = lane & 3;
    float tau_r[2];
    int tpos[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = warp * 16 + g4 + 8 * i;
        const int hl = r / g.P, t = t0 + r % g.P;
        const bool ok = r < g.M && t < g.T;
        tpos[i] = ok ? t : -1;
        tau_r[i] = (ok && bt > 0) ? tau[(size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t] : INFINITY;
    }
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
    float o[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[n][c] = 0.f;
    uint32_t qf[D / 16][4];

    for (int s = 0; s < nsteps; ++s) {
        const int stage = s & 1;
        const int j = s < U ? lst[s] : bt;
        const bool diag = (j == bt);
        if (s + 1 < nsteps) load_kv(s + 1, stage ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (s == 0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                ldsm_x4(qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3],
                        smem_u32(Qs + swz<D>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4))));
        }
        const __nv_bfloat16* Kst = Ks + stage * kBlock * D;
        const __nv_bfloat16* Vst = Vs + stage * kBlock * D;

        // S = Q K^T (16 rows x 64 keys per warp)
        float sacc[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) sacc[n][c] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b0, b1, b2, b3;
                const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int ch = kk * 2 + ((lane >> 3) & 1);
                ldsm_x4(b0, b1, b2, b3, smem_u32(Kst + swz<D>(key, ch)));
                mma_bf16(sacc[2 * np], qf[kk], b0, b1);
                mma_bf16(sacc[2 * np + 1], qf[kk], b2, b3);
            }
        }
        // block weight of each row: x_j from the row sum of S, log2 p_j = e log2(x_j - tau)
        float lp2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float rs = 0.f;
#pragma unroll
            for (int n = 0; n < 8; ++n) rs += sacc[n][2 * i] + sacc[n][2 * i + 1];
            rs += __shfl_xor_sync(0xffffffffu, rs, 1);
            rs += __shfl_xor_sync(0xffffffffu, rs, 2);
            const float x = rs * cxm;
            lp2[i] = diag ? (tpos[i] >= 0 ? 0.f : -INFINITY)
                          : (x > tau_r[i] ? e_pow * __log2f(x - tau_r[i]) : -INFINITY);
        }
        const bool active = (lp2[0] > -INFINITY) || (lp2[1] > -INFINITY);
        if (__any_sync(0xffffffffu, active)) {
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = c >> 1;
                    float l2 = fmaf(sacc[n][c], sm2, lp2[i]);
                    if (diag) {
                        const int key = j * kBlock + n * 8 + 2 * t4 + (c & 1);
                        if (key > tpos[i]) l2 = -INFINITY;
                    }
                    sacc[n][c] = l2;
                    mx[i] = fmaxf(mx[i], l2);
                }
            float scale[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
                mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
                const float m_new = fmaxf(m_r[i], mx[i]);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                scale[i] = exp2f(m_r[i] - m_use);
                m_r[i] = m_new;
                mx[i] = m_use;
            }
            float ls[2] = {0.f, 0.f};
            uint32_t pa[4][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const float p0 = exp2f(sacc[n][0] - mx[0]);
                const float p1 = exp2f(sacc[n][1] - mx[0]);
                const float p2 = exp2f(sacc[n][2] - mx[1]);
                const float p3 = exp2f(sacc[n][3] - mx[1]);
                ls[0] += p0 + p1;
                ls[1] += p2 + p3;
                pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16(p0, p1);
                pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16(p2, p3);
            }
            l_r[0] = l_r[0] * scale[0] + ls[0];
            l_r[1] = l_r[1] * scale[1] + ls[1];
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                o[n][0] *= scale[0]; o[n][1] *= scale[0];
                o[n][2] *= scale[1]; o[n][3] *= scale[1];
            }
            // O += P V
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int dp = 0; dp < D / 16; ++dp) {
                    uint32_t b0, b1, b2, b3;
                    const int key = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int ch = dp * 2 + (lane >> 4);
                    ldsm_x4_t(b0, b1, b2, b3, smem_u32(Vst + swz<D>(key, ch)));
                    mma_bf16(o[2 * dp], pa[kk], b0, b1);
                    mma_bf16(o[2 * dp + 1], pa[kk], b2, b3);
                }
            }
        }
        __syncthreads();
    }

    // ---- epilogue: normalise and store the valid rows
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float l = l_r[i];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int r = warp * 16 + g4 + 8 * i;
        if (tpos[i] < 0) continue;
        const int hl = r / g.P;
        const float inv = 1.0f / l;
        __nv_bfloat16* dst = out + ((size_t)(b * g.Hq + kvh * g.G + hl) * g.T + tpos[i]) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            __nv_bfloat162 h = __floats2bfloat162_rn(o[n][2 * i] * inv, o[n][2 * i + 1] * inv);
            *reinterpret_cast<__nv_bfloat162*>(dst + n * 8 + 2 * t4) = h;
        }
    }
}

// Which Stage-2 kernel runs: the tcgen05 kernel wherever it supports the shape, unless
// DASH_FINE_KERNEL=mma selects the mma.sync kernel (kept for comparison and for groups of
// more than 16 query heads per KV head).
static bool use_mma_kernel() {
    static const int choice = [] {
        const char* e = getenv("DASH_FINE_KERNEL");
        return (e && strcmp(e, "mma") == 0) ? 1 : 0;
    }();
    return choice == 1;
}

cudaError_t launch_fine(const void* q, const void* k, const void* v, void* out,
                        const PrefillGeom& g, char* ws, float alpha, float coarse_scale,
                        cudaStream_t stream, int agg, bool need_tc) {
    if ((need_tc || !use_mma_kernel()) && fine_tc_supported(g))
        return launch_fine_tc(q, k, v, out, g, ws, alpha, coarse_scale, stream, agg);
    if (need_tc) return cudaErrorNotSupported;
    const float cxm = (alpha - 1.0f) * coarse_scale / sqrtf((float)g.d) / (float)kBlock;
    const float e_pow = 1.0f / (alpha - 1.0f);
    const float sm2 = 1.4426950408889634f / sqrtf((float)g.d);
    const float* tau = reinterpret_cast<const float*>(ws + g.off_tau);
    const int* list = reinterpret_cast<const int*>(ws + g.off_list);
    const int* count = reinterpret_cast<const int*>(ws + g.off_count);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const auto* vb = static_cast<const __nv_bfloat16*>(v);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    const size_t sm = (size_t)(kTileRows + 4 * kBlock) * g.d * sizeof(__nv_bfloat16);
    if (g.d == 128) {
        cudaError_t e = cudaFuncSetAttribute(fine_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        fine_mma_kernel<128><<<g.ntiles, 256, sm, stream>>>(qb, kb, vb, ob, tau, list, count, g, cxm, e_pow, sm2);
    } else {
        cudaError_t e = cudaFuncSetAttribute(fine_mma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        fine_mma_kernel<64><<<g.ntiles, 256, sm, stream>>>(qb, kb, vb, ob, tau, list, count, g, cxm, e_pow, sm2);
    }
    return cudaGetLastError();
}

}  // namespace dash
