// backward.cu -- gradients of the causal prefill: dq, dk, dv of a scalar loss whose
// gradient with respect to the output is dout.
//
// "DashAttention: Making Sparse Attention Fully Differentiable with Adaptive Block
// Selection", sections "Core Mechanism" and "Key Concepts": every step of the forward is
// differentiable -- the fine softmax, the log prior log p_j, alpha-entmax over the coarse
// scores and the mean-pooled summaries -- so gradients reach the block selection.  For row
// (b, h, t) with fine probabilities P_i, output o and own block bt:
//     D      = dout . o
//     dl_i   = P_i (dout . v_i - D)                          (softmax backward)
//     dv_i  += P_i dout,   dq += dl_i k_i / sqrt(d),   dk_i += dl_i q / sqrt(d)
//     c_j    = sum over the keys i of block j of dl_i        (d loss / d log p_j, j < bt)
//   on the support (x_j > tau), with g_j = p_j^(2-alpha) = (x_j - tau)^((2-alpha)/(alpha-1))
//   (the alpha-entmax Jacobian diag(g) - g g^T / sum g, applied to d loss / d p_j = c_j / p_j):
//     H_j    = c_j / (x_j - tau),   r = sum_j H_j / sum_j g_j,   ds_j = H_j - r g_j
//     dq    += cs ds_j kbar_j / sqrt(d),   dkbar_j += cs ds_j q / sqrt(d),   dk_i += dkbar_j / 64.
// kbar_j is the mean of block j's keys, so both summary terms fold into the fine products:
// adding cs ds_j / 64 to dl_i for the 64 keys of block j turns dS K into the dq update and
// dS^T Q into the dk update.  The own block has prior 1 and no coarse term.
//
// Kernels, after the coarse stage of the forward (summaries, thresholds, tile lists):
//   bwd_rowdot_kernel  D per row (every path).
// then, where a work tile holds at least 8 positions, the tcgen05 kernels of
// backward_tc.cu (statistics, dq, dk/dv); otherwise (more than 16 query heads per KV head,
// or DASH_BWD_KERNEL=mma) the two mma.sync kernels below:
//   bwd_dq_kernel      one CTA per work tile (query-major).  Pass 1 over the tile's steps
//                      (listed blocks, then the own block) gives each row's log-sum-exp,
//                      sum_j g_j and sum_j g_j kbar_j; pass 2 gives P, dS, c_j and H_j and
//                      accumulates dq with the folded cs H_j / 64; the -cs r sum_j g_j kbar_j
//                      part is applied at the end, when r is known.  Writes dq and, per row,
//                      the log-sum-exp and r.
//   bwd_dkv_kernel     one CTA per (b, KV head, key block j) (key-major): the tiles whose own
//                      block is j, then the tiles whose list holds j.  Recomputes P and dS
//                      per tile, folds cs ds_j / 64 into dS, and accumulates dk and dv of the
//                      block's 64 keys.  Every key belongs to one CTA: no atomics, and the
//                      result does not depend on the schedule.
// x_j is recovered, as in the forward's CUDA-core kernel, from the row sum of the tile's
// Q K^T scores (q . kbar_j is the mean of q . k_i over the block).  bf16 mma.sync m16n8k16
// with fp32 accumulators; K/V (query-major) or Q/dout (key-major) tiles stream through a
// two-stage cp.async ring in XOR-swizzled shared memory.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace dash {

struct BwdConsts {
    float cxm;     // (alpha-1) cs / sqrt(d) / 64: row sum of q.k_i over a block -> x_j
    float e_pow;   // 1 / (alpha-1)
    float gpow;    // (2-alpha) / (alpha-1): g_j = (x_j - tau)^gpow
    float sm2;     // log2(e) / sqrt(d)
    float cs64;    // cs / 64
    float cs;      // coarse_scale
    float isd;     // 1 / sqrt(d)
};

// ------------------------------------------------------------------ D = dout . out per row
__global__ void bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ dout,
                                  const __nv_bfloat16* __restrict__ out, float* __restrict__ drow,
                                  long long nrows, int d) {
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= nrows) return;                       // whole warps leave together
    const __nv_bfloat16* a = dout + row * d;
    const __nv_bfloat16* o = out + row * d;
    float s = 0.f;
    for (int c = lane * 2; c < d; c += 64) {
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(a + c));
        const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o + c));
        s = fmaf(x.x, y.x, fmaf(x.y, y.y, s));
    }
    s = warp_sum(s);
    if (lane == 0) drow[row] = s;
}

// ------------------------------------------------------------------ query-major: dq
template <int D>
__global__ void __launch_bounds__(256, 1)
bwd_dq_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
              const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
              const float* __restrict__ drow, const float* __restrict__ tau,
              const int* __restrict__ list, const int* __restrict__ count,
              const float* __restrict__ ksum, __nv_bfloat16* __restrict__ dq,
              float* __restrict__ lse_out, float* __restrict__ r_out, PrefillGeom g, BwdConsts C) {
    constexpr int CH = D / 8;
    extern __shared__ uint4 smem_u4[];
    __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem_u4);   // [128][D]
    __nv_bfloat16* Gs = Qs + kTileRows * D;                          // dout tile [128][D]
    __nv_bfloat16* Ks = Gs + kTileRows * D;                          // [2][64][D]
    __nv_bfloat16* Vs = Ks + 2 * kBlock * D;                         // [2][64][D]
    float* GK = reinterpret_cast<float*>(Vs + 2 * kBlock * D);       // sum_j g_j kbar_j [128][D]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BH = g.B * g.Hkv;
    const int w = blockIdx.x;
    const int it = g.ntile_bg - 1 - w / BH;           // heaviest tiles first
    const int bg = w % BH;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int t0 = it * g.P;
    const int bt = t0 / kBlock;
    const size_t tile_id = (size_t)bg * g.ntile_bg + it;
    const int U = bt > 0 ? count[tile_id] : 0;
    const int nsteps = U + 1;
    const int* lst = list + tile_id * g.cap;
    const size_t kv_row0 = (size_t)bg * g.T;

    for (int idx = tid; idx < kTileRows * CH; idx += blockDim.x) {
        const int r = idx / CH, c = idx % CH;
        const int hl = r / g.P, t = t0 + r % g.P;
        const bool ok = r < g.M && t < g.T;
        const size_t off = ok ? ((size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t) * D + c * 8 : 0;
        cp_async16(Qs + swz<D>(r, c), q + off, ok ? 16 : 0);
        cp_async16(Gs + swz<D>(r, c), dout + off, ok ? 16 : 0);
    }
    auto load = [&](int s, int stage, bool with_v) {
        const int j = s < U ? lst[s] : bt;
        for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
            const int r = idx / CH, c = idx % CH;
            const int tok = j * kBlock + r;
            const bool ok = tok < g.T;
            const size_t off = (kv_row0 + (ok ? tok : 0)) * D + c * 8;
            cp_async16(Ks + stage * kBlock * D + swz<D>(r, c), k + off, ok ? 16 : 0);
            if (with_v) cp_async16(Vs + stage * kBlock * D + swz<D>(r, c), v + off, ok ? 16 : 0);
        }
    };

    const int g4 = lane >> 2, t4 = lane & 3;
    float tau_r[2], drow_r[2];
    int tpos[2];
    size_t rowid[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = warp * 16 + g4 + 8 * i;
        const int hl = r / g.P, t = t0 + r % g.P;
        const bool ok = r < g.M && t < g.T;
        tpos[i] = ok ? t : -1;
        rowid[i] = ok ? (size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t : 0;
        tau_r[i] = (ok && bt > 0) ? tau[rowid[i]] : INFINITY;
        drow_r[i] = ok ? drow[rowid[i]] : 0.f;
    }

    // S = Q K^T for this warp's 16 rows x 64 keys of stage st
    auto qk = [&](const __nv_bfloat16* Kst, float (&sacc)[8][4]) {
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) sacc[n][c] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t a[4];
            ldsm_x4(a[0], a[1], a[2], a[3], smem_u32(Qs + swz<D>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4))));
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b0, b1, b2, b3;
                const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                ldsm_x4(b0, b1, b2, b3, smem_u32(Kst + swz<D>(key, kk * 2 + ((lane >> 3) & 1))));
                mma_bf16(sacc[2 * np], a, b0, b1);
                mma_bf16(sacc[2 * np + 1], a, b2, b3);
            }
        }
    };
    // log2 of x_j - tau per row (NaN-free: -inf when the row does not select block j)
    auto block_lx = [&](const float (&sacc)[8][4], float (&xm)[2]) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float rs = 0.f;
#pragma unroll
            for (int n = 0; n < 8; ++n) rs += sacc[n][2 * i] + sacc[n][2 * i + 1];
            rs += __shfl_xor_sync(0xffffffffu, rs, 1);
            rs += __shfl_xor_sync(0xffffffffu, rs, 2);
            xm[i] = rs * C.cxm - tau_r[i];
        }
    };

    // ---- pass 1: log-sum-exp, sum_j g_j, sum_j g_j kbar_j
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f}, s1[2] = {0.f, 0.f};
    float gk[2][D / 16][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int m = 0; m < D / 16; ++m)
#pragma unroll
            for (int e = 0; e < 4; ++e) gk[i][m][e] = 0.f;

    load(0, 0, false);
    cp_async_commit();
    for (int s = 0; s < nsteps; ++s) {
        const int stage = s & 1;
        const int j = s < U ? lst[s] : bt;
        const bool diag = (j == bt);
        if (s + 1 < nsteps) load(s + 1, stage ^ 1, false);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        float sacc[8][4];
        qk(Ks + stage * kBlock * D, sacc);
        float lp2[2];
        if (diag) {
            lp2[0] = tpos[0] >= 0 ? 0.f : -INFINITY;
            lp2[1] = tpos[1] >= 0 ? 0.f : -INFINITY;
        } else {
            float xm[2];
            block_lx(sacc, xm);
            float gj[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const bool sel = tpos[i] >= 0 && xm[i] > 0.f;
                const float lx = sel ? __log2f(xm[i]) : 0.f;
                lp2[i] = sel ? C.e_pow * lx : -INFINITY;
                gj[i] = sel ? exp2f(C.gpow * lx) : 0.f;
                s1[i] += gj[i];
            }
            if (__any_sync(0xffffffffu, gj[0] > 0.f || gj[1] > 0.f)) {
                const float4* kb = reinterpret_cast<const float4*>(ksum + ((size_t)bg * g.nbs + j) * D);
#pragma unroll
                for (int m = 0; m < D / 16; ++m) {
                    const float4 kv = __ldg(kb + 4 * m + t4);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        gk[i][m][0] = fmaf(gj[i], kv.x, gk[i][m][0]);
                        gk[i][m][1] = fmaf(gj[i], kv.y, gk[i][m][1]);
                        gk[i][m][2] = fmaf(gj[i], kv.z, gk[i][m][2]);
                        gk[i][m][3] = fmaf(gj[i], kv.w, gk[i][m][3]);
                    }
                }
            }
        }
        if (__any_sync(0xffffffffu, (lp2[0] > -INFINITY) || (lp2[1] > -INFINITY))) {
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = c >> 1;
                    float l2 = fmaf(sacc[n][c], C.sm2, lp2[i]);
                    if (diag && j * kBlock + n * 8 + 2 * t4 + (c & 1) > tpos[i]) l2 = -INFINITY;
                    sacc[n][c] = l2;
                    mx[i] = fmaxf(mx[i], l2);
                }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
                mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
                const float m_new = fmaxf(m_r[i], mx[i]);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                float ls = 0.f;
#pragma unroll
                for (int n = 0; n < 8; ++n) ls += exp2f(sacc[n][2 * i] - m_use) + exp2f(sacc[n][2 * i + 1] - m_use);
                l_r[i] = l_r[i] * exp2f(m_r[i] - m_use) + ls;
                m_r[i] = m_new;
            }
        }
        __syncthreads();
    }
    float lse2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float l = l_r[i];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        lse2[i] = tpos[i] >= 0 ? m_r[i] + __log2f(l) : 0.f;
        const int r = warp * 16 + g4 + 8 * i;
#pragma unroll
        for (int m = 0; m < D / 16; ++m)
            *reinterpret_cast<float4*>(GK + r * D + 16 * m + 4 * t4) =
                make_float4(gk[i][m][0], gk[i][m][1], gk[i][m][2], gk[i][m][3]);
    }

    // ---- pass 2: P, dS, c_j, H_j; dq += (dS + cs H_j / 64) K
    float s2[2] = {0.f, 0.f};
    float dqa[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) dqa[n][c] = 0.f;
    load(0, 0, true);
    cp_async_commit();
    for (int s = 0; s < nsteps; ++s) {
        const int stage = s & 1;
        const int j = s < U ? lst[s] : bt;
        const bool diag = (j == bt);
        if (s + 1 < nsteps) load(s + 1, stage ^ 1, true);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const __nv_bfloat16* Kst = Ks + stage * kBlock * D;
        const __nv_bfloat16* Vst = Vs + stage * kBlock * D;
        float sacc[8][4];
        qk(Kst, sacc);
        float lp2[2], xm[2] = {1.f, 1.f};
        if (diag) {
            lp2[0] = tpos[0] >= 0 ? 0.f : -INFINITY;
            lp2[1] = tpos[1] >= 0 ? 0.f : -INFINITY;
        } else {
            block_lx(sacc, xm);
#pragma unroll
            for (int i = 0; i < 2; ++i)
                lp2[i] = (tpos[i] >= 0 && xm[i] > 0.f) ? C.e_pow * __log2f(xm[i]) : -INFINITY;
        }
        if (!__any_sync(0xffffffffu, (lp2[0] > -INFINITY) || (lp2[1] > -INFINITY))) {
            __syncthreads();
            continue;
        }
        // P in sacc
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int i = c >> 1;
                float l2 = fmaf(sacc[n][c], C.sm2, lp2[i]);
                if (diag && j * kBlock + n * 8 + 2 * t4 + (c & 1) > tpos[i]) l2 = -INFINITY;
                sacc[n][c] = exp2f(l2 - lse2[i]);
            }
        // dP = dout V^T
        float dpa[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) dpa[n][c] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t a[4];
            ldsm_x4(a[0], a[1], a[2], a[3], smem_u32(Gs + swz<D>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4))));
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b0, b1, b2, b3;
                const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                ldsm_x4(b0, b1, b2, b3, smem_u32(Vst + swz<D>(key, kk * 2 + ((lane >> 3) & 1))));
                mma_bf16(dpa[2 * np], a, b0, b1);
                mma_bf16(dpa[2 * np + 1], a, b2, b3);
            }
        }
        // dS = P (dP - D); c_j = row sum; fold cs H_j / 64
        float cj[2] = {0.f, 0.f};
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int i = c >> 1;
                dpa[n][c] = sacc[n][c] * (dpa[n][c] - drow_r[i]);
                cj[i] += dpa[n][c];
            }
        if (!diag) {
            float f[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                cj[i] += __shfl_xor_sync(0xffffffffu, cj[i], 1);
                cj[i] += __shfl_xor_sync(0xffffffffu, cj[i], 2);
                const float h = lp2[i] > -INFINITY ? cj[i] / xm[i] : 0.f;
                s2[i] += h;
                f[i] = C.cs64 * h;
            }
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                dpa[n][0] += f[0]; dpa[n][1] += f[0];
                dpa[n][2] += f[1]; dpa[n][3] += f[1];
            }
        }
        uint32_t da[4][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            da[n >> 1][(n & 1) * 2 + 0] = pack_bf16(dpa[n][0], dpa[n][1]);
            da[n >> 1][(n & 1) * 2 + 1] = pack_bf16(dpa[n][2], dpa[n][3]);
        }
        // dq += dS K
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t b0, b1, b2, b3;
                const int key = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                ldsm_x4_t(b0, b1, b2, b3, smem_u32(Kst + swz<D>(key, dp * 2 + (lane >> 4))));
                mma_bf16(dqa[2 * dp], da[kk], b0, b1);
                mma_bf16(dqa[2 * dp + 1], da[kk], b2, b3);
            }
        }
        __syncthreads();
    }

    // ---- epilogue: r, the -cs r sum_j g_j kbar_j term, scale, store
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        if (tpos[i] < 0) continue;
        const int r = warp * 16 + g4 + 8 * i;
        const float rr = s1[i] > 0.f ? s2[i] / s1[i] : 0.f;
        const float cr = C.cs * rr;
        __nv_bfloat16* dst = dq + rowid[i] * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            const int col = n * 8 + 2 * t4;
            const float2 gkv = *reinterpret_cast<const float2*>(GK + r * D + col);
            const float a0 = (dqa[n][2 * i] - cr * gkv.x) * C.isd;
            const float a1 = (dqa[n][2 * i + 1] - cr * gkv.y) * C.isd;
            *reinterpret_cast<__nv_bfloat162*>(dst + col) = __floats2bfloat162_rn(a0, a1);
        }
        if (t4 == 0) {
            lse_out[rowid[i]] = lse2[i];
            r_out[rowid[i]] = rr;
        }
    }
}

// ------------------------------------------------------------------ key-major: dk, dv
constexpr int kBwdChunk = 1024;   // candidate tiles examined per enumeration round

template <int D>
__global__ void __launch_bounds__(256, 1)
bwd_dkv_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
               const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
               const float* __restrict__ drow, const float* __restrict__ tau,
               const float* __restrict__ lse, const float* __restrict__ rrow,
               const int* __restrict__ list, const int* __restrict__ count,
               __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, PrefillGeom g, BwdConsts C) {
    constexpr int CH = D / 8;
    extern __shared__ uint4 smem_u4[];
    __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem_u4);   // [64][D]
    __nv_bfloat16* Vs = Ks + kBlock * D;                             // [64][D]
    __nv_bfloat16* Qs = Vs + kBlock * D;                             // [2][128][D]
    __nv_bfloat16* Gs = Qs + 2 * kTileRows * D;                      // dout tiles [2][128][D]
    float* mlse = reinterpret_cast<float*>(Gs + 2 * kTileRows * D);  // [2][128]
    float* mdrow = mlse + 2 * kTileRows;                             // [2][128]
    float* mtau = mdrow + 2 * kTileRows;                             // [2][128]
    float* mr = mtau + 2 * kTileRows;                                // [2][128]
    int* mtp = reinterpret_cast<int*>(mr + 2 * kTileRows);           // [2][128]
    float* xs = reinterpret_cast<float*>(mtp + 2 * kTileRows);       // [4][128] partial row sums
    float* cl = xs + 4 * kTileRows;                                  // [4][128]
    float* lps = cl + 4 * kTileRows;                                 // [128] log2 prior - lse
    float* xms = lps + kTileRows;                                    // [128] x_j - tau
    float* fs = xms + kTileRows;                                     // [128] cs ds_j / 64
    int* tl = reinterpret_cast<int*>(fs + kTileRows);                // [kBwdChunk]
    int* wtot = tl + kBwdChunk;                                      // [8]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kw = warp & 3, rb = (warp >> 2) * 64;   // this warp: keys 16 kw.., rows rb..rb+63
    const int th = tid & 127;                         // thread index within the row half
    // the four warps of one row half (warps 4 (rb / 64) .. +3) synchronise on barrier 1 + rb / 64
    auto half_bar = [&]() { asm volatile("bar.sync %0, 128;" :: "r"(1 + (rb >> 6)) : "memory"); };
    const int g4 = lane >> 2, t4 = lane & 3;
    const int BH = g.B * g.Hkv;
    const int j = blockIdx.x / BH;                    // low blocks (most listing tiles) first
    const int bg = blockIdx.x % BH;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const size_t kv_row0 = (size_t)bg * g.T;
    const int it_diag0 = j * kBlock / g.P;
    const int it_past0 = (j + 1) * kBlock / g.P;      // first tile whose own block is after j
    const int it_diag1 = it_past0 < g.ntile_bg ? it_past0 : g.ntile_bg;

    for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
        const int r = idx / CH, c = idx % CH;
        const int tok = j * kBlock + r;
        const bool ok = tok < g.T;
        const size_t off = (kv_row0 + (ok ? tok : 0)) * D + c * 8;
        cp_async16(Ks + swz<D>(r, c), k + off, ok ? 16 : 0);
        cp_async16(Vs + swz<D>(r, c), v + off, ok ? 16 : 0);
    }
    cp_async_commit();

    auto load_tile = [&](int it, int stage) {
        const int t0 = it * g.P;
        const int bt = t0 / kBlock;
        __nv_bfloat16* Qd = Qs + stage * kTileRows * D;
        __nv_bfloat16* Gd = Gs + stage * kTileRows * D;
        for (int idx = tid; idx < kTileRows * CH; idx += blockDim.x) {
            const int r = idx / CH, c = idx % CH;
            const int hl = r / g.P, t = t0 + r % g.P;
            const bool ok = r < g.M && t < g.T;
            const size_t off = ok ? ((size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t) * D + c * 8 : 0;
            cp_async16(Qd + swz<D>(r, c), q + off, ok ? 16 : 0);
            cp_async16(Gd + swz<D>(r, c), dout + off, ok ? 16 : 0);
        }
        if (tid < kTileRows) {
            const int r = tid;
            const int hl = r / g.P, t = t0 + r % g.P;
            const bool ok = r < g.M && t < g.T;
            const size_t row = ok ? (size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t : 0;
            mtp[stage * kTileRows + r] = ok ? t : -1;
            mlse[stage * kTileRows + r] = ok ? lse[row] : 0.f;
            mdrow[stage * kTileRows + r] = ok ? drow[row] : 0.f;
            mtau[stage * kTileRows + r] = (ok && bt > 0) ? tau[row] : INFINITY;
            mr[stage * kTileRows + r] = ok ? rrow[row] : 0.f;
        }
    };
    // partial sums over this warp's 16 keys of a [16 keys x 64 rows] accumulator, per row
    auto col_partial = [&](const float (&acc)[8][4], float* dst) {
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float s = acc[n][e] + acc[n][2 + e];
                s += __shfl_xor_sync(0xffffffffu, s, 4);
                s += __shfl_xor_sync(0xffffffffu, s, 8);
                s += __shfl_xor_sync(0xffffffffu, s, 16);
                if (g4 == 0) dst[kw * kTileRows + rb + n * 8 + 2 * t4 + e] = s;
            }
    };

    float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) { dka[n][c] = 0.f; dva[n][c] = 0.f; }

    for (int base = it_diag0; base < g.ntile_bg; base += kBwdChunk) {
        // ---- enumerate: candidates base + 4 tid + e, kept in ascending order
        int flag[4], cnt = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int it = base + 4 * tid + e;
            bool keep = false;
            if (it < g.ntile_bg) {
                if (it < it_diag1) {
                    keep = true;
                } else {
                    const size_t tile = (size_t)bg * g.ntile_bg + it;
                    const int* L = list + tile * g.cap;
                    int lo = 0, hi = count[tile];   // first entry >= j
                    while (lo < hi) {
                        const int mid = (lo + hi) >> 1;
                        if (L[mid] < j) lo = mid + 1; else hi = mid;
                    }
                    keep = lo < count[tile] && L[lo] == j;
                }
            }
            flag[e] = keep;
            cnt += keep;
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wtot[warp] = incl;
        __syncthreads();
        int woff = 0, ntl = 0;
        for (int w2 = 0; w2 < 8; ++w2) {
            if (w2 < warp) woff += wtot[w2];
            ntl += wtot[w2];
        }
        int pos = woff + incl - cnt;
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (flag[e]) tl[pos++] = base + 4 * tid + e;
        __syncthreads();

        // ---- process the chunk's tiles through the two-stage ring
        if (ntl > 0) load_tile(tl[0], 0);
        cp_async_commit();
        for (int s = 0; s < ntl; ++s) {
            const int stage = s & 1;
            const int it = tl[s];
            const bool diag = it < it_diag1;
            if (s + 1 < ntl) load_tile(tl[s + 1], stage ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
            __syncthreads();
            const __nv_bfloat16* Qst = Qs + stage * kTileRows * D;
            const __nv_bfloat16* Gst = Gs + stage * kTileRows * D;
            const int* tp_s = mtp + stage * kTileRows;

            // S^T = K Q^T: 16 keys x 64 rows
            float st[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int c = 0; c < 4; ++c) st[n][c] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(a[0], a[1], a[2], a[3], smem_u32(Ks + swz<D>(kw * 16 + (lane & 15), kk * 2 + (lane >> 4))));
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    const int row = rb + np * 16 + (lane & 7) + ((lane >> 4) << 3);
                    ldsm_x4(b0, b1, b2, b3, smem_u32(Qst + swz<D>(row, kk * 2 + ((lane >> 3) & 1))));
                    mma_bf16(st[2 * np], a, b0, b1);
                    mma_bf16(st[2 * np + 1], a, b2, b3);
                }
            }
            // per-row values, once per row: the 64 threads th < 64 of each row half own
            // rows rb + th; the half's four warps meet at a named barrier of 128 threads
            if (!diag) col_partial(st, xs);
            half_bar();
            if (th < 64) {
                const int row = rb + th;
                const int tp = tp_s[row];
                float lp = tp >= 0 ? 0.f : -INFINITY, xm = 1.f;
                if (!diag) {
                    const float x = (xs[row] + xs[kTileRows + row] + xs[2 * kTileRows + row] +
                                     xs[3 * kTileRows + row]) * C.cxm;
                    xm = x - mtau[stage * kTileRows + row];
                    lp = (tp >= 0 && xm > 0.f) ? C.e_pow * __log2f(xm) : -INFINITY;
                }
                lps[row] = lp - mlse[stage * kTileRows + row];
                xms[row] = xm;
            }
            half_bar();
            // P^T in st
            const int key0 = j * kBlock + kw * 16 + g4;
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int row = rb + n * 8 + 2 * t4 + e;
                    const float lp = lps[row];
                    const int tp = diag ? tp_s[row] : 0x7fffffff;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float l2 = fmaf(st[n][e + 2 * hh], C.sm2, lp);
                        if (key0 + hh * 8 > tp) l2 = -INFINITY;
                        st[n][e + 2 * hh] = exp2f(l2);
                    }
                }
            // dV += P^T dout
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t pa[4];
                pa[0] = pack_bf16(st[2 * kk][0], st[2 * kk][1]);
                pa[1] = pack_bf16(st[2 * kk][2], st[2 * kk][3]);
                pa[2] = pack_bf16(st[2 * kk + 1][0], st[2 * kk + 1][1]);
                pa[3] = pack_bf16(st[2 * kk + 1][2], st[2 * kk + 1][3]);
#pragma unroll
                for (int dp = 0; dp < D / 16; ++dp) {
                    uint32_t b0, b1, b2, b3;
                    const int row = rb + kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    ldsm_x4_t(b0, b1, b2, b3, smem_u32(Gst + swz<D>(row, dp * 2 + (lane >> 4))));
                    mma_bf16(dva[2 * dp], pa, b0, b1);
                    mma_bf16(dva[2 * dp + 1], pa, b2, b3);
                }
            }
            // dP^T = V dout^T
            float dpt[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int c = 0; c < 4; ++c) dpt[n][c] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(a[0], a[1], a[2], a[3], smem_u32(Vs + swz<D>(kw * 16 + (lane & 15), kk * 2 + (lane >> 4))));
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    const int row = rb + np * 16 + (lane & 7) + ((lane >> 4) << 3);
                    ldsm_x4(b0, b1, b2, b3, smem_u32(Gst + swz<D>(row, kk * 2 + ((lane >> 3) & 1))));
                    mma_bf16(dpt[2 * np], a, b0, b1);
                    mma_bf16(dpt[2 * np + 1], a, b2, b3);
                }
            }
            // dS^T = P^T (dP^T - D)
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float dr = mdrow[stage * kTileRows + rb + n * 8 + 2 * t4 + e];
                    dpt[n][e] = st[n][e] * (dpt[n][e] - dr);
                    dpt[n][e + 2] = st[n][e + 2] * (dpt[n][e + 2] - dr);
                }
            if (!diag) {
                // c_j per row over all 64 keys, then the folded cs ds_j / 64
                col_partial(dpt, cl);
                half_bar();
                if (th < 64) {
                    const int row = rb + th;
                    float f = 0.f;
                    if (lps[row] > -INFINITY) {
                        const float xm = xms[row];
                        const float c = cl[row] + cl[kTileRows + row] + cl[2 * kTileRows + row] +
                                        cl[3 * kTileRows + row];
                        const float gj = exp2f(C.gpow * __log2f(xm));
                        f = C.cs64 * (c / xm - mr[stage * kTileRows + row] * gj);
                    }
                    fs[row] = f;
                }
                half_bar();
#pragma unroll
                for (int n = 0; n < 8; ++n)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float f = fs[rb + n * 8 + 2 * t4 + e];
                        dpt[n][e] += f;
                        dpt[n][2 + e] += f;
                    }
            }
            // dK += dS^T Q
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t pa[4];
                pa[0] = pack_bf16(dpt[2 * kk][0], dpt[2 * kk][1]);
                pa[1] = pack_bf16(dpt[2 * kk][2], dpt[2 * kk][3]);
                pa[2] = pack_bf16(dpt[2 * kk + 1][0], dpt[2 * kk + 1][1]);
                pa[3] = pack_bf16(dpt[2 * kk + 1][2], dpt[2 * kk + 1][3]);
#pragma unroll
                for (int dp = 0; dp < D / 16; ++dp) {
                    uint32_t b0, b1, b2, b3;
                    const int row = rb + kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    ldsm_x4_t(b0, b1, b2, b3, smem_u32(Qst + swz<D>(row, dp * 2 + (lane >> 4))));
                    mma_bf16(dka[2 * dp], pa, b0, b1);
                    mma_bf16(dka[2 * dp + 1], pa, b2, b3);
                }
            }
            __syncthreads();
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- combine the two row halves and store the block's 64 keys
    float* red = reinterpret_cast<float*>(Qs);   // [4 warps][2][16][D] fp32
    if (rb != 0) {
        float* mine = red + kw * 2 * 16 * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int kr = g4 + 8 * (c >> 1), col = n * 8 + 2 * t4 + (c & 1);
                mine[kr * D + col] = dka[n][c];
                mine[16 * D + kr * D + col] = dva[n][c];
            }
    }
    __syncthreads();
    if (rb == 0) {
        const float* other = red + kw * 2 * 16 * D;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int kr = g4 + 8 * hh;
            const int tok = j * kBlock + kw * 16 + kr;
            if (tok >= g.T) continue;
            __nv_bfloat16* dkr = dk + (kv_row0 + tok) * D;
            __nv_bfloat16* dvr = dv + (kv_row0 + tok) * D;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                const int col = n * 8 + 2 * t4;
                const float k0 = (dka[n][2 * hh] + other[kr * D + col]) * C.isd;
                const float k1 = (dka[n][2 * hh + 1] + other[kr * D + col + 1]) * C.isd;
                const float v0 = dva[n][2 * hh] + other[16 * D + kr * D + col];
                const float v1 = dva[n][2 * hh + 1] + other[16 * D + kr * D + col + 1];
                *reinterpret_cast<__nv_bfloat162*>(dkr + col) = __floats2bfloat162_rn(k0, k1);
                *reinterpret_cast<__nv_bfloat162*>(dvr + col) = __floats2bfloat162_rn(v0, v1);
            }
        }
    }
}

// ------------------------------------------------------------------ host side
// Q and dout tiles, two stages of K and V (bf16), sum_j g_j kbar_j per row (fp32)
static size_t bwd_dq_smem(int d) {
    return (size_t)(2 * kTileRows + 4 * kBlock) * d * 2 + (size_t)kTileRows * d * 4; }
// K, V of the block and two stages of Q and dout tiles (bf16); per-row data of two stages
// (log-sum-exp, D, tau, r, position), the two cross-warp row-sum buffers, three per-row
// values of the current tile and the tile list
static size_t bwd_dkv_smem(int d) {
    return (size_t)(2 * kBlock + 4 * kTileRows) * d * 2 + (size_t)(5 * 2 + 2 * 4 + 3) * kTileRows * 4 +
           (size_t)(kBwdChunk + 8) * 4;
}

template <int D>
static cudaError_t launch_bwd_d(const void* q, const void* k, const void* v, const void* out,
                                const void* dout, void* dq, void* dk, void* dv, const PrefillGeom& g,
                                const BwdGeom& bw, char* ws, const BwdConsts& C, bool tc, float alpha,
                                float coarse_scale, cudaStream_t stream) {
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const auto* vb = static_cast<const __nv_bfloat16*>(v);
    const auto* gb = static_cast<const __nv_bfloat16*>(dout);
    float* drow = reinterpret_cast<float*>(ws + bw.off_drow);
    float* lse = reinterpret_cast<float*>(ws + bw.off_lse);
    float* rr = reinterpret_cast<float*>(ws + bw.off_r);
    const float* tau = reinterpret_cast<const float*>(ws + g.off_tau);
    const int* list = reinterpret_cast<const int*>(ws + g.off_list);
    const int* count = reinterpret_cast<const int*>(ws + g.off_count);
    const float* ksum = reinterpret_cast<const float*>(ws + g.off_ksum);

    const long long nrows = (long long)g.B * g.Hq * g.T;
    bwd_rowdot_kernel<<<(unsigned)((nrows + 7) / 8), 256, 0, stream>>>(
        gb, static_cast<const __nv_bfloat16*>(out), drow, nrows, D);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    if (tc) {
        e = launch_bwd_dq_tc(q, k, v, dout, dq, g, bw, ws, alpha, coarse_scale, stream);
    } else {
        const size_t sm1 = bwd_dq_smem(D);
        e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
        if (e != cudaSuccess) return e;
        bwd_dq_kernel<D><<<g.ntiles, 256, sm1, stream>>>(qb, kb, vb, gb, drow, tau, list, count, ksum,
                                                         static_cast<__nv_bfloat16*>(dq), lse, rr, g, C);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;

    if (tc) return launch_bwd_dkv_tc(q, k, v, dout, dk, dv, g, bw, ws, alpha, coarse_scale, stream);
    const size_t sm2 = bwd_dkv_smem(D);
    e = cudaFuncSetAttribute(bwd_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
    if (e != cudaSuccess) return e;
    const int nb = (g.T + kBlock - 1) / kBlock;
    bwd_dkv_kernel<D><<<g.B * g.Hkv * nb, 256, sm2, stream>>>(
        qb, kb, vb, gb, drow, tau, lse, rr, list, count, static_cast<__nv_bfloat16*>(dk),
        static_cast<__nv_bfloat16*>(dv), g, C);
    return cudaGetLastError();
}

// Which kernels run: the tcgen05 ones (backward_tc.cu: statistics, dq, then dk/dv) wherever
// the tile holds at least 8 positions, unless DASH_BWD_KERNEL=mma selects the mma.sync
// kernels above (kept for comparison and for more than 16 query heads per KV head).
static bool use_mma_backward() {
    static const int choice = [] {
        const char* e = getenv("DASH_BWD_KERNEL");
        return (e && strcmp(e, "mma") == 0) ? 1 : 0;
    }();
    return choice == 1;
}

cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out,
                            const void* dout, void* dq, void* dk, void* dv, const PrefillGeom& g,
                            const BwdGeom& bw, char* ws, float alpha, float coarse_scale,
                            cudaStream_t stream) {
    BwdConsts C;
    const float sd = sqrtf((float)g.d);
    C.cxm = (alpha - 1.0f) * coarse_scale / sd / (float)kBlock;
    C.e_pow = 1.0f / (alpha - 1.0f);
    C.gpow = (2.0f - alpha) / (alpha - 1.0f);
    C.sm2 = 1.4426950408889634f / sd;
    C.cs64 = coarse_scale / (float)kBlock;
    C.cs = coarse_scale;
    C.isd = 1.0f / sd;
    const bool tc = fine_tc_supported(g) && !use_mma_backward();
    return g.d == 128 ? launch_bwd_d<128>(q, k, v, out, dout, dq, dk, dv, g, bw, ws, C, tc, alpha, coarse_scale, stream)
                      : launch_bwd_d<64>(q, k, v, out, dout, dq, dk, dv, g, bw, ws, C, tc, alpha, coarse_scale, stream);
}

}  // namespace dash
