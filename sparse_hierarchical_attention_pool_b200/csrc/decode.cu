// decode.cu -- one decode step of DashAttention with a split-KV (flash-decoding) layout.
//
// Same arithmetic as a prefill row t = kv_len - 1 ("DashAttention: Making Sparse Attention
// Fully Differentiable with Adaptive Block Selection", section "Core Mechanism"): coarse
// scores over the cached block summaries of blocks j < bt = t / 64, alpha-entmax weights,
// then softmax over the selected blocks' tokens plus the own block (causal, prior 1) with
// log p as the prior.  Kernels, all launched with shapes known on the host:
//   1. decode_scores : x[b, h, j] for every head of a KV group, each block summary read once
//                      for all G heads (a warp streams 16 summaries of one group);
//   2. decode_select : per (b, kv head): one warp per head solves tau with the row in
//                      registers, the union of the heads' selected blocks becomes the
//                      group's list (own block last), and the last CTA writes the work plan
//                      of the balanced attention pass;
//   3. attention     : decode_attn_tc_kernel (decode_tc.cu) for G <= 8, which also merges
//                      the split groups; otherwise decode_attn below, split-KV over chunks of
//                      16 listed blocks with a two-stage cp.async pipeline, each listed block
//                      read once for every head of the group, partial (max, sum, output) per
//                      chunk and head, and
//   4. decode_combine: merging those partials of each (b, h) into bf16.
// The HBM traffic that matters is step 3: (union blocks + 1) * 64 * d * 2 bytes * 2 per
// (b, kv head).
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "entmax.cuh"
#include "kernels.h"

namespace dash {

constexpr int kSelRegs = 48;        // row values a select lane keeps in registers

// ------------------------------------------------------------------ scores
//
// x[b, h, j] = cx * q[b, h] . kbar[b, g, j] for the G heads of every group and every past
// block j < bt.  A warp takes RW consecutive block summaries of one group and issues all
// their loads at once (lane l holds dims [l D/32, (l + 1) D/32) of each row: one coalesced
// row per instruction); the group's query rows sit in registers (heads padded to GP, a
// power of two <= 8).  Per task of R = 32/GP rows (at most 8) a lane has R * GP partial sums,
// and a butterfly reduce-scatter over the 32 lanes leaves every (row, head) sum complete on
// its own lane with 31 shuffles in all.  Each summary is read from HBM once for all heads.

// Butterfly reduce-scatter of C values per lane over lane offsets O, O/2, ..., 1: at each
// level the lane with bit O set keeps the upper half of its values and receives the
// partner's copy of it; once one value is left, the remaining levels sum it.
template <int C, int O>
__device__ __forceinline__ void reduce_scatter(float* v, int lane) {
    if constexpr (O >= 1) {
        if constexpr (C >= 2) {
            const bool up = (lane & O) != 0;
#pragma unroll
            for (int i = 0; i < C / 2; ++i) {
                const float send = up ? v[i] : v[i + C / 2];
                const float keep = up ? v[i + C / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
            }
            reduce_scatter<C / 2, O / 2>(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
            reduce_scatter<1, O / 2>(v, lane);
        }
    }
}

template <int D, int GP>
struct ScoreShape {
    static constexpr int DPL = D / 32;                 // dims per lane
    static constexpr int R = GP >= 4 ? 32 / GP : 8;    // rows per reduce-scatter
    static constexpr int V = R * GP;                   // partial sums per lane (<= 32)
    static constexpr int RW = 2 * R;                   // rows per warp, loads issued together
    static constexpr int LOGV = V >= 32 ? 5 : V >= 16 ? 4 : V >= 8 ? 3 : V >= 4 ? 2 : V >= 2 ? 1 : 0;
};

template <int D, int GP>
__global__ void __launch_bounds__(256)
decode_scores_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ ksum,
                     const int* __restrict__ kv_len, float* __restrict__ xs, DecodeGeom g, float cx) {
    using S = ScoreShape<D, GP>;
    const int lane = threadIdx.x & 31;
    const long long wtask = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int tpg = (g.nbs + S::RW - 1) / S::RW;
    const int bg = (int)(wtask / tpg);
    if (bg >= g.B * g.Hkv) return;
    const int j0 = (int)(wtask % tpg) * S::RW;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int L = kv_len[b];
    if (L < 1 || L > g.Tmax) return;
    const int bt = (L - 1) / kBlock;
    if (j0 >= bt) return;
    const size_t qrow0 = (size_t)b * g.Hq + (size_t)kvh * g.G;
    // rows past bt load row bt - 1 again (in bounds; their sums are not written)
    const float* src = ksum + (size_t)bg * g.nbs * D + lane * S::DPL;
    float kv[S::RW][S::DPL];
#pragma unroll
    for (int r = 0; r < S::RW; ++r) {
        const size_t jr = (size_t)min(j0 + r, bt - 1);
        if constexpr (S::DPL == 4) {
            const float4 t = __ldg(reinterpret_cast<const float4*>(src + jr * D));
            kv[r][0] = t.x; kv[r][1] = t.y; kv[r][2] = t.z; kv[r][3] = t.w;
        } else {
            const float2 t = __ldg(reinterpret_cast<const float2*>(src + jr * D));
            kv[r][0] = t.x; kv[r][1] = t.y;
        }
    }
    // query rows of the group (heads past G repeat head 0; their sums are not written)
    float qv[GP][S::DPL];
#pragma unroll
    for (int h = 0; h < GP; ++h) {
        const __nv_bfloat16* qh = q + (qrow0 + (h < g.G ? h : 0)) * D + lane * S::DPL;
        if constexpr (S::DPL == 4) {
            const uint2 t = __ldg(reinterpret_cast<const uint2*>(qh));
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&t.x));
            const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&t.y));
            qv[h][0] = a.x; qv[h][1] = a.y; qv[h][2] = c.x; qv[h][3] = c.y;
        } else {
            const uint32_t t = __ldg(reinterpret_cast<const unsigned int*>(qh));
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&t));
            qv[h][0] = a.x; qv[h][1] = a.y;
        }
    }
    const size_t cap = (size_t)g.nbs + 1;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float v[S::V];
#pragma unroll
        for (int r = 0; r < S::R; ++r)
#pragma unroll
            for (int h = 0; h < GP; ++h) {
                float acc = 0.f;
#pragma unroll
                for (int d = 0; d < S::DPL; ++d) acc = fmaf(kv[half * S::R + r][d], qv[h][d], acc);
                v[r * GP + h] = acc;
            }
        reduce_scatter<S::V, 16>(v, lane);
        // value index held by this lane (see reduce_scatter): lane * V/32 + k when V >= 32,
        // else lane >> (5 - log2 V), replicated on 32/V lanes
        if constexpr (S::V >= 32) {
#pragma unroll
            for (int k = 0; k < S::V / 32; ++k) {
                const int idx = lane * (S::V / 32) + k, r = idx / GP, h = idx % GP;
                const int j = j0 + half * S::R + r;
                if (h < g.G && j < bt) xs[(qrow0 + h) * cap + j] = v[k] * cx;
            }
        } else {
            const int idx = lane >> (5 - S::LOGV), r = idx / GP, h = idx % GP;
            const int j = j0 + half * S::R + r;
            if ((lane & ((32 >> S::LOGV) - 1)) == 0 && h < g.G && j < bt) xs[(qrow0 + h) * cap + j] = v[0] * cx;
        }
    }
}

// Groups of more than 8 heads: four threads per block summary, each with a quarter of its d
// values; every head's partial dot product is reduced over the four threads with two
// shuffles.
template <int D>
__global__ void __launch_bounds__(256)
decode_scores_wide_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ ksum,
                          const int* __restrict__ kv_len, float* __restrict__ xs, DecodeGeom g, float cx) {
    constexpr int QD = D / 4;                 // dims per thread
    constexpr int QV = QD / 4;                // float4 per thread
    constexpr int QS = D + 16;                // padded row stride of a query head (floats)
    __shared__ __align__(16) float qs[32 * QS];
    const int bg = blockIdx.x, b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int L = kv_len[b];
    if (L < 1 || L > g.Tmax) return;
    const int bt = (L - 1) / kBlock;
    const int j0 = blockIdx.y * 64;
    if (j0 >= bt) return;
    const int part = threadIdx.x & 3, j = j0 + (threadIdx.x >> 2);
    float4 kv[QV];
#pragma unroll
    for (int i = 0; i < QV; ++i) kv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < bt) {
        const float4* kb = reinterpret_cast<const float4*>(ksum + ((size_t)bg * g.nbs + j) * D + part * QD);
#pragma unroll
        for (int i = 0; i < QV; ++i) kv[i] = __ldg(kb + i);
    }
    for (int i = threadIdx.x; i < g.G * D; i += blockDim.x) {
        const int h = i / D, c = i % D;
        qs[h * QS + (c / QD) * (QD + 4) + c % QD] = __bfloat162float(q[(size_t)(b * g.Hq + kvh * g.G) * D + i]);
    }
    __syncthreads();
    const int cap = g.nbs + 1;
    for (int h0 = 0; h0 < g.G; h0 += 4) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
            if (h0 + hh >= g.G) break;
            const float4* qv = reinterpret_cast<const float4*>(qs + (h0 + hh) * QS + part * (QD + 4));
#pragma unroll
            for (int i = 0; i < QV; ++i) {
                const float4 a = qv[i];
                acc[hh] = fmaf(a.x, kv[i].x, acc[hh]);
                acc[hh] = fmaf(a.y, kv[i].y, acc[hh]);
                acc[hh] = fmaf(a.z, kv[i].z, acc[hh]);
                acc[hh] = fmaf(a.w, kv[i].w, acc[hh]);
            }
        }
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
            acc[hh] += __shfl_xor_sync(0xffffffffu, acc[hh], 1);
            acc[hh] += __shfl_xor_sync(0xffffffffu, acc[hh], 2);
        }
        const int h = h0 + part;
        const float mine = part == 0 ? acc[0] : part == 1 ? acc[1] : part == 2 ? acc[2] : acc[3];
        if (h < g.G && j < bt) xs[(size_t)(b * g.Hq + kvh * g.G + h) * cap + j] = mine * cx;
    }
}

template <int D, int GP>
void launch_scores_gp(const __nv_bfloat16* q, const float* ksum, const int* kv_len, float* xs,
                      const DecodeGeom& g, float cx, cudaStream_t stream) {
    using S = ScoreShape<D, GP>;
    const long long warps = (long long)g.B * g.Hkv * ((g.nbs + S::RW - 1) / S::RW);
    const unsigned grid = (unsigned)((warps + 7) / 8);
    if (grid > 0) decode_scores_kernel<D, GP><<<grid, 256, 0, stream>>>(q, ksum, kv_len, xs, g, cx);
}

template <int D>
void launch_scores(const __nv_bfloat16* q, const float* ksum, const int* kv_len, float* xs,
                   const DecodeGeom& g, float cx, cudaStream_t stream) {
    if (g.G == 1) launch_scores_gp<D, 1>(q, ksum, kv_len, xs, g, cx, stream);
    else if (g.G == 2) launch_scores_gp<D, 2>(q, ksum, kv_len, xs, g, cx, stream);
    else if (g.G <= 4) launch_scores_gp<D, 4>(q, ksum, kv_len, xs, g, cx, stream);
    else if (g.G <= 8) launch_scores_gp<D, 8>(q, ksum, kv_len, xs, g, cx, stream);
    else {
        dim3 gs(g.B * g.Hkv, (g.nbs + 63) / 64 > 0 ? (g.nbs + 63) / 64 : 1);
        decode_scores_wide_kernel<D><<<gs, 256, 0, stream>>>(q, ksum, kv_len, xs, g, cx);
    }
}

// ------------------------------------------------------------------ select

// Row values of one head on one warp: lane l holds x[l + 32 k] for k < kSelRegs in
// registers (-inf past the row's end, which no pass counts); values past that are read from
// memory.
struct WarpRow {
    float r[kSelRegs];
    const float* p;
    int lane, n;
    __device__ __forceinline__ void load(const float* row, int ln, int count) {
        p = row; lane = ln; n = count;
#pragma unroll
        for (int k = 0; k < kSelRegs; ++k) {
            const int j = lane + 32 * k;
            r[k] = j < n ? row[j] : -INFINITY;
        }
    }
    template <class F>
    __device__ __forceinline__ void each(F&& f) const {
#pragma unroll
        for (int k = 0; k < kSelRegs; ++k) f(lane + 32 * k, r[k]);
        for (int j = lane + 32 * kSelRegs; j < n; j += 32) f(j, p[j]);
    }
};

constexpr int kHistBins = 64;       // bins of the histogram start over y = x - m in [-1, 0)

// Histogram start of the threshold solve (the idea of AdaSplash-2, whose abstract appears on
// the listing page "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention":
// a coarse histogram of the scores kept in on-chip memory gives a close initial threshold;
// the construction here is this library's):
// the values y = x - m in [-1, 0) go to bin k = floor((y + 1) * 64) with their count, sum and
// sum of squares, accumulated as integers (y and y^2 in 2^-24 fixed point), so the sums and
// the start do not depend on the order of the shared-memory atomics.  At a bin's lower edge
// e every value of the bins above lies above e, so f(e) = sum_{y > e} (y - e)^(1/(alpha-1))
// is exact there for alpha = 1.5 (S2 - 2 e S1 + e^2 S0) and alpha = 2 (S1 - e S0).  f is
// decreasing, so the highest edge with f >= 1 lies just below the root: Newton starts there
// instead of at -1.
// bins: this warp's shared area (kHistBins counts, then kHistBins sums, kHistBins sums of
// squares).  Every lane returns the start.
struct HistBins {
    unsigned int c[kHistBins];
    unsigned long long s1[kHistBins], s2[kHistBins];
};

template <int MODE>
__device__ __forceinline__ float hist_start(const WarpRow& xr, float m, HistBins* hb) {
    const int lane = threadIdx.x & 31;
    constexpr float kFix = 16777216.0f;                 // 2^24
    for (int i = lane; i < kHistBins; i += 32) { hb->c[i] = 0u; hb->s1[i] = 0ull; hb->s2[i] = 0ull; }
    __syncwarp();
    xr.each([&](int, float v) {
        const float y = v - m;
        if (y > -1.0f) {
            const int k = min(kHistBins - 1, (int)((y + 1.0f) * (float)kHistBins));
            atomicAdd(&hb->c[k], 1u);
            atomicAdd(&hb->s1[k], (unsigned long long)__float2ll_rn(y * kFix));
            atomicAdd(&hb->s2[k], (unsigned long long)__float2ll_rn(y * y * kFix));
        }
    });
    __syncwarp();
    // lane l holds bins 2l, 2l + 1; exact suffix sums over the bins at and above each edge
    long long c0 = hb->c[2 * lane], c1 = hb->c[2 * lane + 1];
    long long p0 = (long long)hb->s1[2 * lane], p1 = (long long)hb->s1[2 * lane + 1];
    long long q0 = (long long)hb->s2[2 * lane], q1 = (long long)hb->s2[2 * lane + 1];
    long long ac = c0 + c1, a1 = p0 + p1, a2 = q0 + q1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long nc = __shfl_down_sync(0xffffffffu, ac, o);
        const long long n1 = __shfl_down_sync(0xffffffffu, a1, o);
        const long long n2 = __shfl_down_sync(0xffffffffu, a2, o);
        if (lane + o < 32) { ac += nc; a1 += n1; a2 += n2; }
    }
    auto f_at = [&](int k, long long S0, long long S1q, long long S2q) {
        const double e = -1.0 + (double)k / kHistBins;
        const double S1 = (double)S1q / kFix, S2 = (double)S2q / kFix;
        return MODE == 1 ? S2 - 2.0 * e * S1 + e * e * (double)S0 : S1 - e * (double)S0;
    };
    const unsigned ok_odd = __ballot_sync(0xffffffffu, f_at(2 * lane + 1, ac - c0, a1 - p0, a2 - q0) >= 1.0);
    const unsigned ok_even = __ballot_sync(0xffffffffu, f_at(2 * lane, ac, a1, a2) >= 1.0);
    const int k_odd = ok_odd ? 2 * (31 - __clz((int)ok_odd)) + 1 : -1;
    const int k_even = ok_even ? 2 * (31 - __clz((int)ok_even)) : 0;
    __syncwarp();
    return -1.0f + (float)max(k_odd, k_even) / (float)kHistBins;
}

// Threshold of one row held by a warp (every lane returns it); MODE as in EntmaxPass::add_t.
// bins != nullptr: start from the histogram edge (alpha = 1.5 and 2), else from u = -1.
template <int MODE>
__device__ __forceinline__ float warp_row_tau(const WarpRow& xr, float m, float alpha, int* no_conv,
                                              HistBins* bins, int cap) {
    float u0 = -1.0f;
    if constexpr (MODE != 0) {
        if (bins) u0 = hist_start<MODE>(xr, m, bins);
    }
    EntmaxSolver sv;
    sv.init(m, alpha, u0, cap);
    float t = m;
    while (true) {
        EntmaxPass ps;
        ps.reset();
        xr.each([&](int, float v) { ps.add_t<MODE>((v - sv.m) - sv.u, sv.e); });
        ps.warp_reduce_t<MODE>();
        if (sv.update(ps, &t, no_conv)) break;
    }
    return t;
}

// Work plan of the balanced attention pass, built by the last select CTA to finish (a
// ticket in the workspace header): offs = exclusive prefix of the list lengths (U = offs[BH]
// blocks in all), and plan[c] = the group holding position floor(U c / n), where CTA c's
// range starts (n = min(nctas, U)).  Called by every thread of every CTA once its count is
// written.
__device__ void decode_plan_tail(const int* count, int* offs, int* plan, WsHeader* hdr, int BH, int nctas) {
    __shared__ int last_sh;
    __shared__ int wsum[32];
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();                              // this CTA's count before its ticket
        last_sh = atomicAdd(&hdr->ticket, 1) == BH - 1;
    }
    __syncthreads();
    if (!last_sh) return;
    __threadfence();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    const int slice = (BH + nwarp - 1) / nwarp;
    const int lo = min(BH, warp * slice), hi = min(BH, lo + slice);
    int sum = 0;
    for (int i = lo + lane; i < hi; i += 32) sum += __ldcg(count + i);
    sum = warp_sum_int(sum);
    if (lane == 0) wsum[warp] = sum;
    __syncthreads();
    int before = 0, U = 0;
    for (int w = 0; w < nwarp; ++w) {
        if (w < warp) before += wsum[w];
        U += wsum[w];
    }
    if (threadIdx.x == 0) offs[BH] = U;
    if (U < nctas) nctas = U;                         // the attention pass uses min(grid, U) CTAs
    for (int i0 = lo; i0 < hi; i0 += 32) {
        const int i = i0 + lane;
        const int v = i < hi ? __ldcg(count + i) : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        const int o0 = before + incl - v, o1 = before + incl;
        if (i < hi) {
            offs[i] = o0;
            if (v > 0) {
                // CTAs whose range starts inside [o0, o1)
                const int c_lo = (int)(((long long)o0 * nctas + U - 1) / U);
                const int c_hi = (int)(((long long)o1 * nctas - 1) / U);
                for (int c = c_lo; c <= c_hi; ++c) plan[c] = i;
            }
        }
        before += __shfl_sync(0xffffffffu, incl, 31);
    }
}

// One CTA of 8 warps per (b, kv head).  Warp w solves the thresholds of heads w, w + 8, ...
// with the row in registers (one warp per head: no cross-warp reduction in a pass).  The
// heads' selected blocks are OR-ed into a bitmap; every thread then takes bitmap words
// w, w + 256, ..., a block-wide scan of their popcounts places the words, and each thread
// writes its words' blocks into the group's list, the own block last.
constexpr int kSelThreads = 256;

__global__ void __launch_bounds__(kSelThreads)
decode_select_kernel(const int* __restrict__ kv_len, const float* __restrict__ xs,
                     float* __restrict__ tau, int* __restrict__ list, int* __restrict__ count,
                     int* __restrict__ done, int* __restrict__ offs, int* __restrict__ plan,
                     __nv_bfloat16* __restrict__ out, WsHeader* __restrict__ hdr, DecodeGeom g,
                     float alpha, int nctas, int hist_init) {
    constexpr int kWords = kMaxT / kBlock / 32;
    __shared__ HistBins hist[kSelThreads / 32];
    constexpr int kWpt = kWords / kSelThreads;        // bitmap words per thread
    __shared__ unsigned bitmap[kWords];
    __shared__ int wtot[kSelThreads / 32];
    const int bg = blockIdx.x, b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = kSelThreads / 32;
    const int cap = g.nbs + 1;
    const int L = kv_len[b];
    const size_t qrow0 = (size_t)b * g.Hq + (size_t)kvh * g.G;
    if (tid == 0) done[bg] = 0;
    if (L < 1 || L > g.Tmax) {
        // no keys: the group's heads get a zero output and no work
        if (tid == 0) count[bg] = 0;
        for (int i = tid; i < g.G * g.d; i += kSelThreads) out[qrow0 * g.d + i] = __float2bfloat16(0.f);
        if (nctas > 0) decode_plan_tail(count, offs, plan, hdr, g.B * g.Hkv, nctas);
        return;
    }
    const int bt = (L - 1) / kBlock;
    const int nw = (bt + 31) / 32;
    for (int i = tid; i < nw; i += kSelThreads) bitmap[i] = 0u;
    __syncthreads();
    int no_conv = 0;
    for (int hl = warp; hl < g.G; hl += nwarp) {
        const size_t row = qrow0 + hl;
        float t = __int_as_float(0x7fc00000);
        WarpRow xr;
        xr.load(xs + row * cap, lane, bt);
        if (bt > 0) {
            float m = -INFINITY;
            xr.each([&](int, float v) { m = fmaxf(m, v); });
            m = warp_max(m);
            HistBins* bins = hist_init ? &hist[warp] : nullptr;
            t = alpha == 1.5f ? warp_row_tau<1>(xr, m, alpha, &no_conv, bins, g.maxit)
              : alpha == 2.0f ? warp_row_tau<2>(xr, m, alpha, &no_conv, bins, g.maxit)
                              : warp_row_tau<0>(xr, m, alpha, &no_conv, bins, g.maxit);
        }
        if (lane == 0) tau[row] = t;
        float nsel = 0.f;
        xr.each([&](int j, float v) {
            if (v > t) {
                nsel += 1.f;
                atomicOr(&bitmap[j >> 5], 1u << (j & 31));
            }
        });
        nsel = warp_sum(nsel);
        if (lane == 0) {
            atomicAdd(&hdr->selected_pairs, (unsigned long long)nsel);
            atomicAdd(&hdr->scored_pairs, (unsigned long long)bt);
        }
    }
    if (no_conv) atomicOr(&hdr->status, kStNoConverge);
    __syncthreads();
    // compaction: thread tid owns words tid * kWpt .. + kWpt - 1
    unsigned wv[kWpt];
    int pc = 0;
#pragma unroll
    for (int k = 0; k < kWpt; ++k) {
        const int wi = tid * kWpt + k;
        wv[k] = wi < nw ? bitmap[wi] : 0u;
        pc += __popc(wv[k]);
    }
    int incl = pc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    int base = 0, total = 0;
    for (int w = 0; w < nwarp; ++w) {
        if (w < warp) base += wtot[w];
        total += wtot[w];
    }
    int pos = base + incl - pc;
    int* dst = list + (size_t)bg * cap;
#pragma unroll
    for (int k = 0; k < kWpt; ++k) {
        unsigned word = wv[k];
        const int wi = tid * kWpt + k;
        while (word) {
            const int bit = __ffs(word) - 1;
            dst[pos++] = wi * 32 + bit;
            word &= word - 1;
        }
    }
    if (tid == 0) {
        dst[total] = bt;                  // own block, always last
        count[bg] = total + 1;
        atomicAdd(&hdr->union_blocks, (unsigned long long)total);
        if (bt > 0) atomicAdd(&hdr->tiles, 1ull);
    }
    if (nctas > 0) decode_plan_tail(count, offs, plan, hdr, g.B * g.Hkv, nctas);
}

template <int D>
__device__ __forceinline__ int swz_d(int row, int c) { return row * D + ((c ^ (row & 7)) << 3); }

template <int D>
__global__ void __launch_bounds__(128)
decode_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                   const __nv_bfloat16* __restrict__ vc, const int* __restrict__ kv_len,
                   const float* __restrict__ xs, const float* __restrict__ tau,
                   const int* __restrict__ list, const int* __restrict__ count,
                   float* __restrict__ part, DecodeGeom g, float e_pow, float sm2) {
    constexpr int CH = D / 8;
    extern __shared__ uint4 smem_u4[];
    __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem_u4);   // [2][64][D]
    __nv_bfloat16* Vs = Ks + 2 * kBlock * D;                          // [2][64][D]
    float* qs = reinterpret_cast<float*>(Vs + 2 * kBlock * D);       // [G][D]
    float* os = qs + g.G * D;                                         // [G][D]
    float* ls = os + g.G * D;                                         // [G][64] logits, then p
    float* m_s = ls + g.G * kBlock;                                   // [G]
    float* l_s = m_s + 32;                                            // [G]
    float* sc_s = l_s + 32;                                           // [G]
    float* lp_s = sc_s + 32;                                          // [G]

    const int bg = blockIdx.x, b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int n = count[bg];
    const int e0 = blockIdx.y * g.chunk;
    if (e0 >= n) return;
    const int e1 = min(n, e0 + g.chunk);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = kv_len[b];
    const int t = L - 1, bt = t / kBlock;
    const int cap = g.nbs + 1;
    const int* lst = list + (size_t)bg * cap;
    const size_t row0 = (size_t)bg * g.Tmax;

    auto load_kv = [&](int e, int stage) {
        const int j = lst[e];
        for (int idx = tid; idx < kBlock * CH; idx += blockDim.x) {
            const int r = idx / CH, c = idx % CH;
            const int tok = j * kBlock + r;
            const bool ok = tok < L;
            const size_t off = (row0 + (ok ? tok : 0)) * D + c * 8;
            cp_async16(Ks + stage * kBlock * D + swz_d<D>(r, c), kc + off, ok ? 16 : 0);
            cp_async16(Vs + stage * kBlock * D + swz_d<D>(r, c), vc + off, ok ? 16 : 0);
        }
    };
    load_kv(e0, 0);
    cp_async_commit();
    for (int i = tid; i < g.G * D; i += blockDim.x) {
        qs[i] = __bfloat162float(q[(size_t)(b * g.Hq + kvh * g.G) * D + i]);
        os[i] = 0.f;
    }
    if (tid < g.G) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }

    for (int e = e0; e < e1; ++e) {
        const int stage = (e - e0) & 1;
        const int j = lst[e];
        const bool diag = (j == bt);
        if (e + 1 < e1) load_kv(e + 1, stage ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        if (tid < g.G) {
            const size_t row = (size_t)(b * g.Hq + kvh * g.G + tid);
            float lp = 0.f;
            if (!diag) {
                const float x = xs[row * cap + j], ta = tau[row];
                lp = x > ta ? e_pow * __log2f(x - ta) : -INFINITY;
            }
            lp_s[tid] = lp;
        }
        __syncthreads();
        const __nv_bfloat16* Kst = Ks + stage * kBlock * D;
        const __nv_bfloat16* Vst = Vs + stage * kBlock * D;
        // logits: thread -> (key, head parity)
        {
            const int key = tid & 63;
            const bool masked = diag && (j * kBlock + key > t);
            for (int hl = tid >> 6; hl < g.G; hl += 2) {
                float acc = 0.f;
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const uint4 u = *reinterpret_cast<const uint4*>(Kst + swz_d<D>(key, c));
                    float f[8];
                    bf16x8_to_float(u, f);
                    const float* qq = qs + hl * D + c * 8;
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc = fmaf(qq[i], f[i], acc);
                }
                const float lp = lp_s[hl];
                ls[hl * kBlock + key] = (masked || lp == -INFINITY) ? -INFINITY : fmaf(acc, sm2, lp);
            }
        }
        __syncthreads();
        // online softmax per head (one warp per head)
        for (int hl = warp; hl < g.G; hl += 4) {
            float a0 = ls[hl * kBlock + lane], a1 = ls[hl * kBlock + lane + 32];
            const float mx = warp_max(fmaxf(a0, a1));
            const float m_old = m_s[hl];
            const float m_new = fmaxf(m_old, mx);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            a0 = exp2f(a0 - m_use);
            a1 = exp2f(a1 - m_use);
            const float sum = warp_sum(a0 + a1);
            ls[hl * kBlock + lane] = a0;
            ls[hl * kBlock + lane + 32] = a1;
            __syncwarp();
            if (lane == 0) {
                const float sc = exp2f(m_old - m_use);
                sc_s[hl] = sc;
                l_s[hl] = l_s[hl] * sc + sum;
                m_s[hl] = m_new;
            }
        }
        __syncthreads();
        // O = O * scale + P V : thread -> (head, pair of dims)
        for (int pidx = tid; pidx < g.G * (D / 2); pidx += blockDim.x) {
            const int hl = pidx / (D / 2), dp = pidx % (D / 2);
            const int dim = dp * 2, c = dim >> 3, off = dim & 7;
            float ax = 0.f, ay = 0.f;
            const float* p = ls + hl * kBlock;
#pragma unroll 8
            for (int key = 0; key < kBlock; ++key) {
                const __nv_bfloat162 vv = *reinterpret_cast<const __nv_bfloat162*>(
                    Vst + key * D + (((c ^ (key & 7)) << 3) + off));
                const float2 vf = __bfloat1622float2(vv);
                ax = fmaf(p[key], vf.x, ax);
                ay = fmaf(p[key], vf.y, ay);
            }
            const float sc = sc_s[hl];
            os[hl * D + dim] = fmaf(os[hl * D + dim], sc, ax);
            os[hl * D + dim + 1] = fmaf(os[hl * D + dim + 1], sc, ay);
        }
        __syncthreads();
    }
    // partial (m, l, o) for every head of the group
    const size_t pbase = ((size_t)bg * g.maxchunks + blockIdx.y) * g.G;
    for (int i = tid; i < g.G * (D + 2); i += blockDim.x) {
        const int hl = i / (D + 2), c = i % (D + 2);
        const float val = c == 0 ? m_s[hl] : (c == 1 ? l_s[hl] : os[hl * D + c - 2]);
        part[(pbase + hl) * (D + 2) + c] = val;
    }
}

template <int D>
__global__ void __launch_bounds__(128)
decode_combine_kernel(const int* __restrict__ count, const float* __restrict__ part,
                      __nv_bfloat16* __restrict__ out, DecodeGeom g) {
    const int bh = blockIdx.x, b = bh / g.Hq, h = bh % g.Hq;
    const int kvh = h / g.G, hl = h % g.G, bg = b * g.Hkv + kvh;
    const int n = count[bg];
    const int nch = (n + g.chunk - 1) / g.chunk;
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c)
        M = fmaxf(M, part[(((size_t)bg * g.maxchunks + c) * g.G + hl) * (D + 2)]);
    const float Mu = M == -INFINITY ? 0.f : M;
    for (int dim = threadIdx.x; dim < D; dim += blockDim.x) {
        float num = 0.f, den = 0.f;
        for (int c = 0; c < nch; ++c) {
            const float* p = part + (((size_t)bg * g.maxchunks + c) * g.G + hl) * (D + 2);
            const float w = exp2f(p[0] - Mu);
            den = fmaf(p[1], w, den);
            num = fmaf(p[2 + dim], w, num);
        }
        out[(size_t)bh * D + dim] = __float2bfloat16(nch > 0 && den > 0.f ? num / den : 0.f);
    }
}

cudaError_t launch_decode(const void* q, const void* kc, const void* vc, const float* ksum,
                          const int* kv_len, void* out, const DecodeGeom& g, char* ws,
                          float alpha, float coarse_scale, cudaStream_t stream,
                          const cudaEvent_t* events, int agg, float* x_dump, float* p_dump) {
    auto mark = [&](int i) {
        return !events || cudaEventRecord(events[i], stream) == cudaSuccess;
    };
    const float cx = (alpha - 1.0f) * coarse_scale / sqrtf((float)g.d);
    const float e_pow = 1.0f / (alpha - 1.0f);
    const float sm2 = 1.4426950408889634f / sqrtf((float)g.d);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    float* xs = reinterpret_cast<float*>(ws + g.off_x);
    float* tau = reinterpret_cast<float*>(ws + g.off_tau);
    int* list = reinterpret_cast<int*>(ws + g.off_list);
    int* count = reinterpret_cast<int*>(ws + g.off_count);
    int* done = reinterpret_cast<int*>(ws + g.off_done);
    int* offs = reinterpret_cast<int*>(ws + g.off_offs);
    int* plan = reinterpret_cast<int*>(ws + g.off_plan);
    float* part = reinterpret_cast<float*>(ws + g.off_part);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(kc);
    const auto* vb = static_cast<const __nv_bfloat16*>(vc);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    const int BH = g.B * g.Hkv;
    const bool fused = decode_tc_supported(g);
    const int nctas = fused ? decode_tc_ctas() : 0;
    cudaError_t e = cudaSuccess;
    if (!mark(0)) return cudaErrorUnknown;
    if (g.d == 128) launch_scores<128>(qb, ksum, kv_len, xs, g, cx, stream);
    else launch_scores<64>(qb, ksum, kv_len, xs, g, cx, stream);
    // DASH_ENTMAX_INIT=histogram starts each threshold solve at the histogram edge; the
    // default, Newton from u = -1, is faster on the rows measured here (the binning pass
    // costs more than the passes it saves)
    const char* init = getenv("DASH_ENTMAX_INIT");
    const int hist_init = (init && strcmp(init, "histogram") == 0) ? 1 : 0;
    decode_select_kernel<<<BH, kSelThreads, 0, stream>>>(kv_len, xs, tau, list, count, done, offs, plan, ob, hdr, g,
                                                         alpha, nctas, hist_init);
    if (!mark(1)) return cudaErrorUnknown;
    if (fused) {
        e = launch_decode_attn_tc(q, kc, vc, kv_len, out, g, ws, e_pow, sm2, nctas, stream, agg, x_dump, p_dump);
        if (e != cudaSuccess) return e;
        if (!mark(2) || !mark(3)) return cudaErrorUnknown;   // no separate merge pass
        return cudaGetLastError();
    }
    // the CUDA-core path has per-head priors only and no parity dump
    if (agg || x_dump) return cudaErrorNotSupported;
    const size_t sm_attn = (size_t)4 * kBlock * g.d * sizeof(__nv_bfloat16)
                         + (size_t)(2 * g.G * g.d + g.G * kBlock + 4 * 32) * sizeof(float);
    e = g.d == 128
        ? cudaFuncSetAttribute(decode_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_attn)
        : cudaFuncSetAttribute(decode_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_attn);
    if (e != cudaSuccess) return e;
    dim3 ga(BH, g.maxchunks);
    if (g.d == 128)
        decode_attn_kernel<128><<<ga, 128, sm_attn, stream>>>(qb, kb, vb, kv_len, xs, tau, list, count, part, g, e_pow, sm2);
    else
        decode_attn_kernel<64><<<ga, 128, sm_attn, stream>>>(qb, kb, vb, kv_len, xs, tau, list, count, part, g, e_pow, sm2);
    if (!mark(2)) return cudaErrorUnknown;
    if (g.d == 128) decode_combine_kernel<128><<<g.B * g.Hq, 128, 0, stream>>>(count, part, ob, g);
    else decode_combine_kernel<64><<<g.B * g.Hq, 128, 0, stream>>>(count, part, ob, g);
    if (!mark(3)) return cudaErrorUnknown;
    return cudaGetLastError();
}

}  // namespace dash
