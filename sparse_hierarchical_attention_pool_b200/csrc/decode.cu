// decode.cu -- one decode step of DashAttention with a split-KV (flash-decoding) layout.
//
// Same arithmetic as a prefill row t = kv_len - 1 ("DashAttention: Making Sparse Attention
// Fully Differentiable with Adaptive Block Selection", section "Core Mechanism"): coarse
// scores over the cached block summaries of blocks j < bt = t / 64, alpha-entmax weights,
// then softmax over the selected blocks' tokens plus the own block (causal, prior 1) with
// log p as the prior.  Four kernels, all launched with shapes known on the host:
//   1. decode_scores : x[b, h, j] for every head of a KV group, four threads per block
//                      summary (the summary is read once for the whole group);
//   2. decode_select : per (b, kv head): a team of warps per head solves tau with the row
//                      in registers, the selected blocks of the group's heads are OR-ed
//                      into one list, the own block last;
//   3. decode_attn   : split-KV over chunks of 16 listed blocks: K/V blocks (16 KB each at
//                      d = 128) stream through a two-stage cp.async pipeline; each listed
//                      block is read once and serves every head of the group; partial
//                      (max, sum, output) per chunk and head;
//   4. decode_combine: merges the partials of each (b, h) and writes bf16.
// The HBM traffic that matters is step 3: (union blocks + 1) * 64 * d * 2 bytes * 2 per
// (b, kv head).
#include "common.cuh"
#include "entmax.cuh"
#include "kernels.h"

namespace dash {

// Four threads per block summary, each holding a quarter of its d values (8 float4 loads
// issued together, so a CTA keeps 32 KB of summaries in flight); every head's partial dot
// product is reduced over the four threads with two shuffles.  The query rows of the group
// sit in shared memory with each quarter padded by one float4 so that the four quarters read
// in one instruction fall in different banks.
template <int D>
__global__ void __launch_bounds__(256)
decode_scores_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ ksum,
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
    if (j >= bt) {
#pragma unroll
        for (int i = 0; i < QV; ++i) kv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
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

constexpr int kSelRegs = 24;   // row values a select lane keeps in registers

// Row values of one head, spread over a team of W warps: lane tl of the team holds
// x[tl + k * 32W] for k < kSelRegs in registers; values past that are read from memory.
struct TeamRow {
    float r[kSelRegs];
    const float* p;
    int tl, stride, n;
    __device__ __forceinline__ void load(const float* row, int team_lane, int team_threads, int count) {
        p = row; tl = team_lane; stride = team_threads; n = count;
#pragma unroll
        for (int k = 0; k < kSelRegs; ++k) {
            const int j = tl + k * stride;
            r[k] = j < n ? row[j] : -INFINITY;
        }
    }
    template <class F>
    __device__ __forceinline__ void each(F&& f) const {
#pragma unroll
        for (int k = 0; k < kSelRegs; ++k) {
            const int j = tl + k * stride;
            if (j < n) f(j, r[k]);
        }
        for (int j = tl + kSelRegs * stride; j < n; j += stride) f(j, p[j]);
    }
};

// Work plan of the balanced attention pass, built by the last select CTA to finish (a
// ticket in the workspace header): offs = exclusive prefix of the list lengths (U = offs[BH]
// blocks in all), and plan[c] = the group holding position floor(U c / n), where CTA c's
// range starts (n = min(nctas, U)).  Called by every thread of every select CTA after its count is written.
__device__ void decode_plan_tail(const int* count, int* offs, int* plan, WsHeader* hdr, int BH, int nctas) {
    __shared__ int last_sh;
    __shared__ int wsum[8];
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
    const int lo = warp * slice, hi = min(BH, lo + slice);
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

// One CTA per (b, kv head).  The 8 warps form G teams (W = 8 / G warps each, one warp per
// head when G >= 8); a team solves its head's threshold with the row in registers, summing
// each pass over the team through shared memory (double-buffered, one named barrier per
// pass).  Selected blocks of all heads are OR-ed into a bitmap and compacted into the
// group's list, the own block last.
__global__ void __launch_bounds__(256)
decode_select_kernel(const int* __restrict__ kv_len, const float* __restrict__ xs,
                     float* __restrict__ tau, int* __restrict__ list, int* __restrict__ count,
                     int* __restrict__ done, int* __restrict__ offs, int* __restrict__ plan,
                     __nv_bfloat16* __restrict__ out, WsHeader* __restrict__ hdr, DecodeGeom g,
                     float alpha, int nctas) {
    __shared__ unsigned bitmap[kMaxT / kBlock / 32];
    __shared__ EntmaxPass red[2][8];
    __shared__ float redm[8];
    const int bg = blockIdx.x, b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    const int cap = g.nbs + 1;
    const int L = kv_len[b];
    if (threadIdx.x == 0) done[bg] = 0;
    if (L < 1 || L > g.Tmax) {
        // no keys: the group's heads get a zero output and no work
        if (threadIdx.x == 0) count[bg] = 0;
        __nv_bfloat16* o = out + ((size_t)b * g.Hq + (size_t)kvh * g.G) * g.d;
        for (int i = threadIdx.x; i < g.G * g.d; i += blockDim.x) o[i] = __float2bfloat16(0.f);
        if (nctas > 0) decode_plan_tail(count, offs, plan, hdr, g.B * g.Hkv, nctas);
        return;
    }
    const int bt = (L - 1) / kBlock;
    const int nw = (bt + 31) / 32;
    for (int i = threadIdx.x; i < nw; i += blockDim.x) bitmap[i] = 0u;
    __syncthreads();
    // team geometry: W warps per head (a power of two), nteam heads in flight
    int W = 1;
    while (W * 2 * g.G <= nwarp) W *= 2;
    const int nteam = nwarp / W, team = warp / W, tw = warp % W;
    const int tl = tw * 32 + lane, tthreads = W * 32;
    auto team_sync = [&]() {
        if (W > 1) asm volatile("bar.sync %0, %1;" :: "r"(team + 1), "r"(tthreads) : "memory");
    };
    int no_conv = 0;
    for (int hl = team; hl < g.G; hl += nteam) {
        const size_t row = (size_t)(b * g.Hq + kvh * g.G + hl);
        float t = __int_as_float(0x7fc00000);
        TeamRow xr;
        xr.load(xs + row * cap, tl, tthreads, bt);
        if (bt > 0) {
            float m = -INFINITY;
            xr.each([&](int, float v) { m = fmaxf(m, v); });
            m = warp_max(m);
            if (W > 1) {
                if (lane == 0) redm[warp] = m;
                team_sync();
                m = -INFINITY;
                for (int v = 0; v < W; ++v) m = fmaxf(m, redm[team * W + v]);
            }
            EntmaxSolver sv;
            sv.init(m, alpha);
            for (int pass = 0;; ++pass) {
                EntmaxPass ps;
                ps.reset();
                xr.each([&](int, float v) { ps.add((v - sv.m) - sv.u, sv.mode, sv.e); });
                ps.warp_reduce();
                if (W > 1) {
                    if (lane == 0) red[pass & 1][warp] = ps;
                    team_sync();
                    ps = red[pass & 1][team * W];
                    for (int v = 1; v < W; ++v) ps.merge(red[pass & 1][team * W + v]);
                }
                if (sv.update(ps, &t, &no_conv)) break;
            }
        }
        if (tw == 0 && lane == 0) tau[row] = t;
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
            if (tw == 0) atomicAdd(&hdr->scored_pairs, (unsigned long long)bt);
        }
        team_sync();                      // the team's reduction slots are reused by its next head
    }
    if (no_conv) atomicOr(&hdr->status, kStNoConverge);
    __syncthreads();
    if (warp == 0) {
        int base = 0;
        int* dst = list + (size_t)bg * cap;
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
            dst[base] = bt;                  // own block, always last
            count[bg] = base + 1;
            atomicAdd(&hdr->union_blocks, (unsigned long long)base);
            if (bt > 0) atomicAdd(&hdr->tiles, 1ull);
        }
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
                          const cudaEvent_t* events) {
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
    float* part = reinterpret_cast<float*>(ws + g.off_part);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(kc);
    const auto* vb = static_cast<const __nv_bfloat16*>(vc);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    const int BH = g.B * g.Hkv;
    dim3 gs(BH, (g.nbs + 63) / 64 > 0 ? (g.nbs + 63) / 64 : 1);
    const size_t sm_attn = (size_t)4 * kBlock * g.d * sizeof(__nv_bfloat16)
                         + (size_t)(2 * g.G * g.d + g.G * kBlock + 4 * 32) * sizeof(float);
    cudaError_t e = cudaSuccess;
    if (g.d == 128) e = cudaFuncSetAttribute(decode_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_attn);
    else e = cudaFuncSetAttribute(decode_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_attn);
    if (e != cudaSuccess) return e;
    dim3 ga(BH, g.maxchunks);
    if (!mark(0)) return cudaErrorUnknown;
    if (g.d == 128) decode_scores_kernel<128><<<gs, 256, 0, stream>>>(qb, ksum, kv_len, xs, g, cx);
    else decode_scores_kernel<64><<<gs, 256, 0, stream>>>(qb, ksum, kv_len, xs, g, cx);
    if (!mark(1)) return cudaErrorUnknown;
    int* done = reinterpret_cast<int*>(ws + g.off_done);
    int* offs = reinterpret_cast<int*>(ws + g.off_offs);
    int* plan = reinterpret_cast<int*>(ws + g.off_plan);
    const bool fused = decode_tc_supported(g);
    const int nctas = fused ? decode_tc_ctas() : 0;
    decode_select_kernel<<<BH, 256, 0, stream>>>(kv_len, xs, tau, list, count, done, offs, plan, ob, hdr, g,
                                                 alpha, nctas);
    if (!mark(2)) return cudaErrorUnknown;
    if (fused) {
        e = launch_decode_attn_tc(q, kc, vc, kv_len, out, g, ws, e_pow, sm2, nctas, stream);
        if (e != cudaSuccess) return e;
    } else if (g.d == 128) {
        decode_attn_kernel<128><<<ga, 128, sm_attn, stream>>>(qb, kb, vb, kv_len, xs, tau, list, count, part, g, e_pow, sm2);
    } else {
        decode_attn_kernel<64><<<ga, 128, sm_attn, stream>>>(qb, kb, vb, kv_len, xs, tau, list, count, part, g, e_pow, sm2);
    }
    if (!mark(3)) return cudaErrorUnknown;
    // the tensor-core attention kernel merges the chunk partials itself
    if (!fused) {
        if (g.d == 128) decode_combine_kernel<128><<<g.B * g.Hq, 128, 0, stream>>>(count, part, ob, g);
        else decode_combine_kernel<64><<<g.B * g.Hq, 128, 0, stream>>>(count, part, ob, g);
    }
    if (!mark(4)) return cudaErrorUnknown;
    return cudaGetLastError();
}

}  // namespace dash
