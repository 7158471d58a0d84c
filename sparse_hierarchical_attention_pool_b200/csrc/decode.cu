// decode.cu -- one decode step of DashAttention with a split-KV (flash-decoding) layout.
//
// Same arithmetic as a prefill row t = kv_len - 1 ("DashAttention: Making Sparse Attention
// Fully Differentiable with Adaptive Block Selection", section "Core Mechanism"): coarse
// scores over the cached block summaries of blocks j < bt = t / 64, alpha-entmax weights,
// then softmax over the selected blocks' tokens plus the own block (causal, prior 1) with
// log p as the prior.  Four kernels, all launched with shapes known on the host:
//   1. decode_scores : x[b, h, j] for every head of a KV group, one warp per block summary
//                      (the summary is read once for the whole group);
//   2. decode_select : per (b, kv head): one warp per head solves tau, the selected blocks
//                      of the group's heads are OR-ed into one list, the own block last;
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

template <int D>
__global__ void __launch_bounds__(256)
decode_scores_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ ksum,
                     const int* __restrict__ kv_len, float* __restrict__ xs, DecodeGeom g, float cx) {
    constexpr int VEC = D / 32;
    __shared__ float qs[32 * D];
    const int bg = blockIdx.x, b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int L = kv_len[b];
    if (L < 1 || L > g.Tmax) return;
    const int bt = (L - 1) / kBlock;
    const int j0 = blockIdx.y * 64;
    if (j0 >= bt) return;
    for (int i = threadIdx.x; i < g.G * D; i += blockDim.x)
        qs[i] = __bfloat162float(q[(size_t)(b * g.Hq + kvh * g.G) * D + i]);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cap = g.nbs + 1;
    for (int jj = warp; jj < 64; jj += 8) {
        const int j = j0 + jj;
        if (j >= bt) break;
        const float* kb = ksum + ((size_t)bg * g.nbs + j) * D + lane * VEC;
        float kv[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) kv[i] = __ldg(kb + i);
        for (int hl = 0; hl < g.G; ++hl) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < VEC; ++i) acc = fmaf(qs[hl * D + lane * VEC + i], kv[i], acc);
            acc = warp_sum(acc);
            if (lane == 0) xs[(size_t)(b * g.Hq + kvh * g.G + hl) * cap + j] = acc * cx;
        }
    }
}

struct GlobalRow {
    const float* p;
    __device__ __forceinline__ float operator()(int j) const { return p[j]; }
};

__global__ void __launch_bounds__(256)
decode_select_kernel(const int* __restrict__ kv_len, const float* __restrict__ xs,
                     float* __restrict__ tau, int* __restrict__ list, int* __restrict__ count,
                     WsHeader* __restrict__ hdr, DecodeGeom g, float alpha) {
    __shared__ unsigned bitmap[kMaxT / kBlock / 32];
    const int bg = blockIdx.x, b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    const int cap = g.nbs + 1;
    const int L = kv_len[b];
    if (L < 1 || L > g.Tmax) {
        if (threadIdx.x == 0) count[bg] = 0;
        return;
    }
    const int bt = (L - 1) / kBlock;
    const int nw = (bt + 31) / 32;
    for (int i = threadIdx.x; i < nw; i += blockDim.x) bitmap[i] = 0u;
    __syncthreads();
    int no_conv = 0;
    for (int hl = warp; hl < g.G; hl += nwarp) {
        const size_t row = (size_t)(b * g.Hq + kvh * g.G + hl);
        const float* xr = xs + row * cap;
        float t = __int_as_float(0x7fc00000);
        if (bt > 0) t = entmax_threshold<true>(GlobalRow{xr}, bt, alpha, &no_conv);
        if (lane == 0) tau[row] = t;
        float nsel = 0.f;
        for (int j = lane; j < bt; j += 32) {
            if (xr[j] > t) {
                nsel += 1.f;
                atomicOr(&bitmap[j >> 5], 1u << (j & 31));
            }
        }
        nsel = warp_sum(nsel);
        if (lane == 0) {
            atomicAdd(&hdr->selected_pairs, (unsigned long long)nsel);
            atomicAdd(&hdr->scored_pairs, (unsigned long long)bt);
        }
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
    decode_select_kernel<<<BH, 256, 0, stream>>>(kv_len, xs, tau, list, count, hdr, g, alpha);
    if (!mark(2)) return cudaErrorUnknown;
    if (g.d == 128) decode_attn_kernel<128><<<ga, 128, sm_attn, stream>>>(qb, kb, vb, kv_len, xs, tau, list, count, part, g, e_pow, sm2);
    else decode_attn_kernel<64><<<ga, 128, sm_attn, stream>>>(qb, kb, vb, kv_len, xs, tau, list, count, part, g, e_pow, sm2);
    if (!mark(3)) return cudaErrorUnknown;
    if (g.d == 128) decode_combine_kernel<128><<<g.B * g.Hq, 128, 0, stream>>>(count, part, ob, g);
    else decode_combine_kernel<64><<<g.B * g.Hq, 128, 0, stream>>>(count, part, ob, g);
    if (!mark(4)) return cudaErrorUnknown;
    return cudaGetLastError();
}

}  // namespace dash
