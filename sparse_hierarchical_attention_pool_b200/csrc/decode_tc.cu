// decode_tc.cu -- split-KV attention of a decode step, streaming the gathered K/V blocks with
// TMA and running the query heads of a KV group on the tensor cores.
//
// Same arithmetic as decode_attn_kernel in decode.cu ("DashAttention: Making Sparse
// Attention Fully Differentiable with Adaptive Block Selection", section "Core Mechanism",
// Stage 2): for every head of KV group (b, g) and every listed block j (the union of the
// group's selected blocks, the own block last), logits q . k / sqrt(d) + log p_j over the
// block's keys (own block: prior 1, keys <= t), online softmax, weighted sum of V.  HBM
// traffic is the listed K/V blocks, each read exactly once.
//
// Work split.  The groups' lists, laid end to end, hold U blocks; CTA c < n = min(grid, U)
// takes the contiguous range [U c / n, U (c + 1) / n), so every CTA streams the same number
// of blocks (at least one) whatever the list lengths.  A range may end inside one group and
// start inside the next; each (CTA, group) piece is a segment.  A group that lies inside one CTA is finished
// there; otherwise each covering CTA writes a partial (max, sum, output) to slot
// CTA + group (distinct for every segment, since both grow along the concatenation), and the
// CTA that brings the group's ticket counter to its number of pieces merges them.  The
// select pass leaves the prefix of the list lengths and, per CTA, the group its range
// starts in.
//
// Inside a CTA, warp 4 (one lane) streams 32-key halves of the listed blocks (K and V,
// 128-byte swizzled TMA boxes) into a 4-stage ring; consumer warp w (0-3) takes every 4th
// half and owns stage w.  Two CTAs share an SM, so one streams while the other sets up or
// merges.  A consumer computes the scores transposed, S^T = K Q^T, with mma.sync m16n8k16
// (the 32 keys are the M rows, the G <= 8 heads of the group the N columns), turns them into
// bf16 weights P^T, transposes those in registers (movmatrix) into the B operand of
// O^T += V^T P^T, and keeps its own online-softmax state; the four states are merged in
// shared memory at the end of every segment.  Block indices and log-priors of the segment
// are staged in shared memory 64 entries at a time.
// Parity dump (x_dump != nullptr, checks only): while staging, every listed past block's
// x_j and the weight p_j the prior applies (0 when x_j <= tau) are written per head to
// x_dump / p_dump [B Hq, Tmax / 64]; each (group, list entry) is staged by one CTA only.
#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"
#include "sm100.cuh"

namespace dash {

constexpr int kDtStages = 4;         // 32-key halves in flight per CTA (one per consumer warp)
constexpr int kDtMaxG = 8;           // query heads per KV group handled here (one n8 tile)
constexpr int kDtKeys = 32;          // keys per pipeline unit
constexpr int kDtTab = 64;           // list entries staged per table fill

template <int D>
struct DtLayout {
    static constexpr uint32_t kHalf = kDtKeys * 128;            // 32 keys x 64 bf16 (one TMA box)
    static constexpr uint32_t kPart = (D / 64) * kHalf;         // K or V of one unit
    static constexpr uint32_t kStage = 2 * kPart;               // K then V
    static constexpr uint32_t kQHalf = kDtMaxG * 128;           // 8 query rows x 64 bf16
    static constexpr uint32_t off_kv = 0;
    static constexpr uint32_t off_q = kDtStages * kStage;
    static constexpr uint32_t off_merge = off_q + (D / 64) * kQHalf;
    // per-warp states [warp][head][2 + D]; reused by the final merge for 2 x kDecodeMaxCtas x 8 floats
    static constexpr uint32_t merge_floats = 4 * kDtMaxG * (D + 2) > 2 * kDecodeMaxCtas * kDtMaxG
                                                 ? 4 * kDtMaxG * (D + 2) : 2 * kDecodeMaxCtas * kDtMaxG;
    static constexpr uint32_t off_tab = off_merge + merge_floats * 4;
    static constexpr uint32_t tab_bytes = kDtTab * kDtMaxG * 4 + kDtTab * 4;   // log-priors, block ids
    static constexpr uint32_t bytes = off_tab + tab_bytes + 1024;
};

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// The CTA whose range [U c / n, U (c + 1) / n) holds list position pos.
__device__ __forceinline__ int dt_cta_of(long long pos, long long U, int n) {
    return (int)(((pos + 1) * n - 1) / U);
}

template <int D>
__global__ void __launch_bounds__(160, 2)
decode_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __nv_bfloat16* __restrict__ q, const int* __restrict__ kv_len,
                      const float* __restrict__ xs, const float* __restrict__ tau,
                      const int* __restrict__ list, const int* __restrict__ offs,
                      const int* __restrict__ plan, float* __restrict__ part, int* __restrict__ done,
                      __nv_bfloat16* __restrict__ out, WsHeader* __restrict__ hdr, DecodeGeom g,
                      float e_pow, float sm2, int agg, float* __restrict__ x_dump, float* __restrict__ p_dump) {
    using L = DtLayout<D>;
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[kDtStages], empty[kDtStages];
    __shared__ int abort_sh;
    __shared__ int ticket_sh;
    __shared__ float wgt_sh[4][kDtMaxG], den_sh[kDtMaxG];
    const int BH = g.B * g.Hkv, cap = g.nbs + 1;
    const long long U = offs[BH];
    // ranges over n = min(grid, U) CTAs, so that every range is non-empty
    const int nC = (int)(U < (long long)gridDim.x ? U : (long long)gridDim.x), cta = blockIdx.x;
    if (cta >= nC) return;                           // whole CTA: nothing listed for it
    const int r_lo = (int)(U * cta / nC), r_hi = (int)(U * (cta + 1) / nC);
    const int bg_first = plan[cta];

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        abort_sh = 0;
        for (int s = 0; s < kDtStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        fence_mbar_init();
    }
    __syncthreads();
    volatile int* abort_flag = &abort_sh;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            long long cnt = 0;
            bool ok = true;
            for (int bg = bg_first, pos = r_lo; ok && pos < r_hi; ++bg) {
                const int o0 = offs[bg], o1 = offs[bg + 1];
                if (o1 <= pos) continue;
                const int seg_hi = min(r_hi, o1);
                for (int e = pos - o0; e < seg_hi - o0 && ok; ++e) {
                    const int j = list[(size_t)bg * cap + e];
                    for (int hk = 0; hk < 2; ++hk, ++cnt) {
                        const int st = (int)(cnt % kDtStages);
                        if (cnt >= kDtStages &&
                            !mbar_wait(smem_u32(&empty[st]), (uint32_t)(((cnt / kDtStages) - 1) & 1), abort_flag)) { ok = false; break; }
                        const int row = bg * g.Tmax + j * kBlock + hk * kDtKeys;
                        const uint32_t dst = base + L::off_kv + st * L::kStage;
                        mbar_arrive_expect_tx(smem_u32(&full[st]), L::kStage);
#pragma unroll
                        for (int h = 0; h < D / 64; ++h) {
                            tma_load_2d(dst + h * L::kHalf, &tm_k, h * 64, row, smem_u32(&full[st]));
                            tma_load_2d(dst + L::kPart + h * L::kHalf, &tm_v, h * 64, row, smem_u32(&full[st]));
                        }
                    }
                }
                pos = seg_hi;
            }
            if (!ok) {
                // let the copies already issued land before the CTA exits: units 0 .. cnt - 1
                // were issued, and stage s last carried unit cnt - 1 - ((cnt - 1 - s) mod stages)
                volatile int dummy = 0;
                for (int s = 0; s < kDtStages; ++s) {
                    if (cnt <= s) continue;
                    const long long last = cnt - 1 - ((cnt - 1 - s) % kDtStages);
                    dummy = 0;
                    mbar_wait(smem_u32(&full[s]), (uint32_t)((last / kDtStages) & 1), &dummy);
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumer warps 0-3
    const int g4 = lane >> 2, t4 = lane & 3;
    float* merge = reinterpret_cast<float*>(base_ptr + L::off_merge);   // [warp][head][D + 2]
    float* lptab = reinterpret_cast<float*>(base_ptr + L::off_tab);     // [entry][8] log2 priors
    int* jtab = reinterpret_cast<int*>(base_ptr + L::off_tab + kDtTab * kDtMaxG * 4);
    auto cons_sync = [&]() { asm volatile("bar.sync 1, 128;" ::: "memory"); };
    long long cnt = 0;
    bool ok = true;
    for (int bg = bg_first, pos = r_lo; pos < r_hi; ++bg) {
        const int o0 = offs[bg], o1 = offs[bg + 1];
        if (o1 <= pos) continue;
        const int seg_hi = min(r_hi, o1);
        const int e_lo = pos - o0, e_hi = seg_hi - o0;
        pos = seg_hi;
        const int b = bg / g.Hkv, kvh = bg % g.Hkv;
        const int t = kv_len[b] - 1, bt = t / kBlock;
        const size_t qrow0 = (size_t)b * g.Hq + (size_t)kvh * g.G;
        // the group's query rows, 128-byte swizzled like the K/V boxes; rows >= G are zero
        for (int idx = tid; idx < kDtMaxG * (D / 8); idx += 128) {
            const int r = idx / (D / 8), c = idx % (D / 8);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < g.G) v = *reinterpret_cast<const uint4*>(q + (qrow0 + r) * D + c * 8);
            *reinterpret_cast<uint4*>(base_ptr + L::off_q + (c >> 3) * L::kQHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = v;
        }
        cons_sync();
        // B operand Q^T (16 dims x 8 heads) of every 16-dim step
        uint32_t qb[D / 16][2];
#pragma unroll
        for (int k2 = 0; k2 < D / 32; ++k2) {
            const int r = lane & 7, c = k2 * 4 + (lane >> 3);
            ldsm_x4(qb[2 * k2][0], qb[2 * k2][1], qb[2 * k2 + 1][0], qb[2 * k2 + 1][1],
                    base + L::off_q + (c >> 3) * L::kQHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
        }
        // state of heads 2 t4 and 2 t4 + 1: running max, row sum over this lane's keys, and
        // O^T rows 16 dt + g4 and 16 dt + g4 + 8
        float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
        float o[D / 16][4];
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
            for (int c = 0; c < 4; ++c) o[dt][c] = 0.f;

        for (int i0 = e_lo; i0 < e_hi; i0 += kDtTab) {
            const int nsub = min(kDtTab, e_hi - i0);
            cons_sync();                               // the previous table is no longer read
            for (int idx = tid; idx < nsub * kDtMaxG; idx += 128) {
                const int i = idx / kDtMaxG, hl = idx % kDtMaxG;
                const int j = list[(size_t)bg * cap + i0 + i];
                float v2 = agg ? 0.f : -INFINITY;
                if (hl < g.G) {
                    if (j == bt) v2 = 0.f;
                    else {
                        const float x = xs[(qrow0 + hl) * cap + j];
                        const float tu = tau[qrow0 + hl];
                        // head aggregation keeps the weight itself for the average below
                        if (x > tu) v2 = agg ? exp2f(e_pow * __log2f(x - tu)) : e_pow * __log2f(x - tu);
                        if (x_dump) {
                            x_dump[(qrow0 + hl) * g.nbs + j] = x;
                            p_dump[(qrow0 + hl) * g.nbs + j] = x > tu ? exp2f(e_pow * __log2f(x - tu)) : 0.f;
                        }
                    }
                }
                lptab[idx] = v2;
                if (hl == 0) jtab[i] = j;
            }
            cons_sync();
            if (agg) {
                // the group's heads share log2 of their mean weight (own block: prior 1)
                for (int i = tid; i < nsub; i += 128) {
                    float pbar = 0.f;
                    for (int hl = 0; hl < g.G; ++hl) pbar += lptab[i * kDtMaxG + hl];
                    pbar *= 1.0f / (float)g.G;
                    const float v2 = jtab[i] == bt ? 0.f : (pbar > 0.f ? __log2f(pbar) : -INFINITY);
                    for (int hl = 0; hl < kDtMaxG; ++hl) lptab[i * kDtMaxG + hl] = hl < g.G ? v2 : -INFINITY;
                }
                cons_sync();
            }
            for (int i = 0; i < nsub; ++i) {
                if ((int)(cnt & 3) != warp && (int)((cnt + 1) & 3) != warp) { cnt += 2; continue; }
                const int j = jtab[i];
                const bool diag = (j == bt);
                const float2 lp = *reinterpret_cast<const float2*>(lptab + i * kDtMaxG + 2 * t4);
                for (int hk = 0; hk < 2; ++hk, ++cnt) {
                    if ((int)(cnt & 3) != warp) continue;
                    const int st = (int)(cnt % kDtStages);
                    const bool got = ok && mbar_wait(smem_u32(&full[st]), (uint32_t)((cnt / kDtStages) & 1), abort_flag);
                    if (!__all_sync(0xffffffffu, got)) { ok = false; continue; }
                    const uint32_t kst = base + L::off_kv + st * L::kStage;
                    const uint32_t vst = kst + L::kPart;
                    // S^T = K Q^T over two 16-key tiles
                    float s[2][4];
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int c = 0; c < 4; ++c) s[mt][c] = 0.f;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            uint32_t a[4];
                            const int key = mt * 16 + (lane & 15);
                            const int c = kk * 2 + (lane >> 4);
                            ldsm_x4(a[0], a[1], a[2], a[3], kst + (c >> 3) * L::kHalf + key * 128 + (((c & 7) ^ (key & 7)) << 4));
                            mma_bf16(s[mt], a, qb[kk][0], qb[kk][1]);
                        }
                    }
                    // logits in log2 units, causal mask on the own block, running max per head
                    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            float l2 = fmaf(s[mt][c], sm2, (c & 1) ? lp.y : lp.x);
                            if (diag) {
                                const int key = j * kBlock + hk * kDtKeys + mt * 16 + g4 + ((c >> 1) << 3);
                                if (key > t) l2 = -INFINITY;
                            }
                            s[mt][c] = l2;
                            if (c & 1) mx1 = fmaxf(mx1, l2); else mx0 = fmaxf(mx0, l2);
                        }
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                    }
                    const float mn0 = fmaxf(m_r[0], mx0), mn1 = fmaxf(m_r[1], mx1);
                    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
                    const float sc0 = exp2f(m_r[0] - mu0), sc1 = exp2f(m_r[1] - mu1);
                    m_r[0] = mn0; m_r[1] = mn1;
                    // P^T in bf16 (the row sums use the rounded weights the product uses),
                    // transposed into the B operand layout of the next product
                    uint32_t pb[2][2];
                    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t h = pack_bf16(exp2f(s[mt][2 * hh] - mu0), exp2f(s[mt][2 * hh + 1] - mu1));
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h));
                            ls0 += f.x;
                            ls1 += f.y;
                            pb[mt][hh] = movmatrix_trans(h);
                        }
                    l_r[0] = l_r[0] * sc0 + ls0;
                    l_r[1] = l_r[1] * sc1 + ls1;
#pragma unroll
                    for (int dt = 0; dt < D / 16; ++dt) {
                        o[dt][0] *= sc0; o[dt][1] *= sc1;
                        o[dt][2] *= sc0; o[dt][3] *= sc1;
                    }
                    // O^T += V^T P^T: two 16-key steps over D / 16 dim tiles
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
                        for (int dt = 0; dt < D / 16; ++dt) {
                            uint32_t a[4];
                            const int key = ks * 16 + (lane & 7) + ((lane >> 4) << 3);
                            const int c = dt * 2 + ((lane >> 3) & 1);
                            ldsm_x4_t(a[0], a[1], a[2], a[3], vst + (c >> 3) * L::kHalf + key * 128 + (((c & 7) ^ (key & 7)) << 4));
                            mma_bf16(o[dt], a, pb[ks][0], pb[ks][1]);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&empty[st]));
                }
            }
        }
        // ---- merge the four warps' states
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float l = l_r[hh];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            const int hl = 2 * t4 + hh;
            if (hl >= g.G) continue;
            float* mrow = merge + ((size_t)warp * kDtMaxG + hl) * (D + 2);
            if (g4 == 0) { mrow[0] = m_r[hh]; mrow[1] = l; }
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
                mrow[2 + dt * 16 + g4] = o[dt][hh];
                mrow[2 + dt * 16 + g4 + 8] = o[dt][2 + hh];
            }
        }
        cons_sync();
        const int c0 = dt_cta_of(o0, U, nC), c1 = dt_cta_of(o1 - 1, U, nC);
        const bool direct = (c0 == c1);
        const size_t slot = (size_t)cta + bg;
        if (tid < g.G) {
            float M = -INFINITY;
#pragma unroll
            for (int wv = 0; wv < 4; ++wv) M = fmaxf(M, merge[((size_t)wv * kDtMaxG + tid) * (D + 2)]);
            const float Mu = M == -INFINITY ? 0.f : M;
            float den = 0.f;
#pragma unroll
            for (int wv = 0; wv < 4; ++wv) {
                const float* mrow = merge + ((size_t)wv * kDtMaxG + tid) * (D + 2);
                const float w = mrow[0] == -INFINITY ? 0.f : exp2f(mrow[0] - Mu);
                wgt_sh[wv][tid] = w;
                den = fmaf(mrow[1], w, den);
            }
            den_sh[tid] = den;
            if (!direct) {
                part[(slot * g.G + tid) * (D + 2)] = M;
                part[(slot * g.G + tid) * (D + 2) + 1] = den;
            }
        }
        cons_sync();
        for (int idx = tid; idx < g.G * D; idx += 128) {
            const int hl = idx / D, dim = idx % D;
            float acc = 0.f;
#pragma unroll
            for (int wv = 0; wv < 4; ++wv) acc = fmaf(merge[((size_t)wv * kDtMaxG + hl) * (D + 2) + 2 + dim], wgt_sh[wv][hl], acc);
            if (direct) {
                const float den = den_sh[hl];
                out[(qrow0 + hl) * D + dim] = __float2bfloat16(den > 0.f ? acc / den : 0.f);
            } else {
                part[(slot * g.G + hl) * (D + 2) + 2 + dim] = acc;
            }
        }
        if (!direct) {
            // the CTA that writes the group's last piece merges all of them
            __threadfence();
            cons_sync();
            const int npieces = c1 - c0 + 1;
            if (tid == 0) ticket_sh = atomicAdd(&done[bg], 1);
            cons_sync();
            if (ticket_sh == npieces - 1) {
                __threadfence();
                float* mw = merge;                               // [piece][head] max, then weight
                float* lw = merge + kDecodeMaxCtas * kDtMaxG;    // [piece][head] sum
                const size_t s0 = (size_t)c0 + bg;
                for (int i = tid; i < npieces * g.G; i += 128) {
                    const float* pp = part + ((s0 + i / g.G) * g.G + i % g.G) * (D + 2);
                    mw[i] = __ldcg(pp);
                    lw[i] = __ldcg(pp + 1);
                }
                cons_sync();
                if (tid < g.G) {
                    float M = -INFINITY;
                    for (int pc = 0; pc < npieces; ++pc) M = fmaxf(M, mw[pc * g.G + tid]);
                    const float Mu = M == -INFINITY ? 0.f : M;
                    float den = 0.f;
                    for (int pc = 0; pc < npieces; ++pc) {
                        const float m = mw[pc * g.G + tid];
                        const float w = m == -INFINITY ? 0.f : exp2f(m - Mu);
                        mw[pc * g.G + tid] = w;
                        den = fmaf(lw[pc * g.G + tid], w, den);
                    }
                    den_sh[tid] = den > 0.f ? 1.f / den : 0.f;
                }
                cons_sync();
                for (int idx = tid; idx < g.G * D; idx += 128) {
                    const int hl = idx / D, dim = idx % D;
                    float acc = 0.f;
                    for (int pc = 0; pc < npieces; ++pc)
                        acc = fmaf(__ldcg(part + ((s0 + pc) * g.G + hl) * (D + 2) + 2 + dim), mw[pc * g.G + hl], acc);
                    out[(qrow0 + hl) * D + dim] = __float2bfloat16(acc * den_sh[hl]);
                }
            }
        }
        cons_sync();                                  // merge buffer and Q rows are reused
    }
    if (tid == 0 && *abort_flag) atomicOr(&hdr->status, kStWaitTimeout);
}

bool decode_tc_supported(const DecodeGeom& g) { return g.G <= kDtMaxG && (g.d == 64 || g.d == 128); }

int decode_tc_ctas() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n < 1) n = 148;
    n *= 2;                                       // two CTAs per SM (4-stage rings, ~87 KB each)
    return n < kDecodeMaxCtas ? n : kDecodeMaxCtas;
}

cudaError_t launch_decode_attn_tc(const void* q, const void* kc, const void* vc, const int* kv_len,
                                  void* out, const DecodeGeom& g, char* ws, float e_pow, float sm2,
                                  int nctas, cudaStream_t stream, int agg, float* x_dump, float* p_dump) {
    if (nctas < 1 || nctas > kDecodeMaxCtas) return cudaErrorInvalidValue;
    CUtensorMap tk, tv;
    const unsigned long long rows = (unsigned long long)g.B * g.Hkv * g.Tmax;
    if (!make_tmap_bf16(&tk, kc, rows, g.d, kDtKeys) || !make_tmap_bf16(&tv, vc, rows, g.d, kDtKeys)) return cudaErrorInvalidValue;
    const float* xs = reinterpret_cast<const float*>(ws + g.off_x);
    const float* tau = reinterpret_cast<const float*>(ws + g.off_tau);
    const int* list = reinterpret_cast<const int*>(ws + g.off_list);
    const int* offs = reinterpret_cast<const int*>(ws + g.off_offs);
    const int* plan = reinterpret_cast<const int*>(ws + g.off_plan);
    float* part = reinterpret_cast<float*>(ws + g.off_part);
    int* done = reinterpret_cast<int*>(ws + g.off_done);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    if (g.d == 128) {
        const int sm = (int)DtLayout<128>::bytes;
        cudaError_t e = cudaFuncSetAttribute(decode_attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        decode_attn_tc_kernel<128><<<nctas, 160, sm, stream>>>(tk, tv, qb, kv_len, xs, tau, list, offs, plan, part, done, ob, hdr, g, e_pow, sm2, agg, x_dump, p_dump);
    } else {
        const int sm = (int)DtLayout<64>::bytes;
        cudaError_t e = cudaFuncSetAttribute(decode_attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        decode_attn_tc_kernel<64><<<nctas, 160, sm, stream>>>(tk, tv, qb, kv_len, xs, tau, list, offs, plan, part, done, ob, hdr, g, e_pow, sm2, agg, x_dump, p_dump);
    }
    return cudaGetLastError();
}

}  // namespace dash
