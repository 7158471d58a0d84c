// backward_tc.cu -- the query-major half of the prefill backward on the 5th-generation
// tensor cores (tcgen05 + TMEM + TMA): per-row statistics, then dq.
//
// "DashAttention: Making Sparse Attention Fully Differentiable with Adaptive Block
// Selection", sections "Core Mechanism" and "Key Concepts".  The arithmetic is the one
// backward.cu states; for row (b, h, t) with log2-domain logits l_i = s_i log2(e)/sqrt(d)
// + log2 p_j(i) and LSE = log2 sum_i 2^l_i:
//   pass 1 (MODE 0, statistics):  LSE, S1 = sum_j g_j and S2 = sum_j H_j, H_j = c_j/(x_j - tau),
//     c_j = sum_{i in j} P_i (dP_i - D), so r = S2 / S1.  c_j needs the final LSE, so each step
//     keeps c^_j = sum_{i in j} 2^(l_i - m) (dP_i - D) relative to the running maximum m of the
//     logits and S2^ = sum_j 2^(m_j - m) c^_j / (x_j - tau) is rescaled with m like the softmax
//     denominator l; at the end S2 = S2^ / l.
//   pass 2 (MODE 1, dq):  P_i = 2^(l_i - LSE), dS_i = P_i (dP_i - D), c_j = sum_{i in j} dS_i,
//     ds_j = c_j/(x_j - tau) - r g_j, dq = (1/sqrt(d)) sum_i (dS_i + cs ds_j(i) / 64) k_i.
//     With r known before the pass, the whole coarse-path gradient of q (the alpha-entmax
//     Jacobian through the scores into q) folds into the dS operand of one product.
// x_j comes, as in the forward's tcgen05 kernel, from two summary columns of the S product
// (block j's summary split into bf16 hi and lo parts appended to the K tile as rows 64 and 72).
//
// One CTA per 128-row work tile, the tile's steps (listed blocks, then the own block) dealt
// alternately to two softmax groups of four warps (one thread per tile row).  Warps:
//   8   TMA producer (one lane): the Q and dout tiles once, then K (+ summary rows) and V of
//       every step, a ring of 4 (MODE 0) or 3 (MODE 1) stages;
//   9   S issuer (one lane): S_s = Q [K_s | kbar_hi | kbar_lo]^T (M=128, N=80) and
//       dP_s = dout V_s^T (M=128, N=64) into the buffers of group s & 1, as soon as the stage
//       is loaded and the group has read its previous S and dP;
//   10  dq issuer (one lane, MODE 1): dq += dS_s K_s (M=128, N=d; K MN-major) as soon as
//       the group has written dS_s; frees the stage;
//   0-7 softmax groups.
// Operands: Q, dout, K, V (for S and dP) and dS K-major; K (for dq) MN-major; 128-byte
// swizzle everywhere (TMA writes it).  Every wait is bounded (~2 s); a CTA that gives up
// sets a status bit, lets its copies and products finish, frees TMEM and exits.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace dash {

template <int D, int MODE>
struct BtLayout {
    static constexpr int kStages = MODE == 0 ? 4 : 3;
    static constexpr uint32_t kQHalf = 128 * 128;               // 128 rows x 64 bf16
    static constexpr uint32_t kQ = (D / 64) * kQHalf;
    static constexpr uint32_t kKRows = 80;                      // 64 keys, kbar hi atom, kbar lo atom
    static constexpr uint32_t kKHalf = kKRows * 128;
    static constexpr uint32_t kK = (D / 64) * kKHalf;
    static constexpr uint32_t kVHalf = 64 * 128;
    static constexpr uint32_t kV = (D / 64) * kVHalf;
    static constexpr uint32_t kStage = kK + kV;
    static constexpr uint32_t kP = 128 * 128;                   // dS: 128 rows x 64 keys bf16
    static constexpr uint32_t off_q = 0;
    static constexpr uint32_t off_do = kQ;
    static constexpr uint32_t off_kv = 2 * kQ;
    static constexpr uint32_t off_ds = off_kv + kStages * kStage;
    static constexpr uint32_t bytes = off_ds + (MODE == 1 ? 2 * kP : 0) + 1024;   // + alignment slack
    // TMEM columns: S of group g at 96 g (80 used), dP of group g at 192 + 64 g, dq at 320
    static constexpr uint32_t colS = 96;
    static constexpr uint32_t colDP = 192;
    static constexpr uint32_t colQ = 320;
};

struct BtConsts {
    float cx;      // (alpha-1) cs / sqrt(d): q . kbar_j -> x_j
    float e_pow;   // 1 / (alpha-1)
    float gpow;    // (2-alpha) / (alpha-1)
    float sm2;     // log2(e) / sqrt(d)
    float cs64;    // cs / 64
    float isd;     // 1 / sqrt(d)
};

enum : int { BT_Q = 0, BT_KV_FULL = 1, BT_KV_EMPTY = 5, BT_S_FULL = 9, BT_S_FREE = 11, BT_P_FULL = 13,
             BT_PV_DONE = 15, BT_DRAIN = 17, BT_DRAIN2 = 18, BT_COUNT = 19 };

template <int D, int MODE>
__global__ void __launch_bounds__(352, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
              __nv_bfloat16* __restrict__ dq, float* __restrict__ lse, float* __restrict__ rrow,
              const float* __restrict__ drow, const float* __restrict__ tau, const int* __restrict__ list,
              const int* __restrict__ count, WsHeader* __restrict__ hdr, PrefillGeom g, BtConsts C) {
    using L = BtLayout<D, MODE>;
    using namespace sm100;
    constexpr int kStages = L::kStages;
    constexpr int kProducerWarp = 8, kMmaSWarp = 9, kMmaQWarp = 10;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[BT_COUNT];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ float4 stat_sh[MODE == 0 ? 2 : 1][kTileRows];   // per group: (m, l, S2^, S1)

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto kv_addr = [&](int st) { return base + L::off_kv + (uint32_t)st * L::kStage; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // group-major order, longest tiles of a KV group first (its K and V stay in L2)
    const int w = blockIdx.x;
    const int bg = w / g.ntile_bg;
    const int it = g.ntile_bg - 1 - w % g.ntile_bg;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int t0 = it * g.P;
    const int bt = t0 / kBlock;
    const size_t tile_id = (size_t)bg * g.ntile_bg + it;
    const int U = bt > 0 ? count[tile_id] : 0;
    const int n = U + 1;
    const int* lst = list + tile_id * g.cap;

    if (tid == 0) {
        abort_sh = 0;
        mbar_init(bar(BT_Q), 1);
        for (int st = 0; st < kStages; ++st) {
            mbar_init(bar(BT_KV_FULL + st), 1);
            mbar_init(bar(BT_KV_EMPTY + st), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BT_S_FULL + i), 1);
            mbar_init(bar(BT_S_FREE + i), 128);
            mbar_init(bar(BT_P_FULL + i), 128);
            mbar_init(bar(BT_PV_DONE + i), 1);
        }
        mbar_init(bar(BT_DRAIN), 1);
        mbar_init(bar(BT_DRAIN2), 1);
        fence_mbar_init();
    }
    // rows of the Q and dout tiles beyond G * P are never loaded: zero them once
    if (g.M < kTileRows && tid < kTileRows && tid >= g.M) {
        for (int h = 0; h < D / 64; ++h) {
            uint4* p = reinterpret_cast<uint4*>(base_ptr + L::off_q + h * L::kQHalf + tid * 128);
            uint4* p2 = reinterpret_cast<uint4*>(base_ptr + L::off_do + h * L::kQHalf + tid * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) { p[c] = make_uint4(0u, 0u, 0u, 0u); p2[c] = make_uint4(0u, 0u, 0u, 0u); }
        }
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(smem_u32(&tmem_base_sh), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int* abort_flag = &abort_sh;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_do);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_hi);
            prefetch_tmap(&tm_lo);
            mbar_arrive_expect_tx(bar(BT_Q), (uint32_t)(2 * g.M * D * 2));
            for (int hl = 0; hl < g.G; ++hl) {
                const int row = (b * g.Hq + kvh * g.G + hl) * g.T + t0;
                for (int h = 0; h < D / 64; ++h) {
                    tma_load_2d(base + L::off_q + h * L::kQHalf + hl * g.P * 128, &tm_q, h * 64, row, bar(BT_Q));
                    tma_load_2d(base + L::off_do + h * L::kQHalf + hl * g.P * 128, &tm_do, h * 64, row, bar(BT_Q));
                }
            }
            int last_armed[kStages];
            for (int st = 0; st < kStages; ++st) last_armed[st] = -1;
            for (int s = 0; s < n; ++s) {
                const int st = s % kStages;
                if (s >= kStages && !mbar_wait(bar(BT_KV_EMPTY + st), ((s / kStages) - 1) & 1, abort_flag)) break;
                const int j = s < U ? lst[s] : bt;
                const int row = bg * g.T + j * kBlock;
                // summary atoms of block j (the own block reads a neighbour's; its x is unused)
                const int srow = g.nbs > 0 ? bg * g.nbs + min(j, g.nbs - 1) : 0;
                mbar_arrive_expect_tx(bar(BT_KV_FULL + st), (uint32_t)((2 * kBlock + 16) * D * 2));
                for (int h = 0; h < D / 64; ++h) {
                    tma_load_2d(kv_addr(st) + h * L::kKHalf, &tm_k, h * 64, row, bar(BT_KV_FULL + st));
                    tma_load_2d(kv_addr(st) + h * L::kKHalf + 64 * 128, &tm_hi, h * 64, srow, bar(BT_KV_FULL + st));
                    tma_load_2d(kv_addr(st) + h * L::kKHalf + 72 * 128, &tm_lo, h * 64, srow, bar(BT_KV_FULL + st));
                    tma_load_2d(kv_addr(st) + L::kK + h * L::kVHalf, &tm_v, h * 64, row, bar(BT_KV_FULL + st));
                }
                last_armed[st] = s;
            }
            if (*abort_flag) {
                volatile int dummy = 0;
                mbar_wait(bar(BT_Q), 0, &dummy);
                for (int st = 0; st < kStages; ++st)
                    if (last_armed[st] >= 0) { dummy = 0; mbar_wait(bar(BT_KV_FULL + st), (last_armed[st] / kStages) & 1, &dummy); }
            }
        }
    } else if (warp == kMmaSWarp) {
        // ------------------------------------------------------------ S and dP issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16(128, L::kKRows, false);
            const uint32_t idesc_p = idesc_bf16(128, 64, false);
            bool ok = mbar_wait(bar(BT_Q), 0, abort_flag);
            for (int s = 0; ok && s < n; ++s) {
                const int st = s % kStages, sb = s & 1;
                if (!mbar_wait(bar(BT_KV_FULL + st), (s / kStages) & 1, abort_flag)) { ok = false; break; }
                if (s >= 2 && !mbar_wait(bar(BT_S_FREE + sb), ((s - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int h = kk >> 2, wk = kk & 3;
                    const uint64_t a = smem_desc_sw128(base + L::off_q + h * L::kQHalf + wk * 32, 16, 1024);
                    const uint64_t bk = smem_desc_sw128(kv_addr(st) + h * L::kKHalf + wk * 32, 16, 1024);
                    mma_bf16_ss(tmem + sb * L::colS, a, bk, idesc_s, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int h = kk >> 2, wk = kk & 3;
                    const uint64_t a = smem_desc_sw128(base + L::off_do + h * L::kQHalf + wk * 32, 16, 1024);
                    const uint64_t bv = smem_desc_sw128(kv_addr(st) + L::kK + h * L::kVHalf + wk * 32, 16, 1024);
                    mma_bf16_ss(tmem + L::colDP + sb * 64, a, bv, idesc_p, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(BT_S_FULL + sb));
                if constexpr (MODE == 0) mma_commit(bar(BT_KV_EMPTY + st));   // the stage's last reader
            }
            if (!ok) {
                mma_commit(bar(BT_DRAIN));
                volatile int dummy = 0;
                mbar_wait(bar(BT_DRAIN), 0, &dummy);
            }
        }
    } else if (warp == kMmaQWarp) {
        // ------------------------------------------------------------ dq issuer
        if constexpr (MODE == 1) {
            if (lane == 0) {
                const uint32_t idesc_q = idesc_bf16(128, D, true);
                bool ok = true;
                for (int p = 0; p < n; ++p) {
                    const int bp = p & 1, stp = p % kStages;
                    if (!mbar_wait(bar(BT_P_FULL + bp), (p >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a = smem_desc_sw128(base + L::off_ds + bp * L::kP + kk * 32, 16, 1024);
                        const uint64_t bk = smem_desc_sw128(kv_addr(stp) + kk * 2048, L::kKHalf, 1024);
                        mma_bf16_ss(tmem + L::colQ, a, bk, idesc_q, (p > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar(BT_PV_DONE + bp));
                    mma_commit(bar(BT_KV_EMPTY + stp));
                }
                if (!ok) {
                    mma_commit(bar(BT_DRAIN2));
                    volatile int dummy = 0;
                    mbar_wait(bar(BT_DRAIN2), 0, &dummy);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax groups
        const int grp = warp >> 2, quarter = warp & 3;
        const int r = quarter * 32 + lane;                  // tile row = TMEM lane
        const int hl = r / g.P, t = t0 + r % g.P;
        const bool valid = r < g.M && t < g.T;
        const int tpos = valid ? t : -1;
        const size_t rowid = valid ? (size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t : 0;
        const float tau_r = (valid && bt > 0) ? tau[rowid] : INFINITY;
        const float drow_r = valid ? drow[rowid] : 0.f;
        const float lse_r = (MODE == 1 && valid) ? lse[rowid] : 0.f;
        const float rr = (MODE == 1 && valid) ? rrow[rowid] : 0.f;
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t s_col = grp * L::colS, p_col = L::colDP + grp * 64;
        uint8_t* const drow_sm = base_ptr + L::off_ds + grp * L::kP + (r >> 3) * 1024 + (r & 7) * 128;
        float m_run = -INFINITY, l_run = 0.f, s2 = 0.f, s1 = 0.f;   // statistics (MODE 0)
        bool ok = true;
        // TMEM loads are warp-collective: every wait result is made warp-uniform
        auto wwait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
            const bool got = mbar_wait(bar_addr, parity, abort_flag);
            return __all_sync(0xffffffffu, got);
        };
        for (int s = grp; s < n; s += 2) {
            const int i2 = s >> 1;
            const int j = s < U ? lst[s] : bt;
            const bool diag = (j == bt);
            if (!(ok && wwait(bar(BT_S_FULL + grp), i2 & 1))) { ok = false; continue; }
            tc_fence_after();
            uint32_t sr[64];
            tmem_ld<64>(lane_addr + s_col, sr);
            const uint32_t qhi = tmem_ld1(lane_addr + s_col + 64);
            const uint32_t qlo = tmem_ld1(lane_addr + s_col + 72);
            tmem_wait_ld();
            const float x = __fmul_rn(__uint_as_float(qhi) + __uint_as_float(qlo), C.cx);
            const float xm = x - tau_r;
            const bool sel = !diag && x > tau_r;
            const float lx = sel ? __log2f(xm) : 0.f;
            const float lp2 = diag ? (tpos >= 0 ? 0.f : -INFINITY) : (sel ? C.e_pow * lx : -INFINITY);
            if (diag) {
                const int key0 = j * kBlock;
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (key0 + i > tpos) sr[i] = __float_as_uint(-INFINITY);
            }
            if constexpr (MODE == 0) {
                // logits, running maximum, denominator, and c^ from dP in two halves
                float mx = -INFINITY;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const float l2 = fmaf(__uint_as_float(sr[i]), C.sm2, lp2);
                    sr[i] = __float_as_uint(l2);
                    mx = fmaxf(mx, l2);
                }
                const float m_new = fmaxf(m_run, mx);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                const float scale = exp2f(m_run - m_use);
                float ls = 0.f, ch = 0.f;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t dp[32];
                    tmem_ld<32>(lane_addr + p_col + hh * 32, dp);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float e = fast_exp2(__uint_as_float(sr[hh * 32 + i]) - m_use);
                        ls += e;
                        ch = fmaf(e, __uint_as_float(dp[i]) - drow_r, ch);
                    }
                }
                tc_fence_before();
                mbar_arrive(bar(BT_S_FREE + grp));
                l_run = l_run * scale + ls;
                s2 = s2 * scale + (sel ? ch / xm : 0.f);
                s1 += sel ? exp2f(C.gpow * lx) : 0.f;
                m_run = m_new;
            } else {
                // dS = P (dP - D) with the final log-sum-exp, c_j, the entmax fold, dS to shared
                const float c0 = lp2 - lse_r;
                float cj = 0.f;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t dp[32];
                    tmem_ld<32>(lane_addr + p_col + hh * 32, dp);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float p = fast_exp2(fmaf(__uint_as_float(sr[hh * 32 + i]), C.sm2, c0));
                        const float ds = p * (__uint_as_float(dp[i]) - drow_r);
                        sr[hh * 32 + i] = __float_as_uint(ds);
                        cj += ds;
                    }
                }
                tc_fence_before();
                mbar_arrive(bar(BT_S_FREE + grp));
                const float f = sel ? C.cs64 * (cj / xm - rr * exp2f(C.gpow * lx)) : 0.f;
                // the dS buffer of this group was last read by its previous dq product
                if (i2 >= 1 && !wwait(bar(BT_PV_DONE + grp), (i2 - 1) & 1)) { ok = false; continue; }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t pk[4];
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(sr[c * 8 + 2 * q2]) + f,
                                                                  __uint_as_float(sr[c * 8 + 2 * q2 + 1]) + f);
                        pk[q2] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    *reinterpret_cast<uint4*>(drow_sm + ((c ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar(BT_P_FULL + grp));
            }
        }
        if constexpr (MODE == 0) {
            // merge the two groups' statistics; group 0 writes LSE and r of its row
            stat_sh[grp][r] = make_float4(m_run, l_run, s2, s1);
            asm volatile("bar.sync %0, %1;" :: "r"(9), "n"(256) : "memory");
            if (grp == 0 && valid && ok) {
                const float4 a = stat_sh[0][r], c = stat_sh[1][r];
                const float M = fmaxf(a.x, c.x);
                const float wa = a.x == -INFINITY ? 0.f : exp2f(a.x - M);
                const float wc = c.x == -INFINITY ? 0.f : exp2f(c.x - M);
                const float l = a.y * wa + c.y * wc;
                const float S2 = (a.z * wa + c.z * wc) / l;
                const float S1 = a.w + c.w;
                lse[rowid] = M + __log2f(l);
                rrow[rowid] = S1 > 0.f ? S2 / S1 : 0.f;
            }
        } else {
            // dq is final once both groups' last products are done (products complete in
            // issue order); each group stores half of the row's columns
            const int last = grp + 2 * ((n - 1 - grp) >> 1);   // this group's last step
            bool done = ok;
            if (grp < n) done = done && wwait(bar(BT_PV_DONE + grp), (last >> 1) & 1);
            asm volatile("bar.sync %0, %1;" :: "r"(9), "n"(256) : "memory");
            if (done) {
                tc_fence_after();
                constexpr int HC = D / 2;
                constexpr int CW = HC < 32 ? HC : 32;
                __nv_bfloat16* dst = valid ? dq + rowid * D + grp * HC : nullptr;
#pragma unroll
                for (int c = 0; c < HC / CW; ++c) {
                    uint32_t o[CW];
                    tmem_ld<CW>(lane_addr + L::colQ + grp * HC + c * CW, o);
                    tmem_wait_ld();
                    if (valid) {
                        uint32_t pk[CW / 2];
#pragma unroll
                        for (int i = 0; i < CW / 2; ++i) {
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * C.isd,
                                                                      __uint_as_float(o[2 * i + 1]) * C.isd);
                            pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                        }
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c * CW);
#pragma unroll
                        for (int i = 0; i < CW / 8; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (tid == 0 && abort_sh) atomicOr(&hdr->status, kStWaitTimeout);
}

// ------------------------------------------------------------------ key-major: dk, dv
//
// One CTA per (b, KV head, pair of key blocks j0 = 2 jp, j1 = 2 jp + 1): the 128 keys of
// the pair are the M dimension of the dk and dv products.  The steps are the work tiles
// whose own block is j0 or j1 or whose list holds j0 or j1, ascending; each carries, per
// block, whether the block is the tile's own block (causal), a listed past block, or
// neither (nothing to add).  Per step:
//   S  = Q [K_j0; K_j1]^T    (M = 128 rows, N = 128 keys)   rows in TMEM lanes, so the
//   dP = dout [V_j0; V_j1]^T                                 per-row block sums (x_j from
//                                                            S, c_j from dS) stay in-thread
//   dV += P^T dout, dK += (dS + cs ds_j / 64)^T Q  (M = 128 keys, N = d, K = 128 rows):
//        P and dS are written row-major ([row][key], bf16) and read as MN-major A.
// Warps: 8 producer (the pair's K and V once; per step the Q and dout tiles into a
// two-stage ring; it also finds the steps: each lane tests one candidate tile -- own block,
// or a binary search of the tile's sorted list -- and a warp ballot keeps them in order;
// a sentinel step ends the loop), 9 S/dP issuer, 10 dK/dV issuer, 0-7 softmax (thread =
// (row, block of the pair): warp w serves TMEM lanes 32 (w % 4).. and block w / 4).
// P and dS share one buffer: dS is written once dV has read P.
template <int D>
struct BkLayout {
    static constexpr uint32_t kHalf = 128 * 128;                // 128 rows x 64 bf16 (one swizzle column)
    static constexpr uint32_t kT = (D / 64) * kHalf;            // a 128-row [rows][D] tile
    static constexpr uint32_t off_k = 0;                        // K of the pair [128 keys][D]
    static constexpr uint32_t off_v = kT;
    static constexpr uint32_t off_ring = 2 * kT;                // stage: Q tile, dout tile
    static constexpr uint32_t kStage = 2 * kT;
    static constexpr uint32_t off_buf = off_ring + 2 * kStage;  // P / dS [2 key halves][128 rows][64]
    static constexpr uint32_t bytes = off_buf + 2 * kHalf + 1024;
    static constexpr uint32_t colS = 0, colDP = 128, colDV = 256, colDK = 256 + D;
};

enum : int { BK_KV = 0, BK_QF = 1, BK_QE = 3, BK_S_FULL = 5, BK_S_FREE = 6, BK_P_FULL = 7, BK_DV_DONE = 8,
             BK_DS_FULL = 9, BK_DK_DONE = 10, BK_DRAIN = 11, BK_DRAIN2 = 12, BK_COUNT = 13 };
enum : int { kModeNone = 0, kModePast = 1, kModeDiag = 2 };

// kind::f16 instruction descriptor with either operand MN-major (bit 15: A, bit 16: B)
__host__ __device__ constexpr uint32_t idesc_bf16_ab(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct BkConsts {
    float cxm;     // (alpha-1) cs / sqrt(d) / 64: row sum of S over a block -> x_j
    float e_pow, gpow, sm2, cs64, isd;
};

template <int D>
__global__ void __launch_bounds__(352, 1)
bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                  const float* __restrict__ lse, const float* __restrict__ rrow, const float* __restrict__ drow,
                  const float* __restrict__ tau, const int* __restrict__ list, const int* __restrict__ count,
                  WsHeader* __restrict__ hdr, PrefillGeom g, BkConsts C) {
    using L = BkLayout<D>;
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[BK_COUNT];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ int info_sh[2];                 // per ring stage: tile | mode0 << 24 | mode1 << 26, or -1

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto q_addr = [&](int st) { return base + L::off_ring + (uint32_t)st * L::kStage; };
    auto do_addr = [&](int st) { return base + L::off_ring + (uint32_t)st * L::kStage + L::kT; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // group-major order: the CTAs in flight share one KV group, whose Q and dout tiles stay
    // in L2 while its pairs re-read them; within a group, low pairs (listed by the most
    // tiles) first
    const int nb = (g.T + kBlock - 1) / kBlock;
    const int npairs = (nb + 1) / 2;
    const int bg = blockIdx.x / npairs;
    const int jp = blockIdx.x % npairs;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int j0 = 2 * jp, j1 = 2 * jp + 1;
    const bool has1 = j1 < nb;

    if (tid == 0) {
        abort_sh = 0;
        mbar_init(bar(BK_KV), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BK_QF + i), 1);
            mbar_init(bar(BK_QE + i), 1);
        }
        mbar_init(bar(BK_S_FULL), 1);
        mbar_init(bar(BK_S_FREE), 256);
        mbar_init(bar(BK_P_FULL), 256);
        mbar_init(bar(BK_DV_DONE), 1);
        mbar_init(bar(BK_DS_FULL), 256);
        mbar_init(bar(BK_DK_DONE), 1);
        mbar_init(bar(BK_DRAIN), 1);
        mbar_init(bar(BK_DRAIN2), 1);
        fence_mbar_init();
    }
    // rows of the Q and dout tiles beyond G * P are never loaded: zero them in both stages
    if (g.M < kTileRows && tid < kTileRows && tid >= g.M) {
        for (int st = 0; st < 2; ++st)
            for (int h = 0; h < 2 * (D / 64); ++h) {
                uint4* p = reinterpret_cast<uint4*>(base_ptr + L::off_ring + st * L::kStage + h * L::kHalf + tid * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) p[c] = make_uint4(0u, 0u, 0u, 0u);
            }
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(smem_u32(&tmem_base_sh), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int* abort_flag = &abort_sh;

    if (warp == 8) {
        // ------------------------------------------------------------ producer and step finder
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_do);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            // K and V of the pair; a missing second block reads rows that are never used
            // (finite data of the next rows, or zeros past the end of the tensor)
            mbar_arrive_expect_tx(bar(BK_KV), (uint32_t)(4 * kBlock * D * 2));
            for (int h = 0; h < D / 64; ++h)
                for (int jb = 0; jb < 2; ++jb) {
                    const int row = bg * g.T + (j0 + jb) * kBlock;
                    tma_load_2d(base + L::off_k + h * L::kHalf + jb * 64 * 128, &tm_k, h * 64, row, bar(BK_KV));
                    tma_load_2d(base + L::off_v + h * L::kHalf + jb * 64 * 128, &tm_v, h * 64, row, bar(BK_KV));
                }
        }
        const int it_first = j0 * kBlock / g.P;
        int s = 0;
        bool ok = true;
        int armed[2] = {-1, -1};
        for (int c0 = it_first; ok && c0 < g.ntile_bg; c0 += 32) {
            const int it = c0 + lane;
            int info = -1;
            if (it < g.ntile_bg) {
                const int bt = it * g.P / kBlock;
                int m0 = bt == j0 ? kModeDiag : kModeNone;
                int m1 = (has1 && bt == j1) ? kModeDiag : kModeNone;
                if (bt > j0) {
                    const size_t tile = (size_t)bg * g.ntile_bg + it;
                    const int* Lst = list + tile * g.cap;
                    const int cnt = count[tile];
                    int lo = 0, hi = cnt;              // first entry >= j0
                    while (lo < hi) {
                        const int mid = (lo + hi) >> 1;
                        if (Lst[mid] < j0) lo = mid + 1; else hi = mid;
                    }
                    if (lo < cnt && Lst[lo] == j0) { m0 = kModePast; ++lo; }
                    if (has1 && bt > j1 && lo < cnt && Lst[lo] == j1) m1 = kModePast;
                }
                if (m0 != kModeNone || m1 != kModeNone) info = it | (m0 << 24) | (m1 << 26);
            }
            unsigned keep = __ballot_sync(0xffffffffu, info >= 0);
            while (keep) {
                const int src = __ffs(keep) - 1;
                keep &= keep - 1;
                const int inf = __shfl_sync(0xffffffffu, info, src);
                if (lane == 0) {
                    const int st = s & 1;
                    if (s >= 2 && !mbar_wait(bar(BK_QE + st), ((s >> 1) - 1) & 1, abort_flag)) ok = false;
                    if (ok) {
                        const int t0 = (inf & 0xFFFFFF) * g.P;
                        info_sh[st] = inf;
                        mbar_arrive_expect_tx(bar(BK_QF + st), (uint32_t)(2 * g.M * D * 2));
                        for (int hl = 0; hl < g.G; ++hl) {
                            const int row = (b * g.Hq + kvh * g.G + hl) * g.T + t0;
                            for (int h = 0; h < D / 64; ++h) {
                                tma_load_2d(q_addr(st) + h * L::kHalf + hl * g.P * 128, &tm_q, h * 64, row, bar(BK_QF + st));
                                tma_load_2d(do_addr(st) + h * L::kHalf + hl * g.P * 128, &tm_do, h * 64, row, bar(BK_QF + st));
                            }
                        }
                        armed[st] = s;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                ++s;
                if (!ok) break;
            }
        }
        if (lane == 0) {
            // the sentinel step: consumers see -1 and leave their loops
            const int st = s & 1;
            if (ok && s >= 2 && !mbar_wait(bar(BK_QE + st), ((s >> 1) - 1) & 1, abort_flag)) ok = false;
            if (ok) {
                info_sh[st] = -1;
                mbar_arrive(bar(BK_QF + st));
            } else {
                *abort_flag = 1;
                volatile int dummy = 0;
                mbar_wait(bar(BK_KV), 0, &dummy);
                for (int st2 = 0; st2 < 2; ++st2)
                    if (armed[st2] >= 0) { dummy = 0; mbar_wait(bar(BK_QF + st2), (armed[st2] >> 1) & 1, &dummy); }
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ S and dP issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_ab(128, 128, false, false);
            bool ok = mbar_wait(bar(BK_KV), 0, abort_flag);
            for (int s = 0; ok; ++s) {
                const int st = s & 1;
                if (!mbar_wait(bar(BK_QF + st), (s >> 1) & 1, abort_flag)) { ok = false; break; }
                if (info_sh[st] < 0) break;
                if (s >= 1 && !mbar_wait(bar(BK_S_FREE), (s - 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int h = kk >> 2, wk = kk & 3;
                    const uint64_t a = smem_desc_sw128(q_addr(st) + h * L::kHalf + wk * 32, 16, 1024);
                    const uint64_t bk = smem_desc_sw128(base + L::off_k + h * L::kHalf + wk * 32, 16, 1024);
                    mma_bf16_ss(tmem + L::colS, a, bk, idesc, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int h = kk >> 2, wk = kk & 3;
                    const uint64_t a = smem_desc_sw128(do_addr(st) + h * L::kHalf + wk * 32, 16, 1024);
                    const uint64_t bv = smem_desc_sw128(base + L::off_v + h * L::kHalf + wk * 32, 16, 1024);
                    mma_bf16_ss(tmem + L::colDP, a, bv, idesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(BK_S_FULL));
            }
            if (!ok) {
                mma_commit(bar(BK_DRAIN));
                volatile int dummy = 0;
                mbar_wait(bar(BK_DRAIN), 0, &dummy);
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ dV and dK issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_ab(128, D, true, true);
            bool ok = true;
            for (int s = 0; ok; ++s) {
                const int st = s & 1;
                if (!mbar_wait(bar(BK_QF + st), (s >> 1) & 1, abort_flag)) { ok = false; break; }
                if (info_sh[st] < 0) break;
                if (!mbar_wait(bar(BK_P_FULL), s & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = smem_desc_sw128(base + L::off_buf + kk * 2048, L::kHalf, 1024);
                    const uint64_t bo = smem_desc_sw128(do_addr(st) + kk * 2048, L::kHalf, 1024);
                    mma_bf16_ss(tmem + L::colDV, a, bo, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(BK_DV_DONE));
                if (!mbar_wait(bar(BK_DS_FULL), s & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = smem_desc_sw128(base + L::off_buf + kk * 2048, L::kHalf, 1024);
                    const uint64_t bq = smem_desc_sw128(q_addr(st) + kk * 2048, L::kHalf, 1024);
                    mma_bf16_ss(tmem + L::colDK, a, bq, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(BK_DK_DONE));
                mma_commit(bar(BK_QE + st));
            }
            if (!ok) {
                mma_commit(bar(BK_DRAIN2));
                volatile int dummy = 0;
                mbar_wait(bar(BK_DRAIN2), 0, &dummy);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax: (row, block)
        const int quarter = warp & 3, kb = warp >> 2;
        const int r = quarter * 32 + lane;
        const int jb = j0 + kb;
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
        uint8_t* const brow = base_ptr + L::off_buf + kb * L::kHalf + (r >> 3) * 1024 + (r & 7) * 128;
        const int hl = r / g.P;
        bool ok = true;
        int nsteps = 0;
        auto wwait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
            const bool got = mbar_wait(bar_addr, parity, abort_flag);
            return __all_sync(0xffffffffu, got);
        };
        for (int s = 0;; ++s) {
            const int st = s & 1;
            if (!wwait(bar(BK_QF + st), (s >> 1) & 1)) { ok = false; break; }
            const int inf = info_sh[st];
            if (inf < 0) break;
            const int it = inf & 0xFFFFFF;
            const int mode = (inf >> (24 + 2 * kb)) & 3;
            const int t0 = it * g.P;
            const int t = t0 + r % g.P;
            const bool valid = r < g.M && t < g.T;
            const int tpos = valid ? t : -1;
            const size_t rowid = valid ? (size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t : 0;
            const float lse_r = valid ? lse[rowid] : 0.f;
            const float d_r = valid ? drow[rowid] : 0.f;
            const float rr = valid ? rrow[rowid] : 0.f;
            const float tau_r = (valid && mode == kModePast) ? tau[rowid] : INFINITY;
            if (!wwait(bar(BK_S_FULL), s & 1)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[64];
            tmem_ld<64>(lane_addr + L::colS + kb * 64, sr);
            tmem_wait_ld();
            float lp2 = -INFINITY, xm = 1.f;
            if (mode == kModeDiag) {
                lp2 = tpos >= 0 ? 0.f : -INFINITY;
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (jb * kBlock + i > tpos) sr[i] = __float_as_uint(-INFINITY);
            } else if (mode == kModePast) {
                float rs = 0.f;
#pragma unroll
                for (int i = 0; i < 64; ++i) rs += __uint_as_float(sr[i]);
                xm = rs * C.cxm - tau_r;
                if (tpos >= 0 && xm > 0.f) lp2 = C.e_pow * __log2f(xm);
            }
            const bool sel = mode == kModePast && lp2 > -INFINITY;
            const float c0 = lp2 - lse_r;
            uint32_t pk[32];
            float cj = 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t dp[32];
                tmem_ld<32>(lane_addr + L::colDP + kb * 64 + hh * 32, dp);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float p0 = fast_exp2(fmaf(__uint_as_float(sr[hh * 32 + i]), C.sm2, c0));
                    const float p1 = fast_exp2(fmaf(__uint_as_float(sr[hh * 32 + i + 1]), C.sm2, c0));
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    pk[(hh * 32 + i) >> 1] = *reinterpret_cast<uint32_t*>(&h2);
                    const float d0 = p0 * (__uint_as_float(dp[i]) - d_r);
                    const float d1 = p1 * (__uint_as_float(dp[i + 1]) - d_r);
                    sr[hh * 32 + i] = __float_as_uint(d0);
                    sr[hh * 32 + i + 1] = __float_as_uint(d1);
                    cj += d0 + d1;
                }
            }
            tc_fence_before();
            mbar_arrive(bar(BK_S_FREE));
            const float f = sel ? C.cs64 * (cj / xm - rr * exp2f(C.gpow * __log2f(xm))) : 0.f;
            // the buffer was last read by the previous step's dK product
            if (s >= 1 && !wwait(bar(BK_DK_DONE), (s - 1) & 1)) { ok = false; break; }
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(brow + ((c ^ (r & 7)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar(BK_P_FULL));
            if (!wwait(bar(BK_DV_DONE), s & 1)) { ok = false; break; }
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t w4[4];
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(sr[c * 8 + 2 * q2]) + f,
                                                              __uint_as_float(sr[c * 8 + 2 * q2 + 1]) + f);
                    w4[q2] = *reinterpret_cast<uint32_t*>(&h2);
                }
                *reinterpret_cast<uint4*>(brow + ((c ^ (r & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar(BK_DS_FULL));
            nsteps = s + 1;
        }
        // ---- epilogue: warps 0-3 store dV, warps 4-7 dK of key lane 32 (warp % 4) + lane
        if (ok && nsteps > 0 && wwait(bar(BK_DK_DONE), (nsteps - 1) & 1)) {
            tc_fence_after();
            const int key = quarter * 32 + lane;           // 0..127 over the pair
            const int tok = (j0 + (key >> 6)) * kBlock + (key & 63);
            const bool kval = tok < g.T;
            const uint32_t col = kb == 0 ? L::colDV : L::colDK;
            const float scale = kb == 0 ? 1.f : C.isd;
            __nv_bfloat16* dst = kval ? (kb == 0 ? dv : dk) + ((size_t)bg * g.T + tok) * D : nullptr;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld<32>(lane_addr + col + c * 32, o);
                tmem_wait_ld();
                if (kval) {
                    uint32_t w4[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * scale,
                                                                  __uint_as_float(o[2 * i + 1]) * scale);
                        w4[i] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w4[4 * i], w4[4 * i + 1], w4[4 * i + 2], w4[4 * i + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (tid == 0 && abort_sh) atomicOr(&hdr->status, kStWaitTimeout);
}

// ------------------------------------------------------------------ host side

cudaError_t launch_bwd_dq_tc(const void* q, const void* k, const void* v, const void* dout, void* dq,
                             const PrefillGeom& g, const BwdGeom& bw, char* ws, float alpha, float coarse_scale,
                             cudaStream_t stream) {
    BtConsts C;
    const float sd = sqrtf((float)g.d);
    C.cx = (alpha - 1.0f) * coarse_scale / sd;
    C.e_pow = 1.0f / (alpha - 1.0f);
    C.gpow = (2.0f - alpha) / (alpha - 1.0f);
    C.sm2 = 1.4426950408889634f / sd;
    C.cs64 = coarse_scale / (float)kBlock;
    C.isd = 1.0f / sd;
    CUtensorMap tq, tdo, tk, tv, thi, tlo;
    const unsigned long long qrows = (unsigned long long)g.B * g.Hq * g.T;
    const unsigned long long kvrows = (unsigned long long)g.B * g.Hkv * g.T;
    const unsigned long long srows = (unsigned long long)g.B * g.Hkv * (g.nbs > 0 ? g.nbs : 1);
    if (!make_tmap_bf16(&tq, q, qrows, g.d, g.P) || !make_tmap_bf16(&tdo, dout, qrows, g.d, g.P) ||
        !make_tmap_bf16(&tk, k, kvrows, g.d, kBlock) || !make_tmap_bf16(&tv, v, kvrows, g.d, kBlock) ||
        !make_tmap_bf16(&thi, ws + g.off_khi, srows, g.d, 8) || !make_tmap_bf16(&tlo, ws + g.off_klo, srows, g.d, 8))
        return cudaErrorInvalidValue;
    float* lse = reinterpret_cast<float*>(ws + bw.off_lse);
    float* rr = reinterpret_cast<float*>(ws + bw.off_r);
    const float* drow = reinterpret_cast<const float*>(ws + bw.off_drow);
    const float* tau = reinterpret_cast<const float*>(ws + g.off_tau);
    const int* list = reinterpret_cast<const int*>(ws + g.off_list);
    const int* count = reinterpret_cast<const int*>(ws + g.off_count);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    auto* dqb = static_cast<__nv_bfloat16*>(dq);
    auto go = [&](auto kernel, int sm) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        kernel<<<g.ntiles, 352, sm, stream>>>(tq, tdo, tk, tv, thi, tlo, dqb, lse, rr, drow, tau, list, count, hdr, g, C);
        return cudaGetLastError();
    };
    cudaError_t e;
    if (g.d == 128) {
        e = go(bwd_tc_kernel<128, 0>, (int)BtLayout<128, 0>::bytes);
        if (e == cudaSuccess) e = go(bwd_tc_kernel<128, 1>, (int)BtLayout<128, 1>::bytes);
    } else {
        e = go(bwd_tc_kernel<64, 0>, (int)BtLayout<64, 0>::bytes);
        if (e == cudaSuccess) e = go(bwd_tc_kernel<64, 1>, (int)BtLayout<64, 1>::bytes);
    }
    return e;
}

cudaError_t launch_bwd_dkv_tc(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                              const PrefillGeom& g, const BwdGeom& bw, char* ws, float alpha, float coarse_scale,
                              cudaStream_t stream) {
    BkConsts C;
    const float sd = sqrtf((float)g.d);
    C.cxm = (alpha - 1.0f) * coarse_scale / sd / (float)kBlock;
    C.e_pow = 1.0f / (alpha - 1.0f);
    C.gpow = (2.0f - alpha) / (alpha - 1.0f);
    C.sm2 = 1.4426950408889634f / sd;
    C.cs64 = coarse_scale / (float)kBlock;
    C.isd = 1.0f / sd;
    CUtensorMap tq, tdo, tk, tv;
    const unsigned long long qrows = (unsigned long long)g.B * g.Hq * g.T;
    const unsigned long long kvrows = (unsigned long long)g.B * g.Hkv * g.T;
    if (!make_tmap_bf16(&tq, q, qrows, g.d, g.P) || !make_tmap_bf16(&tdo, dout, qrows, g.d, g.P) ||
        !make_tmap_bf16(&tk, k, kvrows, g.d, kBlock) || !make_tmap_bf16(&tv, v, kvrows, g.d, kBlock))
        return cudaErrorInvalidValue;
    const float* lse = reinterpret_cast<const float*>(ws + bw.off_lse);
    const float* rr = reinterpret_cast<const float*>(ws + bw.off_r);
    const float* drow = reinterpret_cast<const float*>(ws + bw.off_drow);
    const float* tau = reinterpret_cast<const float*>(ws + g.off_tau);
    const int* list = reinterpret_cast<const int*>(ws + g.off_list);
    const int* count = reinterpret_cast<const int*>(ws + g.off_count);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    const int nb = (g.T + kBlock - 1) / kBlock;
    const int grid = g.B * g.Hkv * ((nb + 1) / 2);
    auto* dkb = static_cast<__nv_bfloat16*>(dk);
    auto* dvb = static_cast<__nv_bfloat16*>(dv);
    auto go = [&](auto kernel, int sm) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        kernel<<<grid, 352, sm, stream>>>(tq, tdo, tk, tv, dkb, dvb, lse, rr, drow, tau, list, count, hdr, g, C);
        return cudaGetLastError();
    };
    return g.d == 128 ? go(bwd_dkv_tc_kernel<128>, (int)BkLayout<128>::bytes)
                      : go(bwd_dkv_tc_kernel<64>, (int)BkLayout<64>::bytes);
}

}  // namespace dash
