// fine_tc.cu -- Stage 2 for prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes exactly what fine_mma.cu computes ("DashAttention: Making Sparse Attention Fully
// Differentiable with Adaptive Block Selection", section "Core Mechanism", Stage 2, and
// section "Key Concepts", hierarchical prior): for every row of a 128-row work tile,
// softmax over the tokens of its selected blocks (log p_j added to the logits) and of its
// own block (causal, prior 1), times V.  x_j, hence p_j, comes from two extra columns of
// the S product: block j's summary, split into bf16 hi and lo parts (kbar = hi + lo to
// 16 significant bits, the operands of the coarse stage), is appended to the K tile as
// rows 64 and 72, so S[:, 64] + S[:, 72] = q . kbar_j for any summary (mean or learned).
//
// One CTA per tile.  The tile's listed blocks (steps s = 0 .. n-1, own block last) are
// dealt alternately to two softmax groups (group s & 1), each with its own TMEM S buffer,
// kPBuf P buffers (its steps take them in turn), O accumulator, row-sum column and running
// max; the two partial softmaxes are merged in the epilogue (exactly as split-KV partials).
// The per-step work of a row is a serial chain (load S, row stats, weights, exponentials,
// P), so two groups keep two chains in flight while sharing the Q tile and every K/V load;
// with kPBuf P buffers a group writes P_s while the tensor core still reads its earlier
// ones, and waits for its previous product only to rescale O.  Warps:
//   8 SPLIT            K producer (one lane): the Q tile once (one 64-column box per head
//                      and half of d), then K and the summary rows of every listed block,
//                      3-stage ring (a stage is free once S of its block is computed);
//   8 SPLIT + 3        V producer (one lane): V of every listed block, 3-stage ring (a stage
//                      is free once the block's P V product is done);
//   8 SPLIT + 1        S issuer (one lane): S_s = Q [K_s | kbar_hi | kbar_lo]^T (M=128, N=80
//                      with the summary atoms at columns 64 and 72) into the S buffer of
//                      group s & 1 as soon as block s is loaded, that group has read
//                      S_{s-2} and the product of step s - 2 kPBuf (same P buffer) has landed, so
//                      S_{s+2} is computed while the group works on step s and a group
//                      that sees S_s may write its P buffer without another wait;
//   8 SPLIT + 2        PV issuer (one lane): O_g += P_s V_s (M=128, N=d) and L_g += P_s 1
//                      (N=16, an all-ones B tile: the softmax denominator summed by the
//                      tensor core over exactly the bf16 P it multiplies) as soon as P_s is
//                      written.  Two issuing threads keep a slow K/V load of a later block
//                      from delaying the PV of an earlier one (tcgen05.commit tracks each
//                      thread's own MMAs);
//   0 .. 8 SPLIT - 1   softmax, group = warp / (4 SPLIT); SPLIT threads per tile row (warps
//                      of one group sharing TMEM lanes 32 (warp % 4).. split the row's keys
//                      and exchange partial row sums and maxima through shared memory behind
//                      a named barrier).  Online softmax in the log2 domain; O_g is rescaled
//                      in TMEM only when the running max grows by more than 2^8.  Of every 8
//                      exponentials, 2 kFinePolyPairs run as a polynomial on the FMA pipe
//                      (poly_exp2) and the rest on the SFU, so that neither unit alone sets
//                      the pace.
// Head aggregation (optional): the rows of a position average their block weights
// through shared memory (one group barrier per step) and share log of the mean as prior.
// Operands: Q, K, P K-major and V MN-major, all 128-byte swizzled (TMA writes that layout).
// Every wait is bounded (~2 s); a CTA that gives up sets a status bit and exits cleanly.
// Selection-ordered tiles (ORD = true): a tile is 128 rows of one KV group chosen by the
// ordering pass (order.cu), with any positions; the softmax threads load their rows of Q,
// every row has its own block (prior 1, causal) and ignores listed blocks after it, and the
// tile's list (selected and own blocks of its rows, ascending) gives every step.
// Dump variant (DUMP = true, parity checks only): for rows with a slot in dump.slot, every
// listed block's x_j (as recomputed here from the summary columns) and the weight p_j the
// prior applies (0 when x_j <= tau) are written to dump.x / dump.p [slot, T / 64].
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace dash {

constexpr int kKStages = 3;            // K (+ summary rows) ring
constexpr int kVStages = 3;            // V ring
constexpr int kPBuf = 2;               // P buffers of each softmax group (its steps take them in turn)
constexpr int kFineSplit = 1;          // threads per tile row in each softmax group
constexpr int kFinePolyPairs = 1;      // pairs of every 4 whose 2^x runs on the FMA pipe
constexpr float kLazyRescale = 8.0f;   // log2 units: p values stay below 2^8 between rescales

// 2^x for x <= 8 on the FMA and integer pipes.  Cody-Waite style split x = n + f with
// n = round(x) (added to the exponent field) and f in [-1/2, 1/2], where 2^f comes from a
// degree-3 polynomial fitted here for the least maximum relative error on that interval
// (iteratively reweighted least squares: max relative error 7.5e-5 in fp32, far below the
// bf16 rounding every P value gets).  Arguments below -125 (masked keys, -inf) give
// 2^-125 (about 2e-38), which no fp32 sum of the row can see.
__device__ __forceinline__ uint64_t poly_exp2_x2(uint64_t x2) {
    using namespace sm100;
    float a, b;
    f2_unpack(x2, a, b);
    a = fmaxf(a, -125.0f);
    b = fmaxf(b, -125.0f);
    const uint64_t xc = f2_pack(__float_as_uint(a), __float_as_uint(b));
    const uint32_t kMagic = 0x4B400000u;                          // 1.5 * 2^23: rounds to an integer
    const uint64_t magic2 = f2_pack(kMagic, kMagic);
    const uint64_t t2 = f2_add(xc, magic2);                       // n in the low mantissa bits
    const uint64_t nmagic2 = f2_pack(0xCB400000u, 0xCB400000u);   // -1.5 * 2^23
    const uint64_t f2 = f2_add(xc, f2_neg(f2_add(t2, nmagic2)));  // f = x - n
    const uint64_t c3 = f2_pack(0x3D61FBB0u, 0x3D61FBB0u);        // 0.0551716685
    const uint64_t c2 = f2_pack(0x3E786F0Eu, 0x3E786F0Eu);        // 0.2426111400
    const uint64_t c1 = f2_pack(0x3F31798Du, 0x3F31798Du);        // 0.6932609677
    const uint64_t c0 = f2_pack(0x3F7FFB49u, 0x3F7FFB49u);        // 0.9999280572
    const uint64_t pf = f2_fma(f2_fma(f2_fma(c3, f2, c2), f2, c1), f2, c0);
    uint32_t plo, phi, tlo, thi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(plo), "=r"(phi) : "l"(pf));
    asm("mov.b64 {%0, %1}, %2;" : "=r"(tlo), "=r"(thi) : "l"(t2));
    // (bits(t) << 23) == n << 23 modulo 2^32: the magic number's bits vanish in the shift
    return f2_pack(plo + (tlo << 23), phi + (thi << 23));
}

template <int D>
struct TcLayout {
    static constexpr uint32_t kQHalf = 128 * 128;               // 128 rows x 64 bf16
    static constexpr uint32_t kQ = (D / 64) * kQHalf;
    static constexpr uint32_t kKRows = 80;                      // 64 keys, kbar hi atom, kbar lo atom
    static constexpr uint32_t kKHalf = kKRows * 128;            // 80 rows x 64 bf16
    static constexpr uint32_t kK = (D / 64) * kKHalf;
    static constexpr uint32_t kVHalf = 64 * 128;                // 64 keys x 64 bf16
    static constexpr uint32_t kV = (D / 64) * kVHalf;
    static constexpr uint32_t kP = 128 * 128;                   // 128 rows x 64 keys bf16
    static constexpr uint32_t off_q = 0;
    static constexpr uint32_t off_k = kQ;                       // K ring
    static constexpr uint32_t off_v = off_k + kKStages * kK;    // V ring
    static constexpr uint32_t off_p = off_v + kVStages * kV;    // P buffers [group][kPBuf]
    static constexpr uint32_t off_ones = off_p + 2 * kPBuf * kP; // 16 x 64 bf16 ones (B of the row sum)
    static constexpr uint32_t bytes = off_ones + 2048 + 1024;   // + alignment slack
    // TMEM columns: S of group 0 and 1, O of group 0 and 1, row sums of group 0 and 1
    static constexpr uint32_t colS = 96;                        // S buffer of group g at g * 96 (80 used)
    static constexpr uint32_t colO = 192;
    static constexpr uint32_t colL = 192 + 2 * D;               // row sums of group g at + g * 32 (16 used)
    // Selection-ordered tiles keep Q in TMEM as the A operand of S (the tensor core then reads
    // only K from shared memory): K step kk (8 columns) in the unused 16-column gaps after
    // the S buffers and the row sums
    __host__ __device__ static constexpr uint32_t colQ(int kk) {
        return ((kk >> 1) == 0 ? 80u : (kk >> 1) == 1 ? 176u : (kk >> 1) == 2 ? 464u : 496u) + (uint32_t)(kk & 1) * 8u;
    }
    static_assert(kKRows <= 80 && colO >= 192 && colL + 32 + 16 <= 496, "Q gaps of TMEM");
    static_assert(D == 64 || colL == 448, "the last two Q gaps follow the row sums of d = 128");
};
constexpr uint32_t kTmemCols = 512;

// barrier slots (P_FULL and PV_DONE per P buffer: index kPBuf group + buffer)
enum : int { B_Q = 0, B_K_FULL = 1, B_K_EMPTY = B_K_FULL + kKStages, B_V_FULL = B_K_EMPTY + kKStages,
             B_V_EMPTY = B_V_FULL + kVStages, B_S_FULL = B_V_EMPTY + kVStages, B_S_FREE = B_S_FULL + 2,
             B_P_FULL = B_S_FREE + 2, B_PV_DONE = B_P_FULL + 2 * kPBuf, B_DRAIN = B_PV_DONE + 2 * kPBuf,
             B_DRAIN2 = B_DRAIN + 1, B_COUNT = B_DRAIN2 + 1 };

template <int D, int SPLIT, bool AGG, bool DUMP, bool ORD>
__global__ void __launch_bounds__((8 * SPLIT + 4) * 32, 1)
fine_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_hi,
               const __grid_constant__ CUtensorMap tm_lo, __nv_bfloat16* __restrict__ out,
               const float* __restrict__ tau, const int* __restrict__ list, const int* __restrict__ count,
               WsHeader* __restrict__ hdr, PrefillGeom g, float cx, float e_pow, float sm2,
               FineDump dump, const __nv_bfloat16* __restrict__ qrows, const int* __restrict__ ord_rows) {
    static_assert(!(ORD && AGG), "head aggregation keeps the position tiles");
    using L = TcLayout<D>;
    using namespace sm100;
    constexpr int kGroupThreads = 128 * SPLIT;  // softmax threads per group
    constexpr int KEYS = 64 / SPLIT;            // keys of a block per softmax thread
    constexpr int OCOLS = D / (2 * SPLIT);      // epilogue output columns per softmax thread
    constexpr int OCW = OCOLS < 32 ? OCOLS : 32;
    constexpr int RCOLS = D / SPLIT;            // O columns a thread rescales in its group
    constexpr int RCW = RCOLS < 32 ? RCOLS : 32;
    constexpr int kProducerWarp = 8 * SPLIT, kMmaSWarp = 8 * SPLIT + 1, kMmaPvWarp = 8 * SPLIT + 2;
    constexpr int kVProducerWarp = 8 * SPLIT + 3;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[B_COUNT];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ float2 xch[2][2][SPLIT][kTileRows]; // [step parity][group][split][row]: partial (sum, max)
    __shared__ float pagg[AGG ? 2 : 1][2][kTileRows];   // [step parity][group][row]: weights for head aggregation
    __shared__ float m_sh[2][kTileRows];        // running max of each group, for the merge

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto k_addr = [&](int st) { return base + L::off_k + (uint32_t)st * L::kK; };
    auto v_addr = [&](int st) { return base + L::off_v + (uint32_t)st * L::kV; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // group-major order (longest tiles of a group first): the CTAs in flight share one KV
    // group, whose K and V stay in L2 while its tiles re-read them
    const int w = blockIdx.x;
    const int ntb = ORD ? g.ord_bg : g.ntile_bg;            // tiles per KV group
    const int bg = w / ntb;
    const int it = ntb - 1 - w % ntb;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int t0 = ORD ? 0 : it * g.P;
    const int bt = ORD ? 0 : t0 / kBlock;                   // own block of a position tile
    const size_t tile_id = (size_t)bg * ntb + it;
    // position tiles: the listed past blocks, then the own block; ordered tiles: the list
    const int U = (ORD || bt > 0) ? count[tile_id] : 0;
    const int n = ORD ? U : U + 1;
    const int* lst = list + tile_id * (ORD ? g.ord_cap : g.cap);

    if (tid == 0) {
        abort_sh = 0;
        mbar_init(bar(B_Q), ORD ? kTileRows : 1);          // ordered tiles: the row loads arrive
        for (int st = 0; st < kKStages; ++st) {
            mbar_init(bar(B_K_FULL + st), 1);
            mbar_init(bar(B_K_EMPTY + st), 1);
        }
        for (int st = 0; st < kVStages; ++st) {
            mbar_init(bar(B_V_FULL + st), 1);
            mbar_init(bar(B_V_EMPTY + st), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_S_FULL + i), 1);
            mbar_init(bar(B_S_FREE + i), kGroupThreads);
        }
        for (int i = 0; i < 2 * kPBuf; ++i) {
            mbar_init(bar(B_P_FULL + i), kGroupThreads);
            mbar_init(bar(B_PV_DONE + i), 1);
        }
        mbar_init(bar(B_DRAIN), 1);
        mbar_init(bar(B_DRAIN2), 1);
        fence_mbar_init();
    }
    // rows of the Q tile beyond G * P are never loaded: zero them once
    if (!ORD && g.M < kTileRows && tid < kTileRows && tid >= g.M) {
        for (int h = 0; h < D / 64; ++h) {
            uint4* p = reinterpret_cast<uint4*>(base_ptr + L::off_q + h * L::kQHalf + tid * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) p[c] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    // the all-ones B operand of the row-sum MMA (any layout: every element is 1)
    if (tid < 128) {
        uint4* p = reinterpret_cast<uint4*>(base_ptr + L::off_ones) + tid;
        *p = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
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
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_hi);
            prefetch_tmap(&tm_lo);
            if (!ORD) {
                mbar_arrive_expect_tx(bar(B_Q), (uint32_t)(g.M * D * 2));
                for (int hl = 0; hl < g.G; ++hl) {
                    const int row = (b * g.Hq + kvh * g.G + hl) * g.T + t0;
                    for (int h = 0; h < D / 64; ++h)
                        tma_load_2d(base + L::off_q + h * L::kQHalf + hl * g.P * 128, &tm_q, h * 64, row, bar(B_Q));
                }
            }
            int last_armed[kKStages];
            for (int st = 0; st < kKStages; ++st) last_armed[st] = -1;
            for (int s = 0; s < n; ++s) {
                const int st = s % kKStages;
                if (s >= kKStages && !mbar_wait(bar(B_K_EMPTY + st), ((s / kKStages) - 1) & 1, abort_flag)) break;
                const int j = s < U ? lst[s] : bt;
                const int row = bg * g.T + j * kBlock;
                // the summary atoms: 8 rows of kbar hi / lo starting at block j (the own block,
                // whose x is not used, reads a neighbour; rows past the array read zeros)
                const int srow = g.nbs > 0 ? bg * g.nbs + min(j, g.nbs - 1) : 0;
                mbar_arrive_expect_tx(bar(B_K_FULL + st), (uint32_t)((kBlock + 16) * D * 2));
                for (int h = 0; h < D / 64; ++h) {
                    tma_load_2d(k_addr(st) + h * L::kKHalf, &tm_k, h * 64, row, bar(B_K_FULL + st));
                    tma_load_2d(k_addr(st) + h * L::kKHalf + 64 * 128, &tm_hi, h * 64, srow, bar(B_K_FULL + st));
                    tma_load_2d(k_addr(st) + h * L::kKHalf + 72 * 128, &tm_lo, h * 64, srow, bar(B_K_FULL + st));
                }
                last_armed[st] = s;
            }
            if (*abort_flag) {
                // let every load this thread started land before the CTA exits
                volatile int dummy = 0;
                if (!ORD) mbar_wait(bar(B_Q), 0, &dummy);
                for (int st = 0; st < kKStages; ++st)
                    if (last_armed[st] >= 0) { dummy = 0; mbar_wait(bar(B_K_FULL + st), (last_armed[st] / kKStages) & 1, &dummy); }
            }
        }
    } else if (warp == kVProducerWarp) {
        // ------------------------------------------------------------ V producer
        if (lane == 0) {
            int last_armed[kVStages];
            for (int st = 0; st < kVStages; ++st) last_armed[st] = -1;
            for (int s = 0; s < n; ++s) {
                const int st = s % kVStages;
                if (s >= kVStages && !mbar_wait(bar(B_V_EMPTY + st), ((s / kVStages) - 1) & 1, abort_flag)) break;
                const int j = s < U ? lst[s] : bt;
                const int row = bg * g.T + j * kBlock;
                mbar_arrive_expect_tx(bar(B_V_FULL + st), (uint32_t)(kBlock * D * 2));
                for (int h = 0; h < D / 64; ++h)
                    tma_load_2d(v_addr(st) + h * L::kVHalf, &tm_v, h * 64, row, bar(B_V_FULL + st));
                last_armed[st] = s;
            }
            if (*abort_flag) {
                volatile int dummy = 0;
                for (int st = 0; st < kVStages; ++st)
                    if (last_armed[st] >= 0) { dummy = 0; mbar_wait(bar(B_V_FULL + st), (last_armed[st] / kVStages) & 1, &dummy); }
            }
        }
    } else if (warp == kMmaSWarp) {
        // ------------------------------------------------------------ S issuer
        // S_s = Q K_s^T into the S buffer of group s & 1, as soon as block s is loaded and the
        // group has read S_{s-2}: it runs ahead of the softmax by up to one step per group.
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16(128, L::kKRows, false);
            bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
            for (int s = 0; ok && s < n; ++s) {
                const int st = s % kKStages, sb = s & 1;
                if (!mbar_wait(bar(B_K_FULL + st), (s / kKStages) & 1, abort_flag)) { ok = false; break; }
                if (s >= 2 && !mbar_wait(bar(B_S_FREE + sb), ((s - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
                // the P buffer step s will use was last read by the product of step
                // s - 2 kPBuf: S_s is computed only after that product landed, so a softmax
                // group that sees S_s may overwrite the buffer
                const int i2 = s >> 1;
                if (i2 >= kPBuf && !mbar_wait(bar(B_PV_DONE + kPBuf * sb + i2 % kPBuf), ((i2 - kPBuf) / kPBuf) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int h = kk >> 2, wk = kk & 3;
                    const uint64_t bk = smem_desc_sw128(k_addr(st) + h * L::kKHalf + wk * 32, 16, 1024);
                    if constexpr (ORD) {
                        mma_bf16_ts(tmem + sb * L::colS, tmem + L::colQ(kk), bk, idesc_s, kk > 0 ? 1u : 0u);
                    } else {
                        const uint64_t a = smem_desc_sw128(base + L::off_q + h * L::kQHalf + wk * 32, 16, 1024);
                        mma_bf16_ss(tmem + sb * L::colS, a, bk, idesc_s, kk > 0 ? 1u : 0u);
                    }
                }
                mma_commit(bar(B_S_FULL + sb));
                mma_commit(bar(B_K_EMPTY + st));
            }
            if (!ok) {
                // every MMA this thread issued must finish before TMEM is released
                mma_commit(bar(B_DRAIN));
                volatile int dummy = 0;
                mbar_wait(bar(B_DRAIN), 0, &dummy);
            }
        }
    } else if (warp == kMmaPvWarp) {
        // ------------------------------------------------------------ PV issuer
        // O_g += P_p V_p and L_g += P_p 1 as soon as P_p is written and V_p has landed; then
        // the V stage of block p and P buffer (p & 1, (p >> 1) % kPBuf) are free again.
        if (lane == 0) {
            const uint32_t idesc_pv = idesc_bf16(128, D, true);
            const uint32_t idesc_l = idesc_bf16(128, 16, false);
            bool ok = true;
            for (int p = 0; p < n; ++p) {
                const int gp = p & 1, i2 = p >> 1, pbuf = kPBuf * gp + i2 % kPBuf, stp = p % kVStages;
                if (!mbar_wait(bar(B_P_FULL + pbuf), (i2 / kPBuf) & 1, abort_flag)) { ok = false; break; }
                if (!mbar_wait(bar(B_V_FULL + stp), (p / kVStages) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t acc = p >= 2 ? 1u : 0u;          // first step of a group overwrites
                const uint32_t pa = base + L::off_p + pbuf * L::kP;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = smem_desc_sw128(pa + kk * 32, 16, 1024);
                    const uint64_t bv = smem_desc_sw128(v_addr(stp) + kk * 2048, L::kVHalf, 1024);
                    mma_bf16_ss(tmem + L::colO + gp * D, a, bv, idesc_pv, (acc || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = smem_desc_sw128(pa + kk * 32, 16, 1024);
                    const uint64_t bo = smem_desc_sw128(base + L::off_ones + kk * 32, 16, 1024);
                    mma_bf16_ss(tmem + L::colL + gp * 32, a, bo, idesc_l, (acc || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(B_PV_DONE + pbuf));
                mma_commit(bar(B_V_EMPTY + stp));
            }
            if (!ok) {
                mma_commit(bar(B_DRAIN2));
                volatile int dummy = 0;
                mbar_wait(bar(B_DRAIN2), 0, &dummy);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax groups
        const int grp = warp / (4 * SPLIT);
        const int wg = warp % (4 * SPLIT);
        const int quarter = wg & 3, sp = wg >> 2;          // TMEM lane quarter, key split
        const int r = quarter * 32 + lane;                  // tile row = TMEM lane
        // the tile row: (head in group, position); ordered tiles read it from the tile's rows
        const int rid = ORD ? ord_rows[tile_id * kTileRows + r] : 0;
        const int hl = ORD ? (rid >= 0 ? rid >> kRowShift : 0) : r / g.P;
        const int t = ORD ? (rid >= 0 ? rid & kRowMask : 0) : t0 + r % g.P;
        const bool valid = ORD ? rid >= 0 : (r < g.M && t < g.T);
        const int tpos = valid ? t : -1;
        const int bt_r = ORD ? t / kBlock : bt;             // the row's own block
        const float tau_r = (valid && bt_r > 0) ? tau[(size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t] : INFINITY;
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
        if constexpr (ORD) {
            // this tile's rows of Q into TMEM, the A operand of S (row r in lane r; zeros for
            // rows the tile does not fill): 16 columns (two K steps, 32 elements) per store
            if (grp == 0 && sp == 0) {
                const uint4* src = reinterpret_cast<const uint4*>(qrows + ((size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t) * D);
#pragma unroll
                for (int f = 0; f < D / 32; ++f) {
                    uint32_t w16[16];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = valid ? src[f * 4 + c] : make_uint4(0u, 0u, 0u, 0u);
                        w16[4 * c] = v.x; w16[4 * c + 1] = v.y; w16[4 * c + 2] = v.z; w16[4 * c + 3] = v.w;
                    }
                    tmem_st16(lane_addr + L::colQ(2 * f), w16);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_Q));
            }
        }
        const int slot = (DUMP && valid) ? dump.slot[(size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t] : -1;
        // parity dump of one listed past block: x_j and the weight the prior applies
        auto dump_block = [&](int j, float x) {
            if constexpr (DUMP) {
                if (slot >= 0 && sp == 0) {
                    dump.x[(size_t)slot * g.nbs + j] = x;
                    dump.p[(size_t)slot * g.nbs + j] = x > tau_r ? exp2f(e_pow * __log2f(x - tau_r)) : 0.f;
                }
            }
        };
        const uint32_t s_col = grp * L::colS + sp * KEYS;   // this thread's keys in its group's S buffer
        const uint32_t o_col = L::colO + grp * D + sp * RCOLS;   // O columns it rescales
        const uint32_t l_col = L::colL + grp * 32;
        uint8_t* const prow0 = base_ptr + L::off_p + (kPBuf * grp) * L::kP + (r >> 3) * 1024 + (r & 7) * 128;
        const int row_bar = 1 + grp * 4 + quarter;          // named barrier of the row's SPLIT warps
        float m_run = -INFINITY;
        bool ok = true;
        // TMEM loads and stores are warp-collective: every wait result is made warp-uniform
        auto wwait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
            const bool got = mbar_wait(bar_addr, parity, abort_flag);
            return __all_sync(0xffffffffu, got);
        };
        auto row_sync = [&]() {
            if constexpr (SPLIT > 1) asm volatile("bar.sync %0, %1;" :: "r"(row_bar), "n"(32 * SPLIT) : "memory");
        };
        // Each warp executes exactly one row barrier per step, even after a failed wait (a
        // failed step skips its work but still synchronises), so the named barriers of the
        // row's warps always match.
        for (int s = grp; s < n; s += 2) {
            const int i2 = s >> 1;                          // this group's step index
            const int j = s < U ? lst[s] : bt;
            const bool diag = (j == bt_r);
            const bool okw = ok && wwait(bar(B_S_FULL + grp), i2 & 1);
            uint32_t sr[KEYS];
            float ps_own = 0.f, pm_own = -INFINITY;
            if (okw) {
                tc_fence_after();
                tmem_ld<KEYS>(lane_addr + s_col, sr);
                // q . kbar_j = q . kbar_hi + q . kbar_lo: the summary columns of the S buffer
                const uint32_t qhi = tmem_ld1(lane_addr + grp * L::colS + 64);
                const uint32_t qlo = tmem_ld1(lane_addr + grp * L::colS + 72);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(bar(B_S_FREE + grp));
                // counted once per row when SPLIT threads share it
                ps_own = sp == 0 ? __uint_as_float(qhi) + __uint_as_float(qlo) : 0.f;
                // own block: keys after the query position are masked
                if (diag) {
                    const int key0 = j * kBlock + sp * KEYS;
#pragma unroll
                    for (int i = 0; i < KEYS; ++i)
                        if (key0 + i > tpos) sr[i] = __float_as_uint(-INFINITY);
                }
                // partial raw max with three-input max
                float m4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) m4[i] = fmaxf(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
#pragma unroll
                for (int i = 4; i < KEYS / 2; ++i) m4[i & 3] = max3(m4[i & 3], __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
                pm_own = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            }
            float rs = ps_own, smax = pm_own;
            if constexpr (SPLIT > 1) {
                // every thread of the row combines the partials in the same order: identical x.
                // Slots alternate with the step parity: a slot is rewritten two steps later,
                // after every thread of the row has passed the barrier in between.
                xch[i2 & 1][grp][sp][r] = make_float2(ps_own, pm_own);
                row_sync();
                rs = 0.f;
                smax = -INFINITY;
#pragma unroll
                for (int k = 0; k < SPLIT; ++k) {
                    const float2 e = xch[i2 & 1][grp][k][r];
                    rs += e.x;
                    smax = fmaxf(smax, e.y);
                }
            }
            float lp2;
            if constexpr (AGG) {
                // head aggregation: the rows of one position (r = hl P + pl for every head hl)
                // average their weights p = (x - tau)^(1/(alpha-1)); every warp of the group
                // passes this barrier once per step, failed step or not
                const float x = __fmul_rn(rs, cx);
                const float pown = (okw && !diag && x > tau_r) ? exp2f(e_pow * __log2f(x - tau_r)) : 0.f;
                if (okw && !diag) dump_block(j, x);
                if (sp == 0) pagg[i2 & 1][grp][r] = pown;
                asm volatile("bar.sync %0, %1;" :: "r"(10 + grp), "n"(kGroupThreads) : "memory");
                float pbar = 0.f;
                for (int h2 = 0; h2 < g.G; ++h2) pbar += pagg[i2 & 1][grp][h2 * g.P + (r % g.P)];
                pbar *= 1.0f / (float)g.G;
                lp2 = diag ? (tpos >= 0 ? 0.f : -INFINITY) : (pbar > 0.f && valid ? __log2f(pbar) : -INFINITY);
                if (!okw) { ok = false; continue; }
            } else {
                if (!okw) { ok = false; continue; }
                const float x = __fmul_rn(rs, cx);
                // past blocks only: an ordered tile also lists blocks after some rows' own
                lp2 = diag ? (tpos >= 0 ? 0.f : -INFINITY)
                           : ((j < bt_r && x > tau_r) ? e_pow * __log2f(x - tau_r) : -INFINITY);
                if (!diag && j < bt_r) dump_block(j, x);
            }
            const bool active = lp2 > -INFINITY;
            const float mx = active ? fmaf(smax, sm2, lp2) : -INFINITY;
            float factor = 1.f;
            bool resc = false;
            if (active) {
                if (m_run == -INFINITY) {
                    m_run = mx;
                } else if (mx > m_run + kLazyRescale) {
                    factor = exp2f(m_run - mx);
                    m_run = mx;
                    resc = true;
                }
            }
            // P buffer pb of this group was last read by its product kPBuf steps back, which
            // had landed before S_s was computed (the S issuer waits for it)
            const int pb = i2 % kPBuf;
            uint8_t* const prow = prow0 + pb * L::kP;
            // p = 2^(s sm2 + log2 p_j - m): packed FMA, exponent on the SFU or the FMA pipe,
            // bf16 pairs
            const float c0 = lp2 - m_run;
            const uint64_t sm2x2 = f2_pack(__float_as_uint(sm2), __float_as_uint(sm2));
            const uint64_t c0x2 = f2_pack(__float_as_uint(c0), __float_as_uint(c0));
#pragma unroll
            for (int c = 0; c < KEYS / 8; ++c) {
                uint32_t pk[4] = {0u, 0u, 0u, 0u};
                if (active) {
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const uint64_t e2 = f2_fma(f2_pack(sr[c * 8 + 2 * q2], sr[c * 8 + 2 * q2 + 1]), sm2x2, c0x2);
                        float e0, e1;
                        if (q2 < kFinePolyPairs) {
                            f2_unpack(poly_exp2_x2(e2), e0, e1);
                        } else {
                            f2_unpack(e2, e0, e1);
                            e0 = fast_exp2(e0);
                            e1 = fast_exp2(e1);
                        }
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(e0, e1);
                        pk[q2] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                }
                const int chunk = sp * (KEYS / 8) + c;
                *reinterpret_cast<uint4*>(prow + ((chunk ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            // rescale after P: the S registers are dead by now; O_grp and L_grp hold the
            // group's previous product only once that product has landed
            if (__any_sync(0xffffffffu, resc)) {
                if (i2 >= 1 && !wwait(bar(B_PV_DONE + kPBuf * grp + (i2 - 1) % kPBuf), ((i2 - 1) / kPBuf) & 1)) {
                    ok = false;
                    continue;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < RCOLS / RCW; ++c) {
                    uint32_t o[RCW];
                    tmem_ld<RCW>(lane_addr + o_col + c * RCW, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < RCW; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
                    tmem_st<RCW>(lane_addr + o_col + c * RCW, o);
                }
                if (sp == 0) {
                    uint32_t o[16];
                    tmem_ld16(lane_addr + l_col, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
                    tmem_st16(lane_addr + l_col, o);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar(B_P_FULL + kPBuf * grp + pb));
        }
        // ---- merge the two groups: out = (O_0 2^(m_0-M) + O_1 2^(m_1-M)) / (L_0 ... + L_1 ...)
        if (sp == 0) m_sh[grp][r] = m_run;
        asm volatile("bar.sync %0, %1;" :: "r"(9), "n"(256 * SPLIT) : "memory");
        const bool has1 = n >= 2;                           // group 1 ran at least one step
        const int last0 = (n - 1) & ~1;                     // last step of group 0
        const int last1 = (n - 1) - ((n - 1) & 1 ? 0 : 1);  // last step of group 1
        const int i0 = last0 >> 1, i1 = last1 >> 1;       // their step indices within the groups
        bool done = ok && wwait(bar(B_PV_DONE + i0 % kPBuf), (i0 / kPBuf) & 1);
        if (has1) done = done && wwait(bar(B_PV_DONE + kPBuf + i1 % kPBuf), (i1 / kPBuf) & 1);
        if (done) {
            tc_fence_after();
            const float m0 = m_sh[0][r], m1 = has1 ? m_sh[1][r] : -INFINITY;
            const float M = fmaxf(m0, m1);
            const float w0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M);
            const float w1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
            const float l0 = __uint_as_float(tmem_ld1(lane_addr + L::colL));
            float l1 = 0.f;
            if (has1) l1 = __uint_as_float(tmem_ld1(lane_addr + L::colL + 32));
            tmem_wait_ld();
            const float inv = 1.0f / (l0 * w0 + (w1 > 0.f ? l1 * w1 : 0.f));
            const int col0 = (grp * SPLIT + sp) * OCOLS;    // this thread's output columns
            __nv_bfloat16* dst = valid ? out + ((size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t) * D + col0 : nullptr;
#pragma unroll
            for (int c = 0; c < OCOLS / OCW; ++c) {
                uint32_t o0[OCW], o1[OCW];
                tmem_ld<OCW>(lane_addr + L::colO + col0 + c * OCW, o0);
                if (has1) tmem_ld<OCW>(lane_addr + L::colO + D + col0 + c * OCW, o1);
                tmem_wait_ld();
                if (valid) {
                    uint32_t pk[OCW / 2];
#pragma unroll
                    for (int i = 0; i < OCW / 2; ++i) {
                        float a0 = __uint_as_float(o0[2 * i]) * w0, a1 = __uint_as_float(o0[2 * i + 1]) * w0;
                        if (w1 > 0.f) {
                            a0 = fmaf(__uint_as_float(o1[2 * i]), w1, a0);
                            a1 = fmaf(__uint_as_float(o1[2 * i + 1]), w1, a1);
                        }
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(a0 * inv, a1 * inv);
                        pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c * OCW);
#pragma unroll
                    for (int i = 0; i < OCW / 8; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (tid == 0 && abort_sh) atomicOr(&hdr->status, kStWaitTimeout);
}

// ------------------------------------------------------------------ host side

bool fine_tc_supported(const PrefillGeom& g) { return g.P >= 8 && (g.d == 64 || g.d == 128); }

cudaError_t launch_fine_tc(const void* q, const void* k, const void* v, void* out, const PrefillGeom& g,
                           char* ws, float alpha, float coarse_scale, cudaStream_t stream, int agg,
                           const FineDump* dump, bool ordered) {
    if (ordered && (agg || g.nbs == 0)) return cudaErrorInvalidValue;
    const float cx = (alpha - 1.0f) * coarse_scale / sqrtf((float)g.d);
    const float e_pow = 1.0f / (alpha - 1.0f);
    const float sm2 = 1.4426950408889634f / sqrtf((float)g.d);
    CUtensorMap tq, tk, tv, thi, tlo;
    const unsigned long long qrows = (unsigned long long)g.B * g.Hq * g.T;
    const unsigned long long kvrows = (unsigned long long)g.B * g.Hkv * g.T;
    // block summaries as bf16 hi / lo [B * Hkv * nbs, d] (at least one row: with no complete
    // block every tile has only its own block and the summary columns are never read)
    const unsigned long long srows = (unsigned long long)g.B * g.Hkv * (g.nbs > 0 ? g.nbs : 1);
    if (!make_tmap_bf16(&tq, q, qrows, g.d, g.P) || !make_tmap_bf16(&tk, k, kvrows, g.d, kBlock) ||
        !make_tmap_bf16(&tv, v, kvrows, g.d, kBlock) || !make_tmap_bf16(&thi, ws + g.off_khi, srows, g.d, 8) ||
        !make_tmap_bf16(&tlo, ws + g.off_klo, srows, g.d, 8))
        return cudaErrorInvalidValue;
    const float* tau = reinterpret_cast<const float*>(ws + g.off_tau);
    const int* list = reinterpret_cast<const int*>(ws + (ordered ? g.off_ord_list : g.off_list));
    const int* count = reinterpret_cast<const int*>(ws + (ordered ? g.off_ord_count : g.off_count));
    const int* ord_rows = ordered ? reinterpret_cast<const int*>(ws + g.off_ord_rows) : nullptr;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    constexpr int threads = (8 * kFineSplit + 4) * 32;
    const FineDump dv = dump ? *dump : FineDump{nullptr, nullptr, nullptr};
    const int grid = ordered ? g.ord_ntiles : g.ntiles;
    auto go = [&](auto kernel, int sm) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        kernel<<<grid, threads, sm, stream>>>(tq, tk, tv, thi, tlo, ob, tau, list, count, hdr, g, cx, e_pow, sm2, dv,
                                              qb, ord_rows);
        return cudaSuccess;
    };
    auto pick = [&](auto dcon) -> cudaError_t {
        constexpr int DD = decltype(dcon)::value;
        const int sm = (int)TcLayout<DD>::bytes;
        if (ordered) return dump ? go(fine_tc_kernel<DD, kFineSplit, false, true, true>, sm)
                                 : go(fine_tc_kernel<DD, kFineSplit, false, false, true>, sm);
        if (dump) return agg ? go(fine_tc_kernel<DD, kFineSplit, true, true, false>, sm)
                             : go(fine_tc_kernel<DD, kFineSplit, false, true, false>, sm);
        return agg ? go(fine_tc_kernel<DD, kFineSplit, true, false, false>, sm)
                   : go(fine_tc_kernel<DD, kFineSplit, false, false, false>, sm);
    };
    cudaError_t e = g.d == 128 ? pick(std::integral_constant<int, 128>{}) : pick(std::integral_constant<int, 64>{});
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace dash
