// fine_tc.cu -- Stage 2 for prefill on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes exactly what fine_mma.cu computes ("DashAttention: Making Sparse Attention Fully
// Differentiable with Adaptive Block Selection", section "Core Mechanism", Stage 2, and
// section "Key Concepts", hierarchical prior): for every row of a 128-row work tile,
// softmax over the tokens of its selected blocks (log p_j added to the logits) and of its
// own block (causal, prior 1), times V.  x_j, hence p_j, comes from the row sums of the
// Q K^T block the kernel computes anyway (q . kbar_j is the mean of q . k_i).
//
// One CTA per tile, 192 threads in three roles:
//   warp 4 (one lane)  TMA producer: the Q tile once (one 64-column box per head and half
//                      of d), then K and V of every listed block through a 3-stage ring;
//   warp 5 (one lane)  MMA issuer: S_s = Q K_s^T into one of two TMEM S buffers (M=128,
//                      N=64), then O += P_{s-1} V_{s-1} into the TMEM O accumulator
//                      (M=128, N=d), so the tensor core computes S_s while the softmax
//                      warps work on S_{s-1};
//   warps 0-3          softmax, one thread per tile row = TMEM lane: load S, block weight,
//                      online softmax in the log2 domain, P (bf16) into shared memory in the
//                      128-byte-swizzled K-major layout the MMA reads; O is rescaled in TMEM
//                      only when the running max grows by more than 2^8 (lazy rescale).
// Operands: Q, K, P K-major and V MN-major, all 128-byte swizzled (TMA writes that layout).
// Every wait is bounded (~2 s); a CTA that gives up sets a status bit and exits cleanly.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace dash {

constexpr int kTcStages = 3;
constexpr int kTcThreads = 192;
constexpr float kLazyRescale = 8.0f;   // log2 units: p values stay below 2^8 between rescales

template <int D>
struct TcLayout {
    static constexpr uint32_t kQHalf = 128 * 128;               // 128 rows x 64 bf16
    static constexpr uint32_t kQ = (D / 64) * kQHalf;
    static constexpr uint32_t kKVHalf = 64 * 128;               // 64 keys x 64 bf16
    static constexpr uint32_t kKV = (D / 64) * kKVHalf;
    static constexpr uint32_t kStage = 2 * kKV;                 // K then V
    static constexpr uint32_t kP = 128 * 128;                   // 128 rows x 64 keys bf16
    static constexpr uint32_t off_q = 0;
    static constexpr uint32_t off_kv = kQ;
    static constexpr uint32_t off_p = kQ + kTcStages * kStage;
    static constexpr uint32_t bytes = off_p + 2 * kP + 1024;    // + alignment slack
};

// barrier slots
enum : int { B_Q = 0, B_KV_FULL = 1, B_KV_EMPTY = 1 + kTcStages, B_S_FULL = 1 + 2 * kTcStages,
             B_S_FREE = B_S_FULL + 2, B_P_FULL = B_S_FREE + 2, B_PV_DONE = B_P_FULL + 2,
             B_DRAIN = B_PV_DONE + 2, B_COUNT = B_DRAIN + 1 };

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
fine_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
               const float* __restrict__ tau, const int* __restrict__ list, const int* __restrict__ count,
               WsHeader* __restrict__ hdr, PrefillGeom g, float cxm, float e_pow, float sm2) {
    using L = TcLayout<D>;
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[B_COUNT];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto kv_addr = [&](int st) { return base + L::off_kv + (uint32_t)st * L::kStage; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int BH = g.B * g.Hkv;
    const int w = blockIdx.x;
    const int it = g.ntile_bg - 1 - w / BH;
    const int bg = w % BH;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int t0 = it * g.P;
    const int bt = t0 / kBlock;
    const size_t tile_id = (size_t)bg * g.ntile_bg + it;
    const int U = bt > 0 ? count[tile_id] : 0;
    const int n = U + 1;                                    // listed past blocks, then the own block
    const int* lst = list + tile_id * g.cap;

    if (tid == 0) {
        abort_sh = 0;
        mbar_init(bar(B_Q), 1);
        for (int st = 0; st < kTcStages; ++st) {
            mbar_init(bar(B_KV_FULL + st), 1);
            mbar_init(bar(B_KV_EMPTY + st), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_S_FULL + i), 1);
            mbar_init(bar(B_S_FREE + i), 128);
            mbar_init(bar(B_P_FULL + i), 128);
            mbar_init(bar(B_PV_DONE + i), 1);
        }
        mbar_init(bar(B_DRAIN), 1);
        fence_mbar_init();
    }
    // rows of the Q tile beyond G * P are never loaded: zero them once
    if (g.M < kTileRows && tid < kTileRows && tid >= g.M) {
        for (int h = 0; h < D / 64; ++h) {
            uint4* p = reinterpret_cast<uint4*>(base_ptr + L::off_q + h * L::kQHalf + tid * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) p[c] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(smem_u32(&tmem_base_sh), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int* abort_flag = &abort_sh;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            mbar_arrive_expect_tx(bar(B_Q), (uint32_t)(g.M * D * 2));
            for (int hl = 0; hl < g.G; ++hl) {
                const int row = (b * g.Hq + kvh * g.G + hl) * g.T + t0;
                for (int h = 0; h < D / 64; ++h)
                    tma_load_2d(base + L::off_q + h * L::kQHalf + hl * g.P * 128, &tm_q, h * 64, row, bar(B_Q));
            }
            int last_armed[kTcStages];
            for (int st = 0; st < kTcStages; ++st) last_armed[st] = -1;
            for (int s = 0; s < n; ++s) {
                const int st = s % kTcStages;
                if (s >= kTcStages && !mbar_wait(bar(B_KV_EMPTY + st), ((s / kTcStages) - 1) & 1, abort_flag)) break;
                const int j = s < U ? lst[s] : bt;
                const int row = bg * g.T + j * kBlock;
                mbar_arrive_expect_tx(bar(B_KV_FULL + st), (uint32_t)(2 * kBlock * D * 2));
                for (int h = 0; h < D / 64; ++h) {
                    tma_load_2d(kv_addr(st) + h * L::kKVHalf, &tm_k, h * 64, row, bar(B_KV_FULL + st));
                    tma_load_2d(kv_addr(st) + L::kKV + h * L::kKVHalf, &tm_v, h * 64, row, bar(B_KV_FULL + st));
                }
                last_armed[st] = s;
            }
            if (*abort_flag) {
                // let every load this thread started land before the CTA exits
                volatile int dummy = 0;
                mbar_wait(bar(B_Q), 0, &dummy);
                for (int st = 0; st < kTcStages; ++st)
                    if (last_armed[st] >= 0) { dummy = 0; mbar_wait(bar(B_KV_FULL + st), (last_armed[st] / kTcStages) & 1, &dummy); }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16(128, 64, false);
            const uint32_t idesc_pv = idesc_bf16(128, D, true);
            auto issue_pv = [&](int p) -> bool {
                const int bp = p & 1, stp = p % kTcStages;
                if (!mbar_wait(bar(B_P_FULL + bp), (p >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t a = smem_desc_sw128(base + L::off_p + bp * L::kP + kk * 32, 16, 1024);
                    const uint64_t bv = smem_desc_sw128(kv_addr(stp) + L::kKV + kk * 2048, L::kKVHalf, 1024);
                    mma_bf16_ss(tmem + 128, a, bv, idesc_pv, (p > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(B_PV_DONE + bp));
                mma_commit(bar(B_KV_EMPTY + stp));
                return true;
            };
            bool ok = mbar_wait(bar(B_Q), 0, abort_flag);
            tc_fence_after();
            for (int s = 0; ok && s < n; ++s) {
                const int st = s % kTcStages, sb = s & 1;
                if (!mbar_wait(bar(B_KV_FULL + st), (s / kTcStages) & 1, abort_flag)) { ok = false; break; }
                if (s >= 2 && !mbar_wait(bar(B_S_FREE + sb), ((s - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int h = kk >> 2, wk = kk & 3;
                    const uint64_t a = smem_desc_sw128(base + L::off_q + h * L::kQHalf + wk * 32, 16, 1024);
                    const uint64_t bk = smem_desc_sw128(kv_addr(st) + h * L::kKVHalf + wk * 32, 16, 1024);
                    mma_bf16_ss(tmem + sb * 64, a, bk, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(B_S_FULL + sb));
                if (s >= 1 && !issue_pv(s - 1)) { ok = false; break; }
            }
            if (ok) ok = issue_pv(n - 1);
            if (!ok) {
                // every MMA this thread issued must finish before TMEM is released
                mma_commit(bar(B_DRAIN));
                volatile int dummy = 0;
                mbar_wait(bar(B_DRAIN), 0, &dummy);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warps 0..3
        const int r = tid;
        const int hl = r / g.P, t = t0 + r % g.P;
        const bool valid = r < g.M && t < g.T;
        const int tpos = valid ? t : -1;
        const float tau_r = (valid && bt > 0) ? tau[(size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t] : INFINITY;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        uint8_t* const prow_base = base_ptr + L::off_p + (r >> 3) * 1024 + (r & 7) * 128;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        // TMEM loads and stores are warp-collective: every wait result is made warp-uniform
        auto wwait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
            const bool got = mbar_wait(bar_addr, parity, abort_flag);
            return __all_sync(0xffffffffu, got);
        };
        for (int s = 0; s < n; ++s) {
            const int sb = s & 1;
            const int j = s < U ? lst[s] : bt;
            const bool diag = (j == bt);
            if (!wwait(bar(B_S_FULL + sb), (s >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            uint32_t sr[64];
            tmem_ld32(lane_addr + sb * 64, sr);
            tmem_ld32(lane_addr + sb * 64 + 32, sr + 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(B_S_FREE + sb));
            float rs = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) rs += __uint_as_float(sr[i]);
            const float x = rs * cxm;
            const float lp2 = diag ? (tpos >= 0 ? 0.f : -INFINITY)
                                   : (x > tau_r ? e_pow * __log2f(x - tau_r) : -INFINITY);
            const bool active = lp2 > -INFINITY;
            float mx = -INFINITY;
            if (active) {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    float l2 = fmaf(__uint_as_float(sr[i]), sm2, lp2);
                    if (diag && j * kBlock + i > tpos) l2 = -INFINITY;
                    sr[i] = __float_as_uint(l2);
                    mx = fmaxf(mx, l2);
                }
            }
            // running max and lazy rescale of the O row in TMEM
            float factor = 1.f;
            bool resc = false;
            if (active) {
                if (m_run == -INFINITY) {
                    m_run = mx;
                } else if (mx > m_run + kLazyRescale) {
                    factor = exp2f(m_run - mx);
                    l_run *= factor;
                    m_run = mx;
                    resc = true;
                }
            }
            if (__any_sync(0xffffffffu, resc)) {
                // O must include PV_{s-1} before it is scaled
                if (!wwait(bar(B_PV_DONE + ((s - 1) & 1)), ((s - 1) >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(lane_addr + 128 + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
                    tmem_st32(lane_addr + 128 + c * 32, o);
                }
                tmem_wait_st();
            }
            // P buffer sb was last read by PV_{s-2}
            if (s >= 2 && !wwait(bar(B_PV_DONE + sb), ((s - 2) >> 1) & 1)) { ok = false; break; }
            float psum = 0.f;
            uint8_t* prow = prow_base + sb * L::kP;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t pk[4];
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    float p0 = 0.f, p1 = 0.f;
                    if (active) {
                        p0 = exp2f(__uint_as_float(sr[c * 8 + 2 * q2]) - m_run);
                        p1 = exp2f(__uint_as_float(sr[c * 8 + 2 * q2 + 1]) - m_run);
                    }
                    psum += p0 + p1;
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    pk[q2] = *reinterpret_cast<uint32_t*>(&h2);
                }
                *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            l_run += psum;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar(B_P_FULL + sb));
        }
        // ---- epilogue: O / l -> bf16
        if (ok && wwait(bar(B_PV_DONE + ((n - 1) & 1)), ((n - 1) >> 1) & 1)) {
            tc_fence_after();
            const float inv = 1.0f / l_run;
            __nv_bfloat16* dst = valid ? out + ((size_t)(b * g.Hq + kvh * g.G + hl) * g.T + t) * D : nullptr;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_addr + 128 + c * 32, o);
                tmem_wait_ld();
                if (valid) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv,
                                                                  __uint_as_float(o[2 * i + 1]) * inv);
                        pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
    if (tid == 0 && abort_sh) atomicOr(&hdr->status, kStWaitTimeout);
}

// ------------------------------------------------------------------ host side

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D map over a [rows, d] bf16 matrix, boxes of 64 columns x box_rows rows, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* ptr, unsigned long long rows, int d, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fine_tc_supported(const PrefillGeom& g) { return g.P >= 8 && (g.d == 64 || g.d == 128); }

cudaError_t launch_fine_tc(const void* q, const void* k, const void* v, void* out, const PrefillGeom& g,
                           char* ws, float alpha, float coarse_scale, cudaStream_t stream) {
    const float cxm = (alpha - 1.0f) * coarse_scale / sqrtf((float)g.d) / (float)kBlock;
    const float e_pow = 1.0f / (alpha - 1.0f);
    const float sm2 = 1.4426950408889634f / sqrtf((float)g.d);
    CUtensorMap tq, tk, tv;
    const unsigned long long qrows = (unsigned long long)g.B * g.Hq * g.T;
    const unsigned long long kvrows = (unsigned long long)g.B * g.Hkv * g.T;
    if (!make_map(&tq, q, qrows, g.d, g.P) || !make_map(&tk, k, kvrows, g.d, kBlock) ||
        !make_map(&tv, v, kvrows, g.d, kBlock))
        return cudaErrorInvalidValue;
    const float* tau = reinterpret_cast<const float*>(ws + g.off_tau);
    const int* list = reinterpret_cast<const int*>(ws + g.off_list);
    const int* count = reinterpret_cast<const int*>(ws + g.off_count);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    if (g.d == 128) {
        const int sm = (int)TcLayout<128>::bytes;
        cudaError_t e = cudaFuncSetAttribute(fine_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        fine_tc_kernel<128><<<g.ntiles, kTcThreads, sm, stream>>>(tq, tk, tv, ob, tau, list, count, hdr, g, cxm, e_pow, sm2);
    } else {
        const int sm = (int)TcLayout<64>::bytes;
        cudaError_t e = cudaFuncSetAttribute(fine_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e != cudaSuccess) return e;
        fine_tc_kernel<64><<<g.ntiles, kTcThreads, sm, stream>>>(tq, tk, tv, ob, tau, list, count, hdr, g, cxm, e_pow, sm2);
    }
    return cudaGetLastError();
}

}  // namespace dash
