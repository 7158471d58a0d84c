// common.cuh -- shared device helpers and the workspace layout of the DashAttention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

namespace dash {

constexpr int kBlock = 64;        // tokens per key block (the only supported block size)
constexpr int kTileRows = 128;    // query rows per work tile (positions x heads of one group)
constexpr int kMaxT = 1 << 20;    // longest supported sequence
constexpr int kCoarseCTAs = 296;  // persistent coarse grid: 2 CTAs on each of 148 SMs
constexpr int kSolveMaxIt = 64;   // iteration cap of the threshold solve

// Device status bits (workspace header).
enum : int { kStNoConverge = 1, kStWaitTimeout = 2 };

// First 256 bytes of every workspace.
struct WsHeader {
    int status;
    int ticket;                   // CTAs of the decode select pass that have finished
    unsigned long long scored_pairs;
    unsigned long long selected_pairs;
    unsigned long long union_blocks;
    unsigned long long tiles;
    unsigned long long fine_steps;   // key blocks the prefill's fine stage processes, over all its tiles
    unsigned long long reserved[26];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Iteration cap of the threshold solves of a call: kSolveMaxIt, or the smaller value of the
// environment variable DASH_DEBUG_SOLVE_CAP (1 .. kSolveMaxIt), which exists to exercise the
// no-convergence status path with a normal, terminating launch.
inline int solve_cap_from_env() {
    const char* e = getenv("DASH_DEBUG_SOLVE_CAP");
    if (!e || !*e) return kSolveMaxIt;
    const long v = strtol(e, nullptr, 10);
    return (v >= 1 && v < kSolveMaxIt) ? (int)v : kSolveMaxIt;
}

// Geometry of a prefill call.  Work tiles are P consecutive positions (inside one key
// block) x the G query heads of one KV head: rows r = head_local * P + pos_local.
// Selection-ordered tiles (tensor-core path, G <= 16): the rows of a KV group are cut into
// windows of kOrderRows rows (W = kOrderRows / G positions x the G heads), each window's rows
// are sorted by a selection signature, and every 128 consecutive sorted rows form a tile
// whose block list is the union of its rows' selected blocks and own blocks.
constexpr int kOrderRows = 4096;
// row ids in the ordered tiles: (head in the KV group << kRowShift) | position (T <= 2^20)
constexpr int kRowShift = 20;
constexpr int kRowMask = (1 << kRowShift) - 1;
static_assert(kMaxT <= (1 << kRowShift), "positions fit the row id");

struct PrefillGeom {
    int B, Hq, Hkv, T, d, G, P, M;   // M = G * P rows used of the 128-row tile
    int ntile_bg;                    // tiles per (b, kv head) = ceil(T / P)
    int ntiles;                      // B * Hkv * ntile_bg
    int nbs;                         // complete blocks = T / 64
    int cap;                         // list capacity per tile = max(1, nbs)
    bool tc;                         // tensor-core Stage 1/2 kernels (needs P >= 8)
    int maxit;                       // iteration cap of the threshold solves
    int nbw;                         // 32-bit words of a row's selection bitmap = ceil(nbs / 32)
    int W;                           // positions per ordering window: a multiple of 64, W G <= 4096
    int ord_tw;                      // ordered tiles of a full window = ceil(W G / 128)
    int ord_bg;                      // ordered tiles per (b, kv head)
    int ord_ntiles;                  // B * Hkv * ord_bg
    int ord_cap;                     // list capacity of an ordered tile = ceil(T / 64)
    size_t off_ksum, off_khi, off_klo, off_tau, off_list, off_count, off_scratch;
    size_t off_rowbits, off_wcnt, off_ord_rows, off_ord_list, off_ord_count, total;
};

inline int pow2_floor(int x) {
    int p = 1;
    while (p * 2 <= x) p *= 2;
    return p;
}

inline bool make_prefill_geom(int B, int Hq, int Hkv, int T, int d, PrefillGeom* g) {
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || T > kMaxT || (Hq % Hkv) != 0) return false;
    if (d != 64 && d != 128) return false;
    if ((long long)B * Hq * T >= (1ll << 31)) return false;
    int G = Hq / Hkv;
    if (G > kTileRows) return false;
    g->B = B; g->Hq = Hq; g->Hkv = Hkv; g->T = T; g->d = d; g->G = G;
    int P = pow2_floor(kTileRows / G);
    if (P > kBlock) P = kBlock;
    g->P = P;
    g->M = G * P;
    g->ntile_bg = (T + P - 1) / P;
    g->ntiles = B * Hkv * g->ntile_bg;
    g->nbs = T / kBlock;
    g->cap = g->nbs > 0 ? g->nbs : 1;
    g->tc = P >= 8;
    g->maxit = solve_cap_from_env();
    g->nbw = (g->nbs + 31) / 32;
    g->W = (kOrderRows / G) / kBlock * kBlock;
    if (g->W < kBlock) g->W = kBlock;
    g->ord_tw = (g->W * G + kTileRows - 1) / kTileRows;
    {
        // full windows have ord_tw tiles each, the last one ceil(its rows / 128)
        const int nwin = (T + g->W - 1) / g->W;
        const long long rlast = (long long)(T - (nwin - 1) * g->W) * G;
        g->ord_bg = (nwin - 1) * g->ord_tw + (int)((rlast + kTileRows - 1) / kTileRows);
    }
    g->ord_ntiles = B * Hkv * g->ord_bg;
    g->ord_cap = (T + kBlock - 1) / kBlock;
    const size_t nsum = (size_t)B * Hkv * (g->nbs > 0 ? g->nbs : 1) * d;
    size_t off = align256(sizeof(WsHeader));
    g->off_ksum = off;    off = align256(off + nsum * sizeof(float));
    g->off_khi = off;     off = align256(off + nsum * 2);            // bf16 hi part of kbar
    g->off_klo = off;     off = align256(off + nsum * 2);            // bf16 lo part: kbar - hi
    g->off_tau = off;     off = align256(off + (size_t)B * Hq * T * sizeof(float));
    g->off_list = off;    off = align256(off + (size_t)g->ntiles * g->cap * sizeof(int));
    g->off_count = off;   off = align256(off + (size_t)g->ntiles * sizeof(int));
    int cgrid = g->ntiles < kCoarseCTAs ? g->ntiles : kCoarseCTAs;
    g->off_scratch = off; // per-CTA score slabs of the CUDA-core coarse kernel only
    if (!g->tc) off = align256(off + (size_t)cgrid * kTileRows * g->cap * sizeof(float));
    // selection-ordered tiles (tensor-core path only): per-row selection bitmaps, the rows
    // of every ordered tile, its block list and count
    g->off_rowbits = off;
    g->off_wcnt = off;
    g->off_ord_rows = off;
    g->off_ord_list = off;
    g->off_ord_count = off;
    if (g->tc && g->nbs > 0) {
        g->off_rowbits = off;   off = align256(off + (size_t)B * Hq * T * g->nbw * sizeof(unsigned));
        // per window, how many of its rows select each block (filled by the coarse stage)
        const int nwin = (T + g->W - 1) / g->W;
        g->off_wcnt = off;      off = align256(off + (size_t)B * Hkv * nwin * g->nbs * sizeof(unsigned));
        g->off_ord_rows = off;  off = align256(off + (size_t)g->ord_ntiles * kTileRows * sizeof(int));
        g->off_ord_list = off;  off = align256(off + (size_t)g->ord_ntiles * g->ord_cap * sizeof(int));
        g->off_ord_count = off; off = align256(off + (size_t)g->ord_ntiles * sizeof(int));
    }
    g->total = off;
    return true;
}

// Workspace of a backward call: the prefill workspace, then per row D = dout . out, the
// log2-domain log-sum-exp of the fine logits and r = sum_j H_j / sum_j g_j (fp32 each).
struct BwdGeom {
    size_t off_drow, off_lse, off_r, total;
};

inline void make_bwd_geom(const PrefillGeom& g, BwdGeom* bw) {
    const size_t rows = (size_t)g.B * g.Hq * g.T * sizeof(float);
    size_t off = g.total;
    bw->off_drow = off; off = align256(off + rows);
    bw->off_lse = off;  off = align256(off + rows);
    bw->off_r = off;    off = align256(off + rows);
    bw->total = off;
}

// Geometry of a decode call.
struct DecodeGeom {
    int B, Hq, Hkv, Tmax, d, G, nbs, chunk, maxchunks;
    int maxit;                       // iteration cap of the threshold solves
    size_t off_x, off_tau, off_list, off_count, off_done, off_offs, off_plan, off_part, total;
};

constexpr int kDecodeChunk = 16;     // list entries (key blocks) per split-KV work item
constexpr int kDecodeMaxCtas = 512;  // CTAs of the balanced split-KV attention pass

inline bool make_decode_geom(int B, int Hq, int Hkv, int Tmax, int d, DecodeGeom* g) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Tmax < 1 || Tmax > kMaxT || (Hq % Hkv) != 0) return false;
    if (d != 64 && d != 128) return false;
    int G = Hq / Hkv;
    if (G > 32) return false;
    g->B = B; g->Hq = Hq; g->Hkv = Hkv; g->Tmax = Tmax; g->d = d; g->G = G;
    g->nbs = Tmax / kBlock;
    g->chunk = kDecodeChunk;
    g->maxchunks = (g->nbs + 1 + kDecodeChunk - 1) / kDecodeChunk;
    g->maxit = solve_cap_from_env();
    int cap = g->nbs + 1;
    size_t off = align256(sizeof(WsHeader));
    g->off_x = off;     off = align256(off + (size_t)B * Hq * cap * sizeof(float));
    g->off_tau = off;   off = align256(off + (size_t)B * Hq * sizeof(float));
    g->off_list = off;  off = align256(off + (size_t)B * Hkv * cap * sizeof(int));
    g->off_count = off; off = align256(off + (size_t)B * Hkv * sizeof(int));
    g->off_done = off;  off = align256(off + (size_t)B * Hkv * sizeof(int));   // partials finished per group
    g->off_offs = off;  off = align256(off + ((size_t)B * Hkv + 1) * sizeof(int));   // prefix of counts
    g->off_plan = off;  off = align256(off + (size_t)kDecodeMaxCtas * sizeof(int));  // first group per CTA
    // partial (m, l, o[d]) per head in group and (b, kv head, chunk) -- or, for the balanced
    // pass, per (CTA + group) slot
    const size_t slots_chunk = (size_t)B * Hkv * g->maxchunks, slots_bal = (size_t)B * Hkv + kDecodeMaxCtas;
    const size_t slots = slots_chunk > slots_bal ? slots_chunk : slots_bal;
    g->off_part = off;  off = align256(off + slots * G * (d + 2) * sizeof(float));
    g->total = off;
    return true;
}

// ------------------------------------------------------------------ small device helpers

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ void bf16x8_to_float(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global->shared copy; src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" :: "n"(N)); }

}  // namespace dash
