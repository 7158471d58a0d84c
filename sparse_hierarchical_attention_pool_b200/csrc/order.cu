// order.cu -- selection-ordered tiles for the tensor-core fine stage.
//
// The fine stage runs 128 query rows of one KV group per tile over the union of their
// selected blocks ("DashAttention: Making Sparse Attention Fully Differentiable with Adaptive
// Block Selection", section "Core Mechanism": the selection is per query row, the gathered
// key/value blocks are shared by the rows of a tile).  Tiles of consecutive positions carry
// rows whose selections are nearly independent, so their union approaches every past block.
// This pass forms tiles from rows with similar selections instead: the rows of a window
// (W = 4096 / G positions, rounded down to whole blocks, x the G heads of a KV group) are
// sorted by a signature and cut into
// tiles of 128.
//
// Signature: one power-iteration step towards the leading principal axis of the window's
// selection matrix S (rows x blocks), started from the block selection counts:
//     c_j = #{rows r of the window : j in S_r},   score_r = sum_{j in S_r} c_j.
// Sorting by it places rows that select the window's common blocks next to each other (a
// spectral ordering of the rows).  The sort is a stable radix sort on (score, row), so the
// tiles, and every result computed from them, are deterministic.
//
// The block counts c_j of every window are accumulated by the coarse stage while it writes
// the row bitmaps.  order_rows_kernel, one CTA of 512 threads per window: a score per row (a
// thread per row, its bitmap words loaded 8 at a time), then a block-wide radix sort on the
// bits the scores use, which gives the rows of every tile.  A row id is
// (head in the KV group << kRowShift) | position, decoded with a shift and a mask.  order_union_kernel, one warp per tile: the OR of its rows' bitmaps (plus their own
// blocks), lanes as bitmap words, compacted into the tile's ascending list.
#include <cub/block/block_radix_sort.cuh>

#include "common.cuh"
#include "kernels.h"

namespace dash {

constexpr int kOrdThreads = 512;
constexpr int kOrdItems = kOrderRows / kOrdThreads;   // rows per thread (scoring) and sort items
constexpr int kTabWords = 16;                           // bitmap words per chunk of lookup tables
constexpr int kKeyBits = 18;                            // sort key: the score's leading 18 bits
constexpr int kSortRadix = 6;                           // radix bits per sort pass

// Bit mask of the valid blocks of word w of a row with bt complete past blocks.
__device__ __forceinline__ unsigned row_word_mask(int w, int bt) {
    const int rem = bt - w * 32;
    return rem >= 32 ? 0xFFFFFFFFu : (rem <= 0 ? 0u : ((1u << rem) - 1u));
}

// bytes of the block sort's storage, rounded up to 16
__host__ __device__ constexpr int order_sort_bytes() {
    return (int)((sizeof(typename cub::BlockRadixSort<unsigned, kOrdThreads, kOrdItems, int, kSortRadix>::TempStorage) + 15) / 16 * 16);
}

__global__ void __launch_bounds__(kOrdThreads, 1)
order_rows_kernel(const unsigned* __restrict__ rowbits, const unsigned* __restrict__ wcnt, int* __restrict__ ord_rows,
                  PrefillGeom g) {
    using Sort = cub::BlockRadixSort<unsigned, kOrdThreads, kOrdItems, int, kSortRadix>;
    // dynamic: the sort's storage, [kOrderRows] row scores (then the window's rows by rank),
    // [kTabWords][4][256] tables, [nbw * 32] block counts
    extern __shared__ __align__(16) unsigned char dyn_raw[];
    typename Sort::TempStorage& sort_tmp = *reinterpret_cast<typename Sort::TempStorage*>(dyn_raw);
    unsigned* const score = reinterpret_cast<unsigned*>(dyn_raw + order_sort_bytes());
    int* const sorted = reinterpret_cast<int*>(score);
    unsigned short* const tab = reinterpret_cast<unsigned short*>(score + kOrderRows);
    unsigned* const cnt = reinterpret_cast<unsigned*>(tab + kTabWords * 1024);
    __shared__ unsigned smax_sh;

    const int nwin = (g.T + g.W - 1) / g.W;
    const int bg = blockIdx.x / nwin, win = blockIdx.x % nwin;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const int p0 = win * g.W, np = min(g.W, g.T - p0); // positions of the window
    const int R = np * g.G;                             // rows: ri = hl * np + (t - p0)
    const int tid = threadIdx.x, lane = tid & 31;
    const size_t row0 = (size_t)(b * g.Hq + kvh * g.G) * g.T;

    const int nbt = (p0 + np - 1) / kBlock + 1;         // blocks 0 .. nbt-1 (own blocks included)
    const int nwm = min(g.nbw, (nbt + 31) / 32);        // bitmap words any row of the window uses
    // the window's block counts, accumulated by the coarse stage
    const unsigned* wc = wcnt + ((size_t)bg * nwin + win) * g.nbs;
    for (int i = tid; i < nwm * 32; i += kOrdThreads) cnt[i] = i < g.nbs ? wc[i] : 0u;
    if (tid == 0) smax_sh = 0u;
    // this thread's rows ri = tid + 512 k: (head in group, position), one division each
    int rh[kOrdItems], rt[kOrdItems];
#pragma unroll
    for (int k = 0; k < kOrdItems; ++k) {
        const int ri = tid + k * kOrdThreads;
        rh[k] = ri < R ? ri / np : -1;
        rt[k] = ri < R ? p0 + ri - rh[k] * np : 0;
    }
    // ---- signature score_r = sum of the counts of the row's selected blocks, through tables
    // of 256 entries per bitmap byte (entry v = the sum of the counts of the byte's set bits;
    // at most 8 x 4096, so 16 bits): four lookups per 32-block word, in chunks of kTabWords
    // words whose tables are rebuilt per chunk
    unsigned sc[kOrdItems];
#pragma unroll
    for (int k = 0; k < kOrdItems; ++k) sc[k] = 0u;
    for (int w0 = 0; w0 < nwm; w0 += kTabWords) {
        const int nwc = min(kTabWords, nwm - w0);
        __syncthreads();                                // counts loaded; previous tables read
        for (int e = tid; e < nwc * 1024; e += kOrdThreads) {
            const unsigned* cc = cnt + 32 * (w0 + (e >> 10)) + 8 * ((e >> 8) & 3);
            const unsigned v = e & 255u;
            unsigned sum = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) sum += ((v >> i) & 1u) ? cc[i] : 0u;
            tab[e] = (unsigned short)sum;
        }
        __syncthreads();
#pragma unroll 1
        for (int k = 0; k < kOrdItems; ++k) {
            if (rh[k] < 0) continue;
            const int t = rt[k], bt = t / kBlock, nwr = (bt + 31) / 32;
            const unsigned* rb = rowbits + (row0 + (size_t)rh[k] * g.T + t) * g.nbw;
            unsigned wv[kTabWords];
#pragma unroll
            for (int w = 0; w < kTabWords; ++w)         // independent loads in flight
                wv[w] = (w < nwc && w0 + w < nwr) ? rb[w0 + w] & row_word_mask(w0 + w, bt) : 0u;
            unsigned s = 0u;
#pragma unroll
            for (int w = 0; w < kTabWords; ++w) {
                if (w >= nwc) break;
                const unsigned short* tw = tab + w * 1024;
                s += tw[wv[w] & 255u] + tw[256 + ((wv[w] >> 8) & 255u)] + tw[512 + ((wv[w] >> 16) & 255u)]
                   + tw[768 + (wv[w] >> 24)];
            }
            sc[k] += s;
        }
    }
    unsigned my_max = 0u;
#pragma unroll
    for (int k = 0; k < kOrdItems; ++k)
        if (rh[k] >= 0) {
            score[tid + k * kOrdThreads] = sc[k];
            my_max = max(my_max, sc[k]);
        }
    my_max = __reduce_max_sync(0xffffffffu, my_max);
    if (lane == 0) atomicMax(&smax_sh, my_max);
    __syncthreads();
    // ---- stable sort on the score's leading kKeyBits bits (rows of nearly equal score keep
    // their window order; blocked arrangement: thread i holds ranks 8 i .. 8 i + 7); padding
    // rows (past R) take the largest key and, being last, sort after every row
    const int nbits = 32 - __clz((int)(smax_sh | 1u));  // bits of max(score)
    const int shift = nbits > kKeyBits ? nbits - kKeyBits : 0;
    const int kbits = nbits - shift;                     // <= kKeyBits
    const unsigned pad = (1u << kbits) - 1u;
    // values: the row ids of the ordered-tile lists, (head in group << 20) | position
    unsigned keys[kOrdItems];
    int vals[kOrdItems];
#pragma unroll
    for (int k = 0; k < kOrdItems; ++k) {
        const int ri = tid * kOrdItems + k;
        const int hl = ri / np;                         // one division per item
        keys[k] = ri < R ? score[ri] >> shift : pad;
        vals[k] = ri < R ? (hl << kRowShift) | (p0 + ri - hl * np) : -1;
    }
    Sort(sort_tmp).Sort(keys, vals, 0, kbits);
    // the scores were read into keys before the sort: their space takes the sorted rows
#pragma unroll
    for (int k = 0; k < kOrdItems; ++k) sorted[tid * kOrdItems + k] = vals[k];
    __syncthreads();
    const int ntw = (R + kTileRows - 1) / kTileRows;
    const size_t tile0 = (size_t)bg * g.ord_bg + (size_t)win * g.ord_tw;
    for (int i = tid; i < ntw * kTileRows; i += kOrdThreads) ord_rows[tile0 * kTileRows + i] = i < R ? sorted[i] : -1;
}

// One warp per ordered tile: the union of its rows' selected blocks and own blocks.  Lanes
// take 32 consecutive bitmap words and OR them over the tile's rows (one coalesced load per
// row), then a scan of the words' popcounts places their set bits in the ascending list.
constexpr int kUnionWarps = 8;

__global__ void __launch_bounds__(kUnionWarps * 32)
order_union_kernel(const unsigned* __restrict__ rowbits, const int* __restrict__ ord_rows, int* __restrict__ ord_list,
                   int* __restrict__ ord_count, WsHeader* __restrict__ hdr, PrefillGeom g) {
    __shared__ int bt_sh[kUnionWarps][kTileRows];                    // own block, -1: no row
    __shared__ const unsigned* rb_sh[kUnionWarps][kTileRows];         // the row's bitmap
    const int lane = threadIdx.x & 31, wl_ = threadIdx.x >> 5;
    const int tile = blockIdx.x * kUnionWarps + wl_;
    if (tile >= g.ord_ntiles) return;                   // whole warp
    const int bg = tile / g.ord_bg;
    const int b = bg / g.Hkv, kvh = bg % g.Hkv;
    const size_t row0 = (size_t)(b * g.Hq + kvh * g.G) * g.T;
    int btmax = 0;
    for (int k = lane; k < kTileRows; k += 32) {
        const int rid = ord_rows[(size_t)tile * kTileRows + k];
        const int t = rid & kRowMask, hl = rid >> kRowShift;
        const int bt = rid >= 0 ? t / kBlock : -1;
        bt_sh[wl_][k] = bt;
        rb_sh[wl_][k] = rowbits + (row0 + (rid >= 0 ? (size_t)hl * g.T + t : 0)) * g.nbw;
        btmax = max(btmax, bt);
    }
    btmax = __reduce_max_sync(0xffffffffu, btmax);
    __syncwarp();
    const int nwt = btmax / 32 + 1;                     // words holding any listed block
    int* dst = ord_list + (size_t)tile * g.ord_cap;
    int total = 0;
    for (int wb = 0; wb < nwt; wb += 32) {
        // lanes = (row offset, word): nwp lanes (a power of two >= the chunk's words) per row,
        // 32 / nwp rows per load, 8 loads in flight; an OR over the row offsets follows
        const int nww = min(32, nwt - wb);
        const int nwp = nww <= 1 ? 1 : 1 << (32 - __clz(nww - 1));
        const int rpl = 32 / nwp;
        const int wl = lane & (nwp - 1), ro = lane / nwp;
        const int w = wb + wl;
        const bool wok = wl < nww;
        unsigned word = 0u;
        for (int k0 = 0; k0 < kTileRows; k0 += 8 * rpl) {
            unsigned wv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {                   // 8 independent loads in flight
                const int row = k0 + k * rpl + ro;
                const int bt = row < kTileRows ? bt_sh[wl_][row] : -1;
                wv[k] = (wok && bt >= 0 && w * 32 < bt) ? rb_sh[wl_][row][w] & row_word_mask(w, bt) : 0u;
                if (wok && bt >= 0 && (bt >> 5) == w) wv[k] |= 1u << (bt & 31);   // own block
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) word |= wv[k];
        }
        for (int o = nwp; o < 32; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
        // lanes 0 .. nww-1 hold words wb .. wb + nww - 1
        const int pc = lane < nww ? __popc(word) : 0;
        int incl = pc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nn = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += nn;
        }
        if (lane < nww) {
            int pos = total + incl - pc;
            while (word) {
                dst[pos++] = (wb + lane) * 32 + __ffs(word) - 1;
                word &= word - 1u;
            }
        }
        total += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        ord_count[tile] = total;
        atomicAdd(&hdr->union_blocks, (unsigned long long)total);
        atomicAdd(&hdr->tiles, 1ull);
        atomicAdd(&hdr->fine_steps, (unsigned long long)total);
    }
}

cudaError_t launch_order_tiles(const PrefillGeom& g, char* ws, cudaStream_t stream) {
    if (!g.tc || g.nbs == 0) return cudaErrorInvalidValue;
    const int nwin = (g.T + g.W - 1) / g.W;
    const unsigned* rowbits = reinterpret_cast<const unsigned*>(ws + g.off_rowbits);
    int* ord_rows = reinterpret_cast<int*>(ws + g.off_ord_rows);
    const int sm = order_sort_bytes() + (kOrderRows + g.nbw * 32) * (int)sizeof(unsigned) +
                   kTabWords * 1024 * (int)sizeof(unsigned short);
    cudaError_t e = cudaFuncSetAttribute(order_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    order_rows_kernel<<<g.B * g.Hkv * nwin, kOrdThreads, sm, stream>>>(
        rowbits, reinterpret_cast<const unsigned*>(ws + g.off_wcnt), ord_rows, g);
    order_union_kernel<<<(g.ord_ntiles + kUnionWarps - 1) / kUnionWarps, kUnionWarps * 32, 0, stream>>>(
        rowbits, ord_rows, reinterpret_cast<int*>(ws + g.off_ord_list), reinterpret_cast<int*>(ws + g.off_ord_count),
        reinterpret_cast<WsHeader*>(ws), g);
    return cudaGetLastError();
}

}  // namespace dash
