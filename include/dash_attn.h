/*
 * dash_attn.h -- C ABI of the B200 (sm_100a) DashAttention forward pass.
 *
 * DashAttention (pages: "DashAttention: Making Sparse Attention Fully Differentiable with
 * Adaptive Block Selection", sections "Core Mechanism" and "Key Concepts"; "DashAttention
 * and the year sparse attention became a field", section "What alpha-entmax changes"):
 *   Stage 0  keys are split into blocks of `block` tokens and mean-pooled into summaries
 *            kbar_j (a zero-initialised learned summary head is exactly mean pooling);
 *   Stage 1  per query head, coarse scores s_j = coarse_scale * (q . kbar_j) / sqrt(d) over
 *            the complete blocks strictly before the query's own block; alpha-entmax
 *            p_j = [(alpha-1) s_j - tau]_+^(1/(alpha-1)), tau chosen so that sum_j p_j = 1,
 *            gives a sparse, variable-size block set;
 *   Stage 2  softmax attention over the tokens of the selected blocks plus the query's own
 *            block (causal, prior weight 1), with logits (q . k_i)/sqrt(d) + log p_block(i).
 * Query head h reads KV head h / (Hq / Hkv).
 *
 * Conventions for every entry point:
 *   - q, k, v, out, caches are bf16, row-major, last dimension d contiguous:
 *       q, out [B, Hq, T, d];  k, v [B, Hkv, T, d];  caches [B, Hkv, Tmax, d].
 *     Every tensor pointer must be 16-byte aligned.
 *   - All pointers are DEVICE pointers owned by the caller unless stated otherwise.  The
 *     library allocates no memory and keeps no state between calls; scratch lives in a
 *     caller-provided workspace whose size the *_workspace_size functions return.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).  Argument errors
 *     are returned at once and nothing is launched.  Calls that use the same workspace
 *     concurrently race.
 *   - Supported: d in {64, 128}; block == 64; Hq % Hkv == 0 and Hq / Hkv <= 128;
 *     1 <= T <= 1048576; alpha > 1 and finite; coarse_scale finite.
 *   - Device-side conditions (a threshold solve that hit its iteration cap) set a status
 *     word inside the workspace; dash_get_device_status reads it.  The environment
 *     variable DASH_DEBUG_SOLVE_CAP=n (1 <= n < 64), read at each call, lowers that cap to
 *     n iterations so that the status path can be exercised with a normal launch; rows
 *     whose solve is cut short get an inexact threshold.
 *   - Other environment switches (all off by default; they choose among kernels that compute
 *     the same result, for comparisons):
 *       DASH_TILES=positions      (read at each prefill) the fine stage runs tiles of
 *                                 consecutive positions instead of selection-ordered tiles;
 *       DASH_ENTMAX_INIT=histogram (read at each call) the threshold solves start at a
 *                                 histogram edge below the root (AdaSplash-2's start) instead
 *                                 of the default subset root (prefill) or u = -1 (decode);
 *       DASH_FINE_KERNEL=mma, DASH_BWD_KERNEL=mma (read once per process) the prefill's fine
 *                                 stage, or its backward, on the mma.sync kernels that serve
 *                                 more than 16 query heads per KV head.
 *   - No C++ exception crosses this interface.
 */
#ifndef DASH_ATTN_H
#define DASH_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DASH_API __attribute__((visibility("default")))
#else
#define DASH_API
#endif

struct CUstream_st;
typedef struct CUstream_st* dash_stream_t;   /* same handle as cudaStream_t */

typedef enum {
    DASH_OK = 0,
    DASH_ERR_ARG = -1,           /* null / misaligned pointer, bad alpha or scale */
    DASH_ERR_SHAPE = -2,         /* unsupported B, H, T, d or block */
    DASH_ERR_DTYPE = -3,         /* reserved: every tensor is bf16 */
    DASH_ERR_UNSUPPORTED = -4,   /* valid request the library does not implement */
    DASH_ERR_WORKSPACE = -5,     /* workspace null, misaligned (256 B) or too small */
    DASH_ERR_CUDA = -6,          /* a CUDA runtime call failed (launch, copy) */
    DASH_ERR_NO_CONVERGE = -7,   /* device status: a tau solve hit its iteration cap */
    DASH_ERR_SCRATCH_LIMIT = -8, /* dash_decode_noalloc: the step needs more scratch than
                                    the library's fixed array holds */
    DASH_ERR_DEVICE_TIMEOUT = -9,/* device status: a kernel's bounded wait gave up (about 2 s);
                                    the outputs of that call are invalid */
    DASH_ERR_SETUP_IN_CAPTURE = -10 /* dash_decode_noalloc: its once-per-device set-up (a symbol
                                    lookup) was due while `stream` was being captured; make
                                    one call outside capture first */
} dash_status;

/* Human-readable name of a status code (static string, never NULL). */
DASH_API const char* dash_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
DASH_API int dash_version(void);

/*
 * Stage 0 (block summaries).  ksum[b, g, j, :] = mean of k[b, g, j*block : (j+1)*block, :]
 * for every COMPLETE block j < T / block, accumulated and stored in fp32.
 *   k     device bf16 [B, Hkv, T, d]
 *   ksum  device fp32 [B, Hkv, T / block, d]   (nothing is written when T < block)
 * Decode callers keep ksum for their KV cache by calling this on the cache (T = Tmax) or
 * on each block as it fills.
 */
DASH_API int dash_block_summary(const void* k, float* ksum, int B, int Hkv, int T, int d, int block,
                       dash_stream_t stream);

/*
 * Stage 0 with a learned summary head ("DashAttention and the year sparse attention became
 * a field", section "What alpha-entmax changes": the chunk summary is a small attention
 * head whose zero initialisation makes it the block mean).  Attention pooling
 * with one query vector per KV head:
 *   ksum[b, g, j, :] = sum_i a_i k[b, g, j*block + i, :],  a = softmax_i(w[g] . k_i / sqrt(d))
 * over the block's keys; w = 0 gives the mean of dash_block_summary (up to rounding).
 *   k     device bf16 [B, Hkv, T, d]
 *   w     device fp32 [Hkv, d], 16-byte aligned (must not be NULL)
 *   ksum  device fp32 [B, Hkv, T / block, d]
 * Use it to keep the summaries of a decode cache for a model with a learned head.
 */
DASH_API int dash_block_summary_w(const void* k, const float* w, float* ksum, int B, int Hkv, int T,
                                  int d, int block, dash_stream_t stream);

/* Bytes of workspace dash_prefill needs (0 when the shape is unsupported). */
DASH_API size_t dash_prefill_workspace_size(int B, int Hq, int Hkv, int T, int d, int block);

/*
 * Full causal prefill: Stages 0-2 for every query row (b, h, t), t in [0, T).
 *   q [B,Hq,T,d], k, v [B,Hkv,T,d] -> out [B,Hq,T,d], all device bf16.
 *   alpha > 1 (1.5 is the pages' inference value); coarse_scale multiplies the coarse
 *   scores only (fine logits always use 1/sqrt(d)).
 *   workspace: device, 256-byte aligned, >= dash_prefill_workspace_size(...) bytes.  It
 *   holds the block summaries, per-row thresholds, per-tile block lists and counters of
 *   this call until the next call that uses it.
 * Rows in block 0 have no past blocks and attend causally to their own block only.
 */
DASH_API int dash_prefill(const void* q, const void* k, const void* v, void* out,
                 int B, int Hq, int Hkv, int T, int d, int block,
                 float alpha, float coarse_scale,
                 void* workspace, size_t ws_bytes, dash_stream_t stream);

/*
 * dash_prefill with the learned summary head of dash_block_summary_w for Stage 0.
 *   w_summary  device fp32 [Hkv, d], 16-byte aligned; NULL is dash_prefill (mean pooling).
 * Returns DASH_ERR_UNSUPPORTED for a non-NULL head when a tile holds fewer than 8
 * positions (more than 16 query heads per KV head): that path's fine kernel recovers
 * q . kbar from the mean of the block's scores, which only the mean summary satisfies.
 */
DASH_API int dash_prefill_w(const void* q, const void* k, const void* v, const float* w_summary, void* out,
                            int B, int Hq, int Hkv, int T, int d, int block, float alpha,
                            float coarse_scale, void* workspace, size_t ws_bytes, dash_stream_t stream);

/* Bytes of workspace dash_prefill_backward needs (0 when the shape is unsupported). */
DASH_API size_t dash_prefill_backward_workspace_size(int B, int Hq, int Hkv, int T, int d, int block);

/*
 * Gradients of dash_prefill ("DashAttention: Making Sparse Attention Fully Differentiable
 * with Adaptive Block Selection", sections "Core Mechanism" and "Key Concepts": the block
 * selection is differentiable, so gradients flow through the fine softmax, the log prior,
 * the alpha-entmax Jacobian on the support, the coarse scores and the mean summaries).
 *   q, k, v    the forward's inputs (device bf16, layouts as dash_prefill);
 *   out        dash_prefill's output for them (device bf16 [B,Hq,T,d]);
 *   dout       d loss / d out (device bf16 [B,Hq,T,d]);
 *   dq         written: d loss / d q  (device bf16 [B,Hq,T,d]);
 *   dk, dv     written: d loss / d k, d loss / d v (device bf16 [B,Hkv,T,d]), including the
 *              summary path into every key of a complete block.
 *   workspace  device, 256-byte aligned, >= dash_prefill_backward_workspace_size(...) bytes;
 *              the call recomputes the summaries, thresholds and tile lists into it.
 * Mean-pooled summaries and per-head priors only (the dash_prefill configuration).  The
 * output is deterministic: no atomics, every gradient element has one writer.
 */
DASH_API int dash_prefill_backward(const void* q, const void* k, const void* v, const void* out,
                                   const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                                   int T, int d, int block, float alpha, float coarse_scale,
                                   void* workspace, size_t ws_bytes, dash_stream_t stream);

/* Flags of dash_prefill_ex / dash_decode_ex. */
#define DASH_HEAD_AGGREGATION 1u

/*
 * dash_prefill with options.
 *   w_summary  learned summary head as in dash_prefill_w (NULL: mean pooling).
 *   flags      0 or DASH_HEAD_AGGREGATION: entmax head aggregation ("DashAttention and the
 *              year sparse attention became a field", section "Non-dispersive attention at
 *              long context").  The G heads of a KV group average their alpha-entmax block
 *              weights at each position, pbar_j = (1/G) sum_h p_hj, and every head of the
 *              group takes log pbar_j as its fine-stage prior (the own block keeps prior 1);
 *              the thresholds and block lists stay per head.
 * Unknown flag bits return DASH_ERR_ARG.  A learned head or head aggregation returns
 * DASH_ERR_UNSUPPORTED when a tile holds fewer than 8 positions (more than 16 query heads
 * per KV head).
 */
DASH_API int dash_prefill_ex(const void* q, const void* k, const void* v, const float* w_summary, void* out,
                             int B, int Hq, int Hkv, int T, int d, int block, float alpha,
                             float coarse_scale, unsigned flags, void* workspace, size_t ws_bytes,
                             dash_stream_t stream);

/*
 * dash_prefill with HOST inputs and output: copies q, k, v from host memory into the
 * caller's device buffers, runs the prefill, copies out back to host memory, asynchronously
 * with respect to the host and ordered after the work already on `stream`; `stream` waits
 * for the last copy (host buffers should be pinned for the copies to overlap).
 * Host pointers: q_host, k_host, v_host (read), out_host (written).  Device pointers:
 * q_dev, k_dev, v_dev, out_dev (same shapes as dash_prefill) and the workspace.
 * The rows of a query head depend only on its queries and its (b, kv head) group's keys and
 * values, so the call pipelines units of one group and a chunk of its heads (about 8 MiB of
 * queries each): the copies of one unit overlap the kernels of others (short-lived helper
 * streams: copies in, copies out, and up to four compute streams, so that the kernels of
 * several units run at once; a group's keys and values are copied once, with its first
 * chunk).  With more than one unit each compute stream works in its own slice of the
 * workspace (after its 256-byte header); the header then holds the OR of every unit's device
 * status bits (dash_get_device_status) and the sums of their statistics (dash_prefill_stats),
 * and the rest of the workspace (thresholds) is unspecified.
 */
DASH_API int dash_prefill_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                      void* q_dev, void* k_dev, void* v_dev, void* out_dev,
                      int B, int Hq, int Hkv, int T, int d, int block,
                      float alpha, float coarse_scale,
                      void* workspace, size_t ws_bytes, dash_stream_t stream);

/*
 * dash_prefill that also records four caller-created CUDA events on `stream`:
 * events[0] before the block-summary kernel, events[1] before the coarse (Stage 1) kernel,
 * events[2] before the fine (Stage 2) kernel and events[3] after it.  `events` is a host
 * array of cudaEvent_t handles; the elapsed times between them are the per-kernel times.
 */
DASH_API int dash_prefill_profiled(const void* q, const void* k, const void* v, void* out,
                                   int B, int Hq, int Hkv, int T, int d, int block,
                                   float alpha, float coarse_scale,
                                   void* workspace, size_t ws_bytes, dash_stream_t stream,
                                   void* const* events);

/* Counters the last dash_prefill or dash_decode wrote into its workspace. */
typedef struct {
    long long scored_pairs;    /* sum over rows of the number of scored past blocks */
    long long selected_pairs;  /* sum over rows of #{j : p_j > 0} */
    long long union_blocks;    /* sum over work tiles of their block lists: the union of their
                                  rows' selected past blocks (position tiles; decode groups) or
                                  of their selected and own blocks (selection-ordered tiles) */
    long long tiles;           /* work tiles with at least one past block */
    int status;                /* device status bits (0 = clean) */
    long long fine_steps;      /* prefill: key blocks the fine stage processes, summed over its
                                  tiles (128 rows each); executed fine FLOPs = 4 d 64 128 x this */
} dash_stats;

/* Synchronises `stream`, then copies the counters out of `workspace` into *out (host). */
DASH_API int dash_prefill_stats(const void* workspace, size_t ws_bytes, dash_stats* out, dash_stream_t stream);
DASH_API int dash_decode_stats(const void* workspace, size_t ws_bytes, dash_stats* out, dash_stream_t stream);

/*
 * Per-row thresholds the last dash_prefill computed: tau_out[b, h, t] (device fp32,
 * [B, Hq, T]) in the (alpha-1)*s space of the entmax formula.  Rows in block 0 get NaN.
 * Same shape arguments as the dash_prefill call that filled the workspace.
 */
DASH_API int dash_prefill_tau(const void* workspace, size_t ws_bytes, float* tau_out,
                     int B, int Hq, int Hkv, int T, int d, int block, dash_stream_t stream);

/*
 * dash_prefill that also reports, for caller-chosen rows, the block weights the fine stage
 * (Stage 2) actually applied: the parity hook of the selection on the prefill's own path
 * ("DashAttention: Making Sparse Attention Fully Differentiable with Adaptive Block
 * Selection", section "Core Mechanism": Stage 1 hands its sparse block weights to Stage 2
 * as a log prior).  Outputs and workspace contents are those of dash_prefill_ex with the
 * same arguments; the kernels run in a variant that also writes the dump.
 *   w_summary, flags  as in dash_prefill_ex.
 *   row_slot  device int32 [B, Hq, T]: slot s in [0, nslots) of each reported row, -1 for
 *             rows not reported (two rows must not share a slot).
 *   x_out     device fp32 [nslots, T / block]: for every block j in the row's work-tile
 *             list, x_j = (alpha - 1) s_j as Stage 2 recomputed it; NaN for blocks not
 *             listed (those get no weight).
 *   p_out     device fp32 [nslots, T / block]: the row's own alpha-entmax weight of block j
 *             that Stage 2 applied, [x_j - tau]_+^(1/(alpha-1)); 0 for unlisted blocks.
 *   The threshold tau of each row is read afterwards with dash_prefill_tau.
 * Returns DASH_ERR_UNSUPPORTED when a tile holds fewer than 8 positions (more than 16
 * query heads per KV head: the CUDA-core fine kernel has no dump variant).
 */
DASH_API int dash_prefill_dump(const void* q, const void* k, const void* v, const float* w_summary, void* out,
                               int B, int Hq, int Hkv, int T, int d, int block, float alpha,
                               float coarse_scale, unsigned flags, const int* row_slot, int nslots,
                               float* x_out, float* p_out, void* workspace, size_t ws_bytes,
                               dash_stream_t stream);

/*
 * Block-weight recomputation for listed rows (an independent fp32 path, for analysis).
 * For each listed row (b, h, t):
 *   rows      device int64 [nrows, 3]
 *   ksum      device fp32 [B, Hkv, T / block, d]  (from dash_block_summary)
 *   out_idx   device int32 [nrows, max_sel]  selected past blocks, ascending
 *   out_p     device fp32  [nrows, max_sel]  their entmax weights
 *   out_count device int32 [nrows]           full support size (may exceed max_sel;
 *                                            only the first max_sel entries are written)
 *   out_tau   device fp32  [nrows]           threshold (NaN when t < block)
 * Scores are serial fp32 dot products of q with the fp32 summaries and the threshold comes
 * from a one-thread solve.  This is NOT dash_prefill's arithmetic (tensor-core products
 * with the summaries split into bf16 hi + lo parts, per-row passes shared by two threads):
 * the two agree to fp32 rounding of the scores.  dash_prefill_dump reports the weights the
 * prefill itself applies.
 */
DASH_API int dash_select_dump(const void* q, const float* ksum, const long long* rows, int nrows, int max_sel,
                     int* out_idx, float* out_p, int* out_count, float* out_tau,
                     int B, int Hq, int Hkv, int T, int d, int block,
                     float alpha, float coarse_scale, dash_stream_t stream);

/* Bytes of workspace dash_decode needs (0 when the shape is unsupported). */
DASH_API size_t dash_decode_workspace_size(int B, int Hq, int Hkv, int Tmax, int d, int block);

/*
 * One decode step: for each sequence b the new token's K/V are already in the cache at
 * position kv_len[b] - 1, and the query attends exactly as row t = kv_len[b] - 1 of a
 * prefill over the first kv_len[b] cache entries would.
 *   q        device bf16 [B, Hq, d]
 *   k_cache, v_cache  device bf16 [B, Hkv, Tmax, d]
 *   ksum     device fp32 [B, Hkv, Tmax / block, d]; blocks j < (kv_len[b]-1)/block must
 *            hold the summaries of the cache (dash_block_summary)
 *   kv_len   device int32 [B], 1 <= kv_len[b] <= Tmax (rows outside the range output 0
 *            and set no status)
 *   out      device bf16 [B, Hq, d]
 */
DASH_API int dash_decode(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d, int block,
                float alpha, float coarse_scale, void* workspace, size_t ws_bytes,
                dash_stream_t stream);

/*
 * dash_decode with options: flags 0 or DASH_HEAD_AGGREGATION (as in dash_prefill_ex).  Head
 * aggregation returns DASH_ERR_UNSUPPORTED for more than 8 query heads per KV head.
 */
DASH_API int dash_decode_ex(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                            const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d, int block,
                            float alpha, float coarse_scale, unsigned flags, void* workspace,
                            size_t ws_bytes, dash_stream_t stream);

/*
 * dash_decode that also reports the block weights its attention kernel applied (the decode
 * step's selection parity hook; see dash_prefill_dump).  Outputs are those of
 * dash_decode_ex with the same arguments.
 *   x_out    device fp32 [B, Hq, Tmax / block]: for every past block j in the (b, KV head)
 *            union list, x_j = (alpha - 1) s_j of head h; NaN for blocks not listed.
 *   p_out    device fp32 [B, Hq, Tmax / block]: head h's own alpha-entmax weight of block j
 *            as applied, [x_j - tau]_+^(1/(alpha-1)); 0 for unlisted blocks.
 *   tau_out  device fp32 [B, Hq]: the thresholds (NaN for rows without past blocks).
 * Returns DASH_ERR_UNSUPPORTED for more than 8 query heads per KV head.
 */
DASH_API int dash_decode_dump(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                              const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d, int block,
                              float alpha, float coarse_scale, unsigned flags, float* x_out, float* p_out,
                              float* tau_out, void* workspace, size_t ws_bytes, dash_stream_t stream);

/*
 * dash_decode that also records four caller-created CUDA events on `stream`: events[0]
 * before the coarse kernels (scores, then thresholds and block lists), events[1] before the
 * attention kernel, events[2] after it (before the partial merge kernel, which only the
 * path for more than 8 query heads per KV group launches) and events[3] at the end.
 */
DASH_API int dash_decode_profiled(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                                  const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d,
                                  int block, float alpha, float coarse_scale, void* workspace,
                                  size_t ws_bytes, dash_stream_t stream, void* const* events);

/*
 * dash_decode without a workspace argument, for callers that cannot allocate device memory
 * where they decode: real-time serving loops that must not take the device-wide
 * synchronisation cudaMalloc / cudaFree can cause, hosts whose device memory belongs to an
 * allocator this library cannot call, and plug-in code that is handed only its input and
 * output buffers.  The pages describe no such entry point; it has no counterpart in the
 * paper.
 *   Arguments, layouts and results are those of dash_decode; the caller still owns and
 *   passes every input and output buffer.
 *   Scratch is one 32 MiB array in device memory that the library declares statically:
 *   every GPU that loads the library holds it until the process exits.  A decode step
 *   whose scratch (dash_decode_workspace_size) exceeds 32 MiB is rejected with
 *   DASH_ERR_SCRATCH_LIMIT before anything is launched (the 96K workload, B=8, Hq=32,
 *   Hkv=8, d=128, needs about 15 MiB).
 *   Set-up: the first call on a device looks the array's device address up
 *   (cudaGetSymbolAddress, with that device current) and caches it with the identity of
 *   the device's context; a call on a context created since (after cudaDeviceReset, for
 *   instance) repeats the lookup.  Make that first call before any stream capture begins:
 *   a set-up that falls due while `stream` is being captured returns
 *   DASH_ERR_SETUP_IN_CAPTURE and launches nothing.
 *   No memory is allocated or freed.  Every call, on every stream, shares the one array
 *   and leaves its contents behind; the counters that must start at zero are cleared at
 *   the start of each call.  Calls whose executions overlap on the GPU (other streams,
 *   other host threads) race on the array and give wrong results: serialise them.
 *   The device status of the last call (a threshold solve that hit its cap, a bounded wait
 *   that gave up) lives in the array; dash_decode_noalloc_status reads it.
 */
DASH_API int dash_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const float* ksum,
                                 const int* kv_len, void* out, int B, int Hq, int Hkv, int Tmax, int d,
                                 int block, float alpha, float coarse_scale, dash_stream_t stream);

/* Synchronises `stream`, then returns the device status the last dash_decode_noalloc on the
 * current device left in the static scratch array: DASH_OK, DASH_ERR_DEVICE_TIMEOUT,
 * DASH_ERR_NO_CONVERGE (as dash_get_device_status), or DASH_ERR_CUDA. */
DASH_API int dash_decode_noalloc_status(dash_stream_t stream);

/* Synchronises `stream` and returns DASH_OK, DASH_ERR_DEVICE_TIMEOUT when a kernel that used
 * `workspace` gave up a bounded wait, DASH_ERR_NO_CONVERGE when one recorded a failed
 * threshold solve, or DASH_ERR_CUDA. */
DASH_API int dash_get_device_status(const void* workspace, dash_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DASH_ATTN_H */
