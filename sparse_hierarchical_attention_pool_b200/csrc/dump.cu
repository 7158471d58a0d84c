// dump.cu -- block weights of listed rows (Stage 1 only), an independent fp32 recomputation
// for analysis, and the fill kernel of the prefill / decode parity dumps.
//
// select_dump_kernel: x_j accumulated with one fp32 fma chain over the head dimension in
// order against the fp32 summaries, times (alpha - 1) cs / sqrt(d); tau from the
// single-thread solve of entmax.cuh; p_j = (x_j - tau)^(1/(alpha-1)) for x_j > tau.  One CTA
// per listed row.  This is not the prefill's own arithmetic (its scores are tensor-core
// products with the summaries split into bf16 hi + lo parts): the weights the prefill
// applies come from the dump variant of the fine kernel (fine_tc.cu).
#include "common.cuh"
#include "entmax.cuh"
#include "kernels.h"

namespace dash {

struct SmemRow {
    const float* p;
    __device__ __forceinline__ float operator()(int j) const { return p[j]; }
};

template <int D>
__global__ void __launch_bounds__(128)
select_dump_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ ksum,
                   const long long* __restrict__ rows, int max_sel, int* __restrict__ out_idx,
                   float* __restrict__ out_p, int* __restrict__ out_count, float* __restrict__ out_tau,
                   int B, int Hq, int Hkv, int T, float alpha, float cx) {
    extern __shared__ float xsm[];          // [T / 64]
    __shared__ float qs[D];
    const int r = blockIdx.x;
    const long long b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
    const float qnan = __int_as_float(0x7fc00000);
    if (b < 0 || b >= B || h < 0 || h >= Hq || t < 0 || t >= T) {
        if (threadIdx.x == 0) { out_count[r] = 0; out_tau[r] = qnan; }
        return;
    }
    const int G = Hq / Hkv, nbs = T / kBlock;
    const int g = (int)(h / G), bt = (int)(t / kBlock);
    for (int i = threadIdx.x; i < D; i += blockDim.x)
        qs[i] = __bfloat162float(q[((size_t)(b * Hq + h) * T + t) * D + i]);
    __syncthreads();
    const float* kb = ksum + ((size_t)b * Hkv + g) * nbs * D;
    for (int j = threadIdx.x; j < bt; j += blockDim.x) {
        float acc = 0.f;
        for (int kk = 0; kk < D; ++kk) acc = fmaf(qs[kk], kb[(size_t)j * D + kk], acc);
        xsm[j] = acc * cx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (bt == 0) {
            out_count[r] = 0;
            out_tau[r] = qnan;
            return;
        }
        int nc = 0;
        const float tau = entmax_threshold<false>(SmemRow{xsm}, bt, alpha, &nc);
        const float e = 1.0f / (alpha - 1.0f);
        int c = 0;
        for (int j = 0; j < bt; ++j) {
            const float z = xsm[j] - tau;
            if (z > 0.f) {
                if (c < max_sel) {
                    out_idx[(size_t)r * max_sel + c] = j;
                    out_p[(size_t)r * max_sel + c] = e == 2.0f ? z * z : (e == 1.0f ? z : powf(z, e));
                }
                ++c;
            }
        }
        out_count[r] = c;
        out_tau[r] = tau;
    }
}

__global__ void dump_fill_kernel(float* __restrict__ x, float* __restrict__ p, size_t n) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        x[i] = __int_as_float(0x7fc00000);
        p[i] = 0.f;
    }
}

cudaError_t launch_dump_fill(float* x, float* p, size_t n, cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const size_t blocks = (n + 255) / 256;
    dump_fill_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(x, p, n);
    return cudaGetLastError();
}

cudaError_t launch_select_dump(const void* q, const float* ksum, const long long* rows, int nrows,
                               int max_sel, int* out_idx, float* out_p, int* out_count,
                               float* out_tau, int B, int Hq, int Hkv, int T, int d, float alpha,
                               float coarse_scale, cudaStream_t stream) {
    if (nrows == 0) return cudaSuccess;
    const float cx = (alpha - 1.0f) * coarse_scale / sqrtf((float)d);
    const size_t sm = (size_t)(T / kBlock + 1) * sizeof(float);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    if (d == 128) {
        cudaError_t e = cudaFuncSetAttribute(select_dump_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        select_dump_kernel<128><<<nrows, 128, sm, stream>>>(qb, ksum, rows, max_sel, out_idx, out_p, out_count,
                                                            out_tau, B, Hq, Hkv, T, alpha, cx);
    } else {
        cudaError_t e = cudaFuncSetAttribute(select_dump_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        select_dump_kernel<64><<<nrows, 128, sm, stream>>>(qb, ksum, rows, max_sel, out_idx, out_p, out_count,
                                                           out_tau, B, Hq, Hkv, T, alpha, cx);
    }
    return cudaGetLastError();
}

}  // namespace dash
