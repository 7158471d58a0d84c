// entmax.cuh -- alpha-entmax threshold solve on the GPU.
//
// alpha-entmax ("DashAttention: Making Sparse Attention Fully Differentiable with Adaptive
// Block Selection", section "Key Concepts"; "DashAttention and the year sparse attention
// became a field", section "What alpha-entmax changes"):
//     p_j = [x_j - tau]_+^e,  x_j = (alpha - 1) s_j,  e = 1 / (alpha - 1),  sum_j p_j = 1.
//
// Let m = max_j x_j and y_j = x_j - m <= 0.  The shifted threshold u = tau - m lies in
// [-1, 0): p_max <= 1 gives u >= -1, and f(u) = sum_j [y_j - u]_+^e falls from >= 1 at
// u = -1 to 0 at u = 0.  f is continuous and strictly decreasing there, and convex when
// e >= 1 (alpha <= 2), so Newton's method started at u = -1 climbs monotonically to the
// root.  Every pass over the row also gives the support S = {y_j > u} and its power sums;
// for alpha = 2 and alpha = 1.5 the root of sum_S (y_j - u)^e = 1 has a closed form:
//     alpha = 2   : u* = u + (Z1 - 1) / Z0
//     alpha = 1.5 : u* = u + (Z2 - 1) / (Z1 + sqrt(Z1^2 - Z0 (Z2 - 1)))
// with Z_k = sum_S (y_j - u)^k.  When u* stays below every member of S, S is the final
// support and u* is exact; otherwise a Newton step is taken.  Other alpha: safeguarded
// Newton (bisection when a step leaves the bracket) until the step is below 2.5e-7.
//
// The row is read through an accessor x(j), j in [0, n); the solve runs either on one
// thread (STRIDE 1) or on a whole warp (lanes take j = lane, lane + 32, ...; sums are
// reduced with shuffles so every lane returns the same value).
#pragma once

#include "common.cuh"

namespace dash {

template <bool WARP, class Acc>
__device__ float entmax_threshold(const Acc& x, int n, float alpha, int* no_converge) {
    const int j0 = WARP ? (threadIdx.x & 31) : 0;
    const int js = WARP ? 32 : 1;
    float m = -INFINITY;
    for (int j = j0; j < n; j += js) m = fmaxf(m, x(j));
    if (WARP) m = warp_max(m);
    const float e = 1.0f / (alpha - 1.0f);
    const int mode = alpha == 2.0f ? 2 : (alpha == 1.5f ? 1 : 0);
    float lo = -1.0f, hi = 0.0f, u = -1.0f;
    for (int it = 0; it < kSolveMaxIt; ++it) {
        float z0 = 0.f, z1 = 0.f, z2 = 0.f, fe = 0.f, de = 0.f, minz = INFINITY;
        for (int j = j0; j < n; j += js) {
            float z = (x(j) - m) - u;
            if (z > 0.f) {
                z0 += 1.f;
                z1 += z;
                z2 = fmaf(z, z, z2);
                minz = fminf(minz, z);
                if (mode == 0) {
                    float zp = __powf(z, e - 1.0f);
                    de += zp;
                    fe = fmaf(zp, z, fe);
                }
            }
        }
        if (WARP) {
            z0 = warp_sum(z0); z1 = warp_sum(z1); z2 = warp_sum(z2);
            fe = warp_sum(fe); de = warp_sum(de); minz = warp_min(minz);
        }
        if (mode == 2) { fe = z1; de = z0; }
        if (mode == 1) { fe = z2; de = z1; }
        if (fe >= 1.0f) lo = u; else hi = u;
        if (mode != 0 && fe >= 1.0f) {
            float delta = mode == 2
                ? (z1 - 1.0f) / z0
                : (z2 - 1.0f) / (z1 + sqrtf(fmaxf(fmaf(z1, z1, -z0 * (z2 - 1.0f)), 0.0f)));
            if (delta < minz) return m + (u + delta);
        }
        float step = (fe - 1.0f) / (e * de);
        if (fabsf(step) <= 2.5e-7f) return m + (u + step);
        float un = u + step;
        if (!(un > lo && un < hi)) un = 0.5f * (lo + hi);
        u = un;
    }
    *no_converge = 1;
    return m + u;
}

}  // namespace dash
