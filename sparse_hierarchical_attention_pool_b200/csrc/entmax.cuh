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
// Any start u0 in [-1, 0) works: from below (f(u0) >= 1) Newton climbs monotonically; from
// above, the first step of a convex decreasing f lands at or below the root.
//
// The iteration is written as a per-pass accumulator (EntmaxPass) and an update
// (EntmaxSolver::update) so that callers can stream a row's values through any memory:
// the single-thread and warp solves below, and the tensor-memory coarse kernel.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dash {

// Power sums of one pass over (part of) a row at the current shifted threshold u.
struct EntmaxPass {
    float z0, z1, z2, fe, de, minz;
    unsigned mb;                                   // add_sat: least bits(z) - 1 over the values
    __device__ __forceinline__ void reset() { z0 = z1 = z2 = fe = de = 0.f; minz = INFINITY; mb = 0xFFFFFFFFu; }
    // Saturating form of add_t for alpha = 1.5 (MODE 1) and alpha = 2 (MODE 2), taking
    // y = x - m <= 0 and u >= -1: z = y - u is at most -u <= 1, so [z]_+ is the saturated
    // difference, one instruction, rounded exactly as y - u.  The count of positive z is
    // sat(sat(z+ 2^127) 2^127), exactly 1 for every positive fp32 (denormals included), and
    // the least positive z comes from an unsigned minimum of bits(z+) - 1, in which z+ = 0
    // wraps to the largest value.  The sums equal add_t's, with fewer compare and select
    // instructions.
    template <int MODE>
    __device__ __forceinline__ void add_sat(float y, float u) {
        static_assert(MODE == 1 || MODE == 2, "closed-form modes only");
        float zp, t, cnt;
        asm("sub.sat.f32 %0, %1, %2;" : "=f"(zp) : "f"(y), "f"(u));
        asm("mul.sat.f32 %0, %1, 0f7F000000;" : "=f"(t) : "f"(zp));
        asm("mul.sat.f32 %0, %1, 0f7F000000;" : "=f"(cnt) : "f"(t));
        z0 += cnt;
        z1 += zp;
        if constexpr (MODE == 1) z2 = fmaf(zp, zp, z2);
        mb = min(mb, __float_as_uint(zp) - 1u);
    }
    // after add_sat: the least positive z into minz
    __device__ __forceinline__ void seal() {
        if (mb != 0xFFFFFFFFu) minz = fminf(minz, __uint_as_float(mb + 1u));
    }
    // z = y - u for one value (mode 0 = general alpha needs the powers)
    __device__ __forceinline__ void add(float z, int mode, float e) {
        if (z > 0.f) {
            z0 += 1.f;
            z1 += z;
            z2 = fmaf(z, z, z2);
            minz = fminf(minz, z);
            if (mode == 0) {
                const float zp = __powf(z, e - 1.0f);
                de += zp;
                fe = fmaf(zp, z, fe);
            }
        }
    }
    // Branch-free form for a solver mode known at compile time (1: alpha = 1.5, 2: alpha = 2,
    // 0: any other alpha), accumulating only the sums that mode's update reads.
    template <int MODE>
    __device__ __forceinline__ void add_t(float z, float e) {
        const bool pos = z > 0.f;
        const float zp = pos ? z : 0.f;
        if constexpr (MODE != 0) {
            z0 += pos ? 1.f : 0.f;
            z1 += zp;
            minz = fminf(minz, pos ? z : INFINITY);
        }
        if constexpr (MODE == 1) z2 = fmaf(zp, zp, z2);
        if constexpr (MODE == 0) {
            const float zq = pos ? __powf(z, e - 1.0f) : 0.f;
            de += zq;
            fe = fmaf(zq, zp, fe);
        }
    }
    template <int MODE>
    __device__ __forceinline__ void warp_reduce_t() {
        if constexpr (MODE != 0) { z0 = warp_sum(z0); z1 = warp_sum(z1); minz = warp_min(minz); }
        if constexpr (MODE == 1) z2 = warp_sum(z2);
        if constexpr (MODE == 0) { fe = warp_sum(fe); de = warp_sum(de); }
    }
    __device__ __forceinline__ void merge(const EntmaxPass& o) {
        z0 += o.z0; z1 += o.z1; z2 += o.z2; fe += o.fe; de += o.de; minz = fminf(minz, o.minz);
    }
    __device__ __forceinline__ void warp_reduce() {
        z0 = warp_sum(z0); z1 = warp_sum(z1); z2 = warp_sum(z2);
        fe = warp_sum(fe); de = warp_sum(de); minz = warp_min(minz);
    }
};

// Pairs of values through add_sat's steps with f32x2 arithmetic for the shift x - m and the
// three sums (f32x2 has no saturating forms: [z]_+ and the count stay scalar).  Each sum is
// kept in two lanes, added in finish(), so its order of additions differs from add_t's.  The
// count takes one saturating multiply, sat(z 2^127), which is exactly 1 for every positive z
// that occurs: the largest weight (-u*)^e is at least 1 / n for n blocks, every iterate stays
// at or below u* / 2 (Newton from below, bisection midpoints), so |u| >= (1/n)^(alpha-1) / 2
// (above 2^-16 for n <= 2^14), and z = y - u > 0 with y in (u, 0] is at least one unit in the
// last place of u, far above 2^-127.
struct EntmaxPassX2 {
    uint64_t s0, s1, s2;                           // (lane a, lane b): count, sum z, sum z^2
    unsigned mb;
    __device__ __forceinline__ void reset() { s0 = s1 = s2 = 0ull; mb = 0xFFFFFFFFu; }
    // x2 = (x_a, x_b), nm2 = (-m, -m)
    template <int MODE>
    __device__ __forceinline__ void add2(uint64_t x2, uint64_t nm2, float u) {
        static_assert(MODE == 1 || MODE == 2, "closed-form modes only");
        using namespace sm100;
        float ya, yb, za, zb, ca, cb;
        f2_unpack(f2_add(x2, nm2), ya, yb);
        asm("sub.sat.f32 %0, %1, %2;" : "=f"(za) : "f"(ya), "f"(u));
        asm("sub.sat.f32 %0, %1, %2;" : "=f"(zb) : "f"(yb), "f"(u));
        asm("mul.sat.f32 %0, %1, 0f7F000000;" : "=f"(ca) : "f"(za));
        asm("mul.sat.f32 %0, %1, 0f7F000000;" : "=f"(cb) : "f"(zb));
        const uint64_t z2 = f2_pack(__float_as_uint(za), __float_as_uint(zb));
        s0 = f2_add(s0, f2_pack(__float_as_uint(ca), __float_as_uint(cb)));
        s1 = f2_add(s1, z2);
        if constexpr (MODE == 1) s2 = f2_fma(z2, z2, s2);
        mb = min(mb, min(__float_as_uint(za) - 1u, __float_as_uint(zb) - 1u));
    }
    __device__ __forceinline__ EntmaxPass finish() const {
        using namespace sm100;
        EntmaxPass p;
        p.reset();
        float a, b;
        f2_unpack(s0, a, b); p.z0 = a + b;
        f2_unpack(s1, a, b); p.z1 = a + b;
        f2_unpack(s2, a, b); p.z2 = a + b;
        p.mb = mb;
        p.seal();
        return p;
    }
};

struct EntmaxSolver {
    float m, u, lo, hi, e;
    int mode, it, maxit;
    __device__ __forceinline__ void init(float row_max, float alpha, float u0 = -1.0f, int cap = kSolveMaxIt) {
        m = row_max;
        u = u0; lo = -1.0f; hi = 0.0f;
        e = 1.0f / (alpha - 1.0f);
        mode = alpha == 2.0f ? 2 : (alpha == 1.5f ? 1 : 0);
        it = 0;
        maxit = cap;
    }
    // One iteration from the pass sums.  Returns true when tau (in x space) is final.
    __device__ __forceinline__ bool update(EntmaxPass p, float* tau, int* no_converge) {
        if (mode == 2) { p.fe = p.z1; p.de = p.z0; }
        if (mode == 1) { p.fe = p.z2; p.de = p.z1; }
        if (p.fe >= 1.0f) lo = u; else hi = u;
        if (mode != 0 && p.fe >= 1.0f) {
            const float delta = mode == 2
                ? (p.z1 - 1.0f) / p.z0
                : (p.z2 - 1.0f) / (p.z1 + sqrtf(fmaxf(fmaf(p.z1, p.z1, -p.z0 * (p.z2 - 1.0f)), 0.0f)));
            if (delta < p.minz) { *tau = m + (u + delta); return true; }
        }
        const float step = (p.fe - 1.0f) / (e * p.de);
        if (fabsf(step) <= 2.5e-7f) { *tau = m + (u + step); return true; }
        float un = u + step;
        if (!(un > lo && un < hi)) un = 0.5f * (lo + hi);
        u = un;
        if (++it >= maxit) { *no_converge = 1; *tau = m + u; return true; }
        return false;
    }
};

// Start from a subset.  For any subset S of the row, sum_S [y - u]_+^e <= f(u), so the root
// u_S of the subset's equation lies at or below the row's root: Newton may start there.  With
// S the row's largest values the start is close (typically one or two passes remain instead
// of the five to ten from u = -1).

// Keep the K largest values seen, in descending order (registers, static indexing).
template <int K>
__device__ __forceinline__ void topk_insert(float (&tk)[K], float v) {
    if (v > tk[K - 1]) {
#pragma unroll
        for (int i = K - 1; i > 0; --i) tk[i] = v > tk[i - 1] ? tk[i - 1] : (v > tk[i] ? v : tk[i]);
        tk[0] = fmaxf(tk[0], v);
    }
}

// Root u_S in shifted units of the subset y(0..N) (values x - m <= 0, -inf ignored; y is an
// accessor), one thread; MODE as in EntmaxPass::add_t.  Returns a start in [-1, 0) at or
// below u_S.
template <int N, int MODE, class Y>
__device__ __forceinline__ float subset_start(const Y& y, float alpha) {
    EntmaxSolver sv;
    sv.init(0.0f, alpha);
    float t = -1.0f;
    int nc = 0;
    for (int it = 0; it < 24; ++it) {
        EntmaxPass ps;
        ps.reset();
#pragma unroll
        for (int i = 0; i < N; ++i) ps.add_t<MODE>(y(i) - sv.u, sv.e);
        if (sv.update(ps, &t, &nc)) return (nc || !(t >= -1.0f)) ? sv.lo : fminf(t, -1e-30f);
    }
    return sv.lo;
}

// Whole-row solve through an accessor x(j), j in [0, n): on one thread (WARP = false) or
// on a whole warp (lanes take j = lane, lane + 32, ...; every lane returns the same value).
template <bool WARP, class Acc>
__device__ float entmax_threshold(const Acc& x, int n, float alpha, int* no_converge, int cap = kSolveMaxIt) {
    const int j0 = WARP ? (threadIdx.x & 31) : 0;
    const int js = WARP ? 32 : 1;
    float m = -INFINITY;
    for (int j = j0; j < n; j += js) m = fmaxf(m, x(j));
    if (WARP) m = warp_max(m);
    EntmaxSolver sv;
    sv.init(m, alpha, -1.0f, cap);
    float tau = m - 1.0f;
    while (true) {
        EntmaxPass ps;
        ps.reset();
        for (int j = j0; j < n; j += js) ps.add((x(j) - m) - sv.u, sv.mode, sv.e);
        if (WARP) ps.warp_reduce();
        if (sv.update(ps, &tau, no_converge)) break;
    }
    return tau;
}

}  // namespace dash
