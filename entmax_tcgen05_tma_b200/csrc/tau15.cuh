// tau15.cuh -- the 1.5-entmax threshold from a row's candidate scores, shared by the forward kernels
// (fwd.cu, fwd_dense.cu).
//
// Page "svd-sst2-roberta-adasplash", sections 2.2-2.3 (Theorem 1: on a fixed support S the
// threshold solves sum_S (S_ij - tau)^2 = 4 in closed form; Theorem 2: bisection on a bracket
// that holds the root) and the model cards' bracket [max - 2, max - 2/sqrt(n)].
#pragma once
#include "common.cuh"

namespace entmax {

// Exact threshold (raw units: sum (v - t)^2 = c4 over the kept values) of the set {a0..a3}
// (a0 >= a1 >= a2 >= a3, missing values -inf), lowered by a rounding margin.  Any subset of a
// row gives a lower bound of the row's tau: adding scores can only raise the threshold.
__device__ __forceinline__ float top4_bound(float a0, float a1, float a2, float a3, float c4) {
    const float z[4] = {a0, a1, a2, a3};
    const float inv[4] = {1.f, 0.5f, 1.f / 3.f, 0.25f};
    float sum = 0.f, sq = 0.f, bound = a0 - sqrtf(c4);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        sum += z[k];
        sq = fmaf(z[k], z[k], sq);
        const float mu = sum * inv[k];
        const float delta = fmaf(c4 - sq, inv[k], mu * mu);
        if (delta >= 0.f) {
            const float tk = mu - sqrtf(delta);
            if (tk <= z[k]) bound = tk;
        }
    }
    return bound - 1e-5f * sqrtf(c4);
}

__device__ __forceinline__ void top4_insert(float v, float& a0, float& a1, float& a2, float& a3) {
    if (v > a3) {
        if (v > a2) {
            a3 = a2;
            if (v > a1) {
                a2 = a1;
                if (v > a0) { a1 = a0; a0 = v; } else { a1 = v; }
            } else {
                a2 = v;
            }
        } else {
            a3 = v;
        }
    }
}


// tau of one row in shifted scaled units (x = scale * S - scale * m, so the row max is 0), from the
// row's candidates (both partitions, partition 0 first) split evenly over a lane pair: lane h holds
// entries h, h + 2, ... (NC registers, -inf where unused).  The lists: float lcv[2][CAPW][TILE],
// entry k of partition p of row r at lcv[(p CAPW + k) TILE + r], n0 entries in partition 0.
// Bisection of [lo, hi], a sub-bracket of [-2, -2/sqrt(n)] that still holds the root (the caller's
// bounds: g(lo) >= 1, g(hi) <= 1; g(-2) >= 1 from the max alone, g(-2/sqrt n) <= 1); every four
// halvings the warp stops if no lane pair has a candidate strictly inside its bracket: the support
// is then fixed and the closed-form root on it is exact.  Returns tau_x.
template <int NC, int CAPW>
__device__ __forceinline__ float solve_tau(const float* lcv, int r, int h, int nh, int n0, float scale, float ms,
                                           float lo, float hi) {
    float x[NC];
#pragma unroll
    for (int k = 0; k < NC; ++k) {
        const int e = 2 * k + h;  // entry e of the row's two lists, partition 0's n0 entries first
        x[k] = k < nh ? fmaf(scale, lcv[(e < n0 ? e : CAPW + (e - n0)) * TILE + r], -ms) : -INFINITY;
    }
    // the candidates as packed pairs: a halving costs a packed subtraction, two maxima and a packed
    // fma per pair
    uint64_t x2[NC / 2];
#pragma unroll
    for (int k = 0; k < NC; k += 2) x2[k >> 1] = f2pack(x[k], x[k + 1]);
    bool settled = false;
    for (int it = 0; it < 25; ++it) {
        const float mid = 0.5f * (lo + hi);
        const uint64_t mid2 = f2pack(mid, mid);
        uint64_t ga = 0, gb = 0;
#pragma unroll
        for (int k = 0; k < NC / 2; k += 2) {
            const uint64_t da = f2relu(f2sub(x2[k], mid2)), db = f2relu(f2sub(x2[k + 1], mid2));
            ga = f2fma(da, da, ga);
            gb = f2fma(db, db, gb);
        }
        float g0, g1, g2, g3;
        f2unpack(ga, g0, g1);
        f2unpack(gb, g2, g3);
        float gs = (g0 + g1) + (g2 + g3);
        gs += __shfl_xor_sync(0xffffffffu, gs, 1);
        if (0.25f * gs > 1.f) lo = mid;
        else hi = mid;
        if ((it & 3) == 3 || it == 24) {
            int und = 0;
#pragma unroll
            for (int k = 0; k < NC; ++k) und += (x[k] > lo && x[k] < hi) ? 1 : 0;
            und += __shfl_xor_sync(0xffffffffu, und, 1);
            settled = und == 0;
            if (__all_sync(0xffffffffu, settled)) break;
        }
    }
    // closed-form root of sum_S (x - tau)^2 = 4 on S = {x > final midpoint}
    const float mid = 0.5f * (lo + hi);
    float K = 0.f, S1 = 0.f, S2 = 0.f;
#pragma unroll
    for (int k = 0; k < NC; ++k) {
        if (x[k] > mid) {
            K += 1.f;
            S1 += x[k];
            S2 = fmaf(x[k], x[k], S2);
        }
    }
    K += __shfl_xor_sync(0xffffffffu, K, 1);
    S1 += __shfl_xor_sync(0xffffffffu, S1, 1);
    S2 += __shfl_xor_sync(0xffffffffu, S2, 1);
    float tau_x = mid;
    if (K > 0.f) {
        const float mu = S1 / K;
        const float var = fmaxf(S2 / K - mu * mu, 0.f);
        const float tc = mu - sqrtf(fmaxf(4.f / K - var, 0.f));
        // with the support settled the root lies in the bracket (clamp only absorbs rounding);
        // otherwise keep it only if it does
        if (settled) tau_x = fminf(fmaxf(tc, lo), hi);
        else if (tc >= lo && tc <= hi) tau_x = tc;
    }
    return tau_x;
}

// Sum of a fixed-point value over the 32 lanes of a warp.
__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// tau of one row whose values x (scaled, shifted so that the row max is 0; -inf where unused) are
// spread over the 32 lanes of a warp, NPL per lane: the same bisection of [lo, hi] with the
// every-four-halvings stop and the closed-form finish as solve_tau, with warp-wide sums.  The sums
// are taken in 64-bit fixed point (2^-40 units; every term lies in [-4, 4] on the bracket, which is
// inside [-2, 0]): integer addition is associative, so the result does not depend on which lane
// holds which value.
template <int NPL>
__device__ __forceinline__ float solve_tau_warp(const float (&x)[NPL], float lo, float hi) {
    constexpr float FX = 1099511627776.f;  // 2^40
    constexpr long long FOUR = 4ll << 40;
    bool settled = false;
    for (int it = 0; it < 25; ++it) {
        const float mid = 0.5f * (lo + hi);
        long long g = 0;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
            const float d = fmaxf(x[k] - mid, 0.f);
            g += __float2ll_rn(d * d * FX);
        }
        g = warp_sum_ll(g);
        if (g > FOUR) lo = mid;
        else hi = mid;
        if ((it & 3) == 3 || it == 24) {
            int und = 0;
#pragma unroll
            for (int k = 0; k < NPL; ++k) und |= (x[k] > lo && x[k] < hi) ? 1 : 0;
            settled = !__any_sync(0xffffffffu, und);
            if (settled) break;
        }
    }
    const float mid = 0.5f * (lo + hi);
    long long K = 0, S1 = 0, S2 = 0;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
        if (x[k] > mid) {
            K += 1;
            S1 += __float2ll_rn(x[k] * FX);
            S2 += __float2ll_rn(x[k] * x[k] * FX);
        }
    }
    K = warp_sum_ll(K);
    S1 = warp_sum_ll(S1);
    S2 = warp_sum_ll(S2);
    float tau_x = mid;
    if (K > 0) {
        const double kd = (double)K, s1 = (double)S1 / (double)FX, s2 = (double)S2 / (double)FX;
        const float mu = (float)(s1 / kd);
        const float var = fmaxf((float)(s2 / kd) - mu * mu, 0.f);
        const float tc = mu - sqrtf(fmaxf(4.f / (float)K - var, 0.f));
        if (settled) tau_x = fminf(fmaxf(tc, lo), hi);
        else if (tc >= lo && tc <= hi) tau_x = tc;
    }
    return tau_x;
}

}  // namespace entmax
