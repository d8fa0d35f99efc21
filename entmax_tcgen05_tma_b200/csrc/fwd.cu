// fwd.cu -- forward pass of 1.5-entmax attention on sm_100a.
//
// Computes, for every query row i of every (b, h) (page "svd-sst2-roberta-adasplash",
// sections 2.2-2.3 and 3; model cards "roberta-base-adasplash" / "distilbert-sst2-adasplash"):
//   S_ij = scale * Q_i . K_j over the allowed keys (key padding, causal, window),
//   tau_i with sum_j max(0, (S_ij - tau_i)/2)^2 = 1, by bisection on [max-2, max-2/sqrt(n)],
//   O_i = sum_j max(0, (S_ij - tau_i)/2)^2 V_j.
//
// One CTA per 128-query tile.  Phases:
//  1. Score passes (common.cuh pipeline): QK^T on tcgen05, 128 keys per block, fp32 scores in TMEM.
//     Pass A reduces every row to its maximum m_i over the allowed keys and the four largest
//     maxima of its 32-key chunks (branch-free: three-input max trees).  Pass B keeps the row's
//     *candidates*, the scores above m_i - 2 (scaled units) -- the bisection's lower bracket end,
//     so the support is a subset of them -- as (score, key) lists in shared memory.  When the
//     tile's key blocks fit in TMEM at once (at most four blocks: L <= 512, or a causal window)
//     the scores are computed once and read twice ("resident"); otherwise the blocks are streamed
//     twice, the second time recomputing the scores.
//  2. tau per row on the candidate list (two threads per row, candidates in registers): halvings
//     of [m-2, m-2/sqrt(n)] until no candidate is left strictly inside the bracket (at most 25),
//     then the root of sum_S (S_ij - tau)^2 = 4 in closed form on the support S so fixed.
//  3. O_i = sum p_ij V_j over the support with one warp per row: lane l accumulates dimensions
//     2l, 2l+1.  Resident tiles gather V rows from shared memory (TMA-loaded during phase 2);
//     streamed tiles gather them from L2 (prefetched when the candidate was listed).
//  4. Rows with more candidates than a list holds are redone exactly by the whole CTA on CUDA
//     cores (scores into shared memory, bisection with block reductions).
//
// Support extraction (the XT instantiation, for the backward that is given tau alone): pass B alone,
// cut at the given tau_i instead of a lower bound, lists the row's support directly; its entries
// are written as saved supports (phase 2's save step) and nothing else runs: no pass A, no tau
// solve, no O.
#include <cuda_bf16.h>
#include <math.h>
#include "common.cuh"
#include "tau15.cuh"
#include "internal.h"

namespace entmax {
namespace {

using P = Pipe<128, 4, 4, 2>;  // 128-key blocks, 4-deep ring, 4 TMEM buffers, 2 epilogue warpgroups
using PipeCtl = P::Ctl;
constexpr int BLK = P::BLK, NSTAGE = P::NSTAGE, NBUF = P::NBUF;
constexpr int NUM_EPI = P::NUM_EPI;
// Two producer/MMA warp pairs: on a streamed tile pair p feeds epilogue warpgroup p alone (its own
// K-ring stages 2p, 2p + 1 and TMEM buffers p, p + 2), so the warpgroups never wait on each other's
// MMAs; on a resident tile pair 0 feeds both.
constexpr int WARP_PRODUCER = P::WARP_PRODUCER, WARP_MMA = P::WARP_MMA;
constexpr int WARP_PRODUCER2 = WARP_MMA + 1, WARP_MMA2 = WARP_MMA + 2;
constexpr int NUM_THREADS = P::NUM_THREADS + 64, NUM_WARPS = NUM_THREADS / 32;
static_assert(NSTAGE == 4 && NBUF == 4, "two pipelines of two stages and two buffers each");
constexpr int BLK_BYTES = P::BLK_BYTES, TMEM_COLS = P::TMEM_COLS, MAX_BLOCKS = P::MAX_BLOCKS;
constexpr int STAGE_FLOATS = NUM_EPI * 32;  // per-thread staging of one 32-value chunk
static_assert(NSTAGE >= NBUF, "a resident tile's V blocks are staged in the streamed-block ring");

constexpr int CAP = 128;              // candidates per row, split between the two warpgroups
constexpr int CAPW = CAP / 2;

// shared-memory layout (bytes from the 1024-aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + TILE_BYTES;               // K ring; V blocks of a resident tile in phase 3
constexpr int OFF_CV = OFF_B + NSTAGE * BLK_BYTES;      // float [CAP][TILE]
constexpr int OFF_CJ = OFF_CV + CAP * TILE * 4;         // u16   [CAP][TILE]
constexpr int OFF_STAGE = OFF_CJ + CAP * TILE * 2;      // float [NUM_EPI][32]
constexpr int OFF_BITS = OFF_STAGE + STAGE_FLOATS * 4;  // u32   [MASK_WORDS]
constexpr int OFF_BLK = OFF_BITS + MASK_WORDS * 4;      // u16   [MAX_BLOCKS]
constexpr int OFF_VSLOT = OFF_BLK + MAX_BLOCKS * 2;     // u8    [MAX_BLOCKS] ring slot of key block kb's V rows
constexpr int OFF_SUPP = OFF_VSLOT + MAX_BLOCKS;        // int   [2][TILE] support size per partition
constexpr int OFF_ROWS = OFF_SUPP + 2 * TILE * 4;       // RowOut[2][TILE] per-warpgroup row state
constexpr int OFF_RED = OFF_ROWS + 2 * TILE * 32;       // float [NUM_THREADS]
constexpr int OFF_FLAGS = OFF_RED + NUM_THREADS * 4;    // u32   [TILE/32] rows redone by the fallback
constexpr int OFF_VBAR = OFF_FLAGS + 16;                // u64   mbarrier: V blocks landed
constexpr int OFF_CTL = OFF_VBAR + 16;
constexpr int SMEM_USED = OFF_CTL + (int)sizeof(PipeCtl);
constexpr int SMEM_BYTES = SMEM_USED + 1024;
// scratch reused by the fallback after phase 3: one score row
constexpr int OFF_SCRATCH = 0;
constexpr int SCRATCH_BYTES = OFF_CV;
static_assert(MAX_L * 4 <= SCRATCH_BYTES, "fallback score row must fit the score-pass buffers");
static_assert(OFF_SUPP % 16 == 0 && OFF_ROWS % 16 == 0 && OFF_VBAR % 8 == 0, "alignment");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// Per-warpgroup row state: pass-A four largest scores and allowed-key count over the warpgroup's
// keys, pass-B candidate count of its partition and overflow flag.
struct __align__(16) RowOut {
    float a0, a1, a2, a3;
    int nallow;
    int n;
    int ovf;
    int pad_;
};
// General alpha (am1 = alpha - 1, p = max(0, am1 (x - tau))^(1/am1) in scaled units x = scale S):
// lower bound (raw units) of the row's tau from the four largest chunk maxima z0 >= .. >= z3 (scores
// of the row; missing values -inf).  Any subset's threshold is at most the row's.  Start: at
// tau = z_k - k^(-am1)/(am1 scale) each of the k largest adds at least 1/k, so that is a bound for
// every k (wk[k] = (k+1)^(-am1) / (am1 scale)).  Then three Newton steps on the four-score
// constraint g4(t) = sum max(0, u_i - t)^e = 1 (u_i = am1 scale (z_i - z0), e = 1/am1): g4 is
// convex and decreasing (e >= 1), so from a point with g4 >= 1 the Newton iterates rise towards
// the four-score threshold without passing it -- each is still a bound.  Lowered by a rounding
// margin.
__device__ __forceinline__ float gen_bound(float a0, float a1, float a2, float a3, const float (&wk)[4],
                                           float am1, float e, float scale) {
    float b = fmaxf(fmaxf(a0 - wk[0], a1 - wk[1]), fmaxf(a2 - wk[2], a3 - wk[3]));
    const float c = am1 * scale;  // raw -> y units
    const float u[4] = {0.f, c * (a1 - a0), c * (a2 - a0), c * (a3 - a0)};
    float t = c * (b - a0);
#pragma unroll
    for (int step = 0; step < 3; ++step) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float d = u[k] - t;
            const float w = pow_pos(d, e - 1.f);
            s0 += w;
            s1 = fmaf(w, fmaxf(d, 0.f), s1);
        }
        if (s0 > 0.f) t += fmaxf(s1 - 1.f, 0.f) / (e * s0);
    }
    b = fmaxf(b, a0 + t / c);
    return b - 1e-5f * wk[0];
}

// Named barrier over the 8 epilogue warps (id 3; 0 is __syncthreads).
__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync 3, %0;" ::"n"(NUM_EPI) : "memory");
}

// Bounded mbarrier wait whose outcome the whole warp shares (the warp-collective tcgen05 loads
// that follow must be executed by all lanes or none).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int* abort_flag, const WaitCfg& wc) {
    return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, wc));
}

// Maximum of the chunk values whose bit (k) is set in vm (bit k <-> value k), -inf if none.
__device__ __forceinline__ float masked_max(const float (&v)[32], uint32_t vm) {
    float a = -INFINITY, b = -INFINITY, c = -INFINITY, d = -INFINITY;
    if (vm == 0xffffffffu) {
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
            a = fmaxf(a, v[k]);
            b = fmaxf(b, v[k + 1]);
            c = fmaxf(c, v[k + 2]);
            d = fmaxf(d, v[k + 3]);
        }
    } else if (vm != 0u) {
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
            a = fmaxf(a, ((vm >> k) & 1u) ? v[k] : -INFINITY);
            b = fmaxf(b, ((vm >> (k + 1)) & 1u) ? v[k + 1] : -INFINITY);
            c = fmaxf(c, ((vm >> (k + 2)) & 1u) ? v[k + 2] : -INFINITY);
            d = fmaxf(d, ((vm >> (k + 3)) & 1u) ? v[k + 3] : -INFINITY);
        }
    }
    return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// v[q] for a thread-dependent q in [0, 32): a tree of selects on the bits of q, 16 + 8 + 4 + 2 + 1 of them
// (no indexed register access, no shared memory).
__device__ __forceinline__ float pick32(const float (&v)[32], int q) {
    float a[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) a[k] = (q & 16) ? v[16 + k] : v[k];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = (q & 8) ? a[8 + k] : a[k];
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = (q & 4) ? a[4 + k] : a[k];
#pragma unroll
    for (int k = 0; k < 2; ++k) a[k] = (q & 2) ? a[2 + k] : a[k];
    return (q & 1) ? a[1] : a[0];
}

// Reads chunks 2 half and 2 half + 1 of the (resident) score buffer of block n and calls f(v, c).
template <class F>
__device__ __forceinline__ void for_half_block(const PipeCtl* ctl, int n, int half, F&& f) {
    float va[32], vb[32];
    tmem_ld32(P::taddr(ctl, n, 2 * half), va);
    tmem_ld32(P::taddr(ctl, n, 2 * half + 1), vb);
    tmem_wait_ld(va);
    tmem_wait_ld(vb);
    f(va, 2 * half);
    f(vb, 2 * half + 1);
}

// General alpha: tau of one row in units y = am1 (scale S - ms) (row max 0, every p term is
// (y - t)^e with e = 1/am1), candidates split over a lane pair as in solve_tau.  First Newton's
// method from lo over all candidates (below); rows of a warp that it has not settled go on with: bisection of
// [lo, hi] (g(lo) >= 1 >= g(hi)) with the same every-four-halvings stop once no candidate lies
// strictly inside the bracket and g(lo) <= 1.5; then Newton's method on the support
// S = {y > midpoint} so fixed, started at lo: on S, phi(t) = sum (y - t)^e - 1 is convex and
// decreasing with phi(lo) >= 0, so the iterates rise monotonically to the root without passing it
// (one step is exact when e = 1).  Far from the root a large e makes Newton crawl (each step
// closes about 1/e of the gap), hence the g(lo) <= 1.5 condition: from there six steps reach fp32
// precision for e up to 20.  Not settled after 25 halvings: the final midpoint.  Returns t in y
// units.
template <int NC>
__device__ __forceinline__ float solve_tau_gen(const float* lcv, int r, int h, int nh, int n0, float scale, float ms,
                                               float am1, float e, float lo, float hi) {
    float y[NC];
#pragma unroll
    for (int k = 0; k < NC; ++k) {
        const int en = 2 * k + h;
        y[k] = k < nh ? am1 * fmaf(scale, lcv[(en < n0 ? en : CAPW + (en - n0)) * TILE + r], -ms) : -INFINITY;
    }
    // Newton's method from lo on all candidates: g is convex and decreasing (e >= 1), g(lo) >= 1, so
    // the iterates rise monotonically to the root; stop when every row of the warp moved by less
    // than 2e-7 (y units).  Rows that have not by then continue with the bisection below from the
    // raised lower end.
    bool conv = false;
    {
        const float em1 = e - 1.f;
#pragma unroll 1
        for (int step = 0; step < 8; ++step) {
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int k = 0; k < NC; ++k) {
                const float d = y[k] - lo;
                const float w = pow_pos(d, em1);
                s0 += w;
                s1 = fmaf(w, fmaxf(d, 0.f), s1);
            }
            s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
            const float dt = s0 > 0.f ? fmaxf(s1 - 1.f, 0.f) / (e * s0) : 0.f;
            lo = fminf(lo + dt, hi);
            conv = dt <= 2e-7f;
            if (__all_sync(0xffffffffu, conv)) break;
        }
        if (__all_sync(0xffffffffu, conv)) return lo;
    }
    bool settled = false;
    float glo = conv ? 1.f : INFINITY;  // g(lo), once known (a converged Newton lo is at the root)
    for (int it = 0; it < 25; ++it) {
        const float mid = 0.5f * (lo + hi);
        float g0 = 0.f, g1 = 0.f, g2 = 0.f, g3 = 0.f;
#pragma unroll
        for (int k = 0; k < NC; k += 4) {
            g0 += pow_pos(y[k] - mid, e);
            g1 += pow_pos(y[k + 1] - mid, e);
            g2 += pow_pos(y[k + 2] - mid, e);
            g3 += pow_pos(y[k + 3] - mid, e);
        }
        float gs = (g0 + g1) + (g2 + g3);
        gs += __shfl_xor_sync(0xffffffffu, gs, 1);
        if (gs > 1.f) {
            lo = mid;
            glo = gs;
        } else {
            hi = mid;
        }
        if ((it & 3) == 3 || it == 24) {
            int und = 0;
#pragma unroll
            for (int k = 0; k < NC; ++k) und += (y[k] > lo && y[k] < hi) ? 1 : 0;
            und += __shfl_xor_sync(0xffffffffu, und, 1);
            settled = und == 0 && glo <= 1.5f;
            if (__all_sync(0xffffffffu, settled)) break;
        }
    }
    const float mid = 0.5f * (lo + hi);
    float t = lo;
    const float em1 = e - 1.f;
#pragma unroll 1
    for (int step = 0; step < 6; ++step) {
        float s0 = 0.f, s1 = 0.f;  // sum over S of (y - t)^(e-1) and of (y - t)^e
#pragma unroll
        for (int k = 0; k < NC; ++k) {
            if (y[k] > mid) {
                const float b = y[k] - t;
                const float w = pow_pos(b, em1);
                s0 += w;
                s1 = fmaf(w, b, s1);
            }
        }
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        if (s0 > 0.f) t += (s1 - 1.f) / (e * s0);
    }
    return settled ? fminf(fmaxf(t, lo), hi) : mid;
}

__device__ __forceinline__ void fma_bf16x8(float (&acc)[8], float w, const uint4& x) {
    const uint32_t u[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        acc[2 * k] = fmaf(w, bf16lo(u[k]), acc[2 * k]);
        acc[2 * k + 1] = fmaf(w, bf16hi(u[k]), acc[2 * k + 1]);
    }
}

// Writes row r's support (both partitions, h_ij = sqrt(p_ij) in cv; b_ij for general alpha) to the saved lists as
// (j, b_ij), b_ij = am1 (S_ij - tau_i) scaled (= sqrt(p_ij) at alpha 1.5), and
// counts each key once per row that holds it.  Run by the row's two threads (h = 0, 1) after phase 2;
// rows redone on CUDA cores (mode 2) or with more than SAVE_CAP entries are marked unsaved.
template <bool GEN>
__device__ __forceinline__ void save_row_support(const SavedSupport& sv, const float* cv, const uint16_t* cj,
                                                 const int* supp_cnt, int r, int h, int mode, size_t head_row0,
                                                 size_t key_row0, int i, int L) {
    const int s0 = supp_cnt[r], s1 = supp_cnt[TILE + r];
    const bool saved = mode != 2 && s0 + s1 <= SAVE_CAP;
    if (i >= L) return;
    const size_t row = head_row0 + i;
    if (!saved) {
        if (h == 0) {
            sv.row_cnt[row] = -1;
            sv.unsaved_rows[atomicAdd(sv.unsaved_cnt, 1)] = (int)row;
        }
        return;
    }
    if (h == 0) sv.row_cnt[row] = s0 + s1;
    const int n = h == 0 ? s0 : s1, base = h == 0 ? 0 : s0;
    const int slot0 = h * CAPW;
    for (int e = 0; e < n; ++e) {
        const int j = cj[(slot0 + e) * TILE + r];
        sv.row_j[row * SAVE_CAP + base + e] = (uint16_t)j;
        // h = sqrt(p) (alpha 1.5) or b = am1 (x - tau) (generic): saved as is
        sv.row_sp[row * SAVE_CAP + base + e] = cv[(slot0 + e) * TILE + r];
        atomicAdd(sv.key_cnt + key_row0 + j, 1);
    }
}

// Block-wide sum of two floats (all NUM_THREADS threads call it).  red: >= 64 floats.
__device__ __forceinline__ float2 block_sum2(float a, float b, float* red) {
    a = warp_sum(a);
    b = warp_sum(b);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) {
        red[warp] = a;
        red[16 + warp] = b;
    }
    __syncthreads();
    float sa = 0.f, sb = 0.f;
#pragma unroll
    for (int w = 0; w < NUM_WARPS; ++w) {
        sa += red[w];
        sb += red[16 + w];
    }
    return make_float2(sa, sb);
}

__device__ __forceinline__ float block_max(float a, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[32 + warp] = a;
    __syncthreads();
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < NUM_WARPS; ++w) m = fmaxf(m, red[32 + w]);
    return m;
}

// Phase 4: the whole CTA recomputes one row exactly on CUDA cores.  alpha 1.5: bisection of
// [m - 2, m - 2/sqrt(n)] and the closed-form root once the support is fixed.  General alpha
// (GEN, am1 = alpha - 1): the same in units y = am1 (s - m), bracket [-1, -n^(-am1)], and Newton's
// method from the lower end on the fixed support once also g(lower end) <= 1.5 (as in
// solve_tau_gen).
template <bool GEN>
__device__ __noinline__ void fallback_row(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                                          const __nv_bfloat16* __restrict__ V, const uint32_t* bits, float* sbuf,
                                          float* red, HeadRef hq, HeadRef hkv, int bh, int i, int L,
                                          int causal, int window, float scale, float am1, int nallow, void* O,
                                          int out_f32, float* tau, float* otil, float* rsum) {
    const int tid = threadIdx.x;
    float* qf = red + 64;  // 64 floats (red[0..63] holds reduction partials)
    __syncthreads();
    if (tid < HEAD_DIM) qf[tid] = __bfloat162float(Q[hq.row(i) * HEAD_DIM + tid]);
    __syncthreads();
    int lo, hi;
    row_key_range(i, L, causal, window, lo, hi);
    const int span = hi - lo + 1;
    float mloc = -INFINITY;
    for (int e = tid; e < span; e += NUM_THREADS) {
        const int j = lo + e;
        float s = -INFINITY;
        if ((bits[j >> 5] >> (j & 31)) & 1u) {
            const uint4* kr = reinterpret_cast<const uint4*>(K + hkv.row(j) * HEAD_DIM);
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w = kr[c];
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    acc = fmaf(qf[c * 8 + 2 * t], bf16lo(ws[t]), acc);
                    acc = fmaf(qf[c * 8 + 2 * t + 1], bf16hi(ws[t]), acc);
                }
            }
            s = scale * acc;
        }
        sbuf[e] = s;
        mloc = fmaxf(mloc, s);
    }
    const float m = block_max(mloc, red);
    const float ex = 1.f / am1;
    // alpha 1.5 works on the scores s, general alpha on y = am1 (s - m)
    auto unit = [&](float s) { return GEN ? am1 * (s - m) : s; };
    float blo = GEN ? -1.f : m - 2.f;
    float bhi = GEN ? -pow_pos((float)nallow, -am1) : m - 2.f / sqrtf((float)nallow);
    // Newton's method from blo (g(blo) >= 1; g convex and decreasing, so the iterates rise to the
    // root without passing it), at most eight steps; converged: the support is {y > blo} up to
    // scores within 1e-6 of the root.  Otherwise the bisection below continues from the raised blo.
    bool conv = false;
    for (int step = 0; step < 8 && !conv; ++step) {
        float s0 = 0.f, s1 = 0.f;  // GEN: sum (y-t)^(e-1), sum (y-t)^e; 1.5: sum (s-t), sum (s-t)^2
        for (int e = tid; e < span; e += NUM_THREADS) {
            const float d = unit(sbuf[e]) - blo;
            if (d > 0.f) {
                const float w = GEN ? pow_pos(d, ex - 1.f) : d;
                s0 += w;
                s1 = fmaf(w, d, s1);
            }
        }
        const float2 sums = block_sum2(s0, s1, red);  // uniform across the CTA
        const float g = GEN ? sums.y : 0.25f * sums.y;
        const float dg = GEN ? ex * sums.x : 0.5f * sums.x;
        const float dt = dg > 0.f ? fmaxf(g - 1.f, 0.f) / dg : 0.f;
        blo = fminf(blo + dt, bhi);
        conv = dt <= 1e-6f;
    }
    bool resolved = false;
    float glo = conv ? 1.f : INFINITY;  // g(blo) once known (general alpha: Newton needs g(blo) <= 1.5)
    for (int it = 0; it < (conv ? 0 : 25); ++it) {
        const float mid = 0.5f * (blo + bhi);
        float gl = 0.f, inside = 0.f;
        for (int e = tid; e < span; e += NUM_THREADS) {
            const float s = unit(sbuf[e]);
            if (s > mid) {
                if (GEN) {
                    gl += pow_pos(s - mid, ex);
                } else {
                    const float d = 0.5f * (s - mid);
                    gl = fmaf(d, d, gl);
                }
            }
            if (s > blo && s < bhi) inside += 1.f;
        }
        const float2 r2 = block_sum2(gl, inside, red);
        if (r2.y == 0.f && (!GEN || glo <= 1.5f)) {
            resolved = true;
            break;
        }
        if (r2.x > 1.f) {
            blo = mid;
            glo = r2.x;
        } else {
            bhi = mid;
        }
    }
    float t;
    if (conv) {
        resolved = true;  // Newton converged: the support is {scores >= blo}
    } else if (!resolved) {
        // one more count: the last halving may have emptied the bracket
        float inside = 0.f;
        for (int e = tid; e < span; e += NUM_THREADS) {
            const float s = unit(sbuf[e]);
            if (s > blo && s < bhi) inside += 1.f;
        }
        resolved = block_sum2(inside, 0.f, red).x == 0.f && (!GEN || glo <= 1.5f);
    }
    // support of the finish: the scores at or above the bracket's upper end once none lies inside
    // the bracket, or at or above blo after a converged Newton phase
    const float cut = conv ? blo : bhi;
    if (GEN) {
        // Newton's method on the fixed support {y >= bhi}, from blo (monotone, see solve_tau_gen)
        float tt = blo;
        if (conv) {
            t = blo;
        } else if (resolved) {
            for (int step = 0; step < 6; ++step) {
                float s0 = 0.f, s1 = 0.f;
                for (int e = tid; e < span; e += NUM_THREADS) {
                    const float y = unit(sbuf[e]);
                    if (y >= bhi) {
                        const float b = y - tt;
                        const float w = pow_pos(b, ex - 1.f);
                        s0 += w;
                        s1 = fmaf(w, b, s1);
                    }
                }
                const float2 sums = block_sum2(s0, s1, red);
                if (sums.x > 0.f) tt += (sums.y - 1.f) / (ex * sums.x);
            }
            t = fminf(fmaxf(tt, blo), bhi);
        } else {
            t = 0.5f * (blo + bhi);
        }
    } else if (resolved) {
        float k = 0.f, s1 = 0.f, s2 = 0.f;
        for (int e = tid; e < span; e += NUM_THREADS) {
            const float s = sbuf[e];
            if (s >= cut) {
                const float x = s - m;
                k += 1.f;
                s1 += x;
                s2 = fmaf(x, x, s2);
            }
        }
        const float2 a = block_sum2(k, s1, red);
        const float2 b2 = block_sum2(s2, 0.f, red);
        const float mu = a.y / a.x;
        const float var = fmaxf(b2.x / a.x - mu * mu, 0.f);
        t = m + mu - sqrtf(fmaxf(4.f / a.x - var, 0.f));
        t = fminf(fmaxf(t, blo), bhi);
    } else {
        t = 0.5f * (blo + bhi);
    }
    // O_i (and, alpha 1.5 with otil, Otil_i = sum h_ij V_j and r_i = sum h_ij): thread -> (dimension d,
    // key phase ph)
    constexpr int PH = NUM_THREADS / HEAD_DIM;
    const int d = tid % HEAD_DIM, ph = tid / HEAD_DIM;
    const bool aux = !GEN && otil != nullptr;
    float acc = 0.f, acc2 = 0.f, hsum = 0.f;
    for (int e = ph; e < span; e += PH) {
        const float s = unit(sbuf[e]);
        if (s > t) {
            float p, hv = 0.f;
            if (GEN) {
                p = pow_pos(s - t, ex);
            } else {
                hv = 0.5f * (s - t);
                p = hv * hv;
            }
            const float v = __bfloat162float(V[hkv.row(lo + e) * HEAD_DIM + d]);
            acc = fmaf(p, v, acc);
            acc2 = fmaf(hv, v, acc2);
            hsum += hv;
        }
    }
    __syncthreads();
    red[tid] = acc;
    __syncthreads();
    if (tid < HEAD_DIM) {
        float o = 0.f;
#pragma unroll
        for (int p = 0; p < PH; ++p) o += red[tid + p * HEAD_DIM];
        const size_t oi = hq.row(i) * HEAD_DIM + tid;
        if (out_f32) reinterpret_cast<float*>(O)[oi] = o;
        else reinterpret_cast<__nv_bfloat16*>(O)[oi] = __float2bfloat16_rn(o);
        if (tid == 0) tau[(size_t)bh * L + i] = GEN ? m + t * ex : t;
    }
    if (aux) {  // uniform across the CTA
        __syncthreads();
        red[tid] = acc2;
        __syncthreads();
        if (tid < HEAD_DIM) {
            float o = 0.f;
#pragma unroll
            for (int p = 0; p < PH; ++p) o += red[tid + p * HEAD_DIM];
            otil[((size_t)bh * L + i) * HEAD_DIM + tid] = o;
        }
        // every (dimension, phase) thread summed h over its phase's keys: the d = 0 threads hold r_i
        __syncthreads();
        red[tid] = d == 0 ? hsum : 0.f;
        __syncthreads();
        if (tid == 0) {
            float rs = 0.f;
#pragma unroll
            for (int p = 0; p < PH; ++p) rs += red[p * HEAD_DIM];
            rsum[(size_t)bh * L + i] = rs;
        }
    }
    __syncthreads();
}

// Streamed tile, pipeline p: local job m loads and multiplies listed block half_block(p, m) -- first
// the pass-A blocks 2k (k < nA, k = p mod 2), then the pass-B blocks k = p mod 2 -- through K-ring
// stage 2p + (m & 1) into TMEM buffer p + 2 (m & 1); both alternate, so their completion parity is
// (m >> 1) & 1.
__device__ __forceinline__ int half_block(int p, int m, int mA) { return m < mA ? 2 * (p + 2 * m) : p + 2 * (m - mA); }

__device__ __noinline__ void produce_half(PipeCtl* ctl, const WaitCfg& wc, const CUtensorMap* map_a,
                                          const CUtensorMap* map_b, HeadRef ha, HeadRef hb, int a_row0,
                                          const uint16_t* blk_list, uint8_t* smem_a, uint8_t* smem_b, int p, int mA,
                                          int mB) {
    if (p == 0) {
        mbar_arrive_expect_tx(smem_u32(&ctl->full_a), TILE_BYTES);
        tma_load_3d(smem_u32(smem_a), map_a, 0, ha.c1(a_row0), ha.c2(a_row0), smem_u32(&ctl->full_a));
    }
    int issued = 0;
    for (int m = 0; m < mA + mB; ++m) {
        const int st = 2 * p + (m & 1);
        const uint32_t ph = (uint32_t)(m >> 1) & 1u;
        if (!wait_bounded(smem_u32(&ctl->empty_b[st]), ph ^ 1u, &ctl->abort_flag, wc)) break;
        mbar_arrive_expect_tx(smem_u32(&ctl->full_b[st]), BLK_BYTES);
        const int row = (int)(blk_list[half_block(p, m, mA)] & ~FULL_BLOCK) * BLK;
        tma_load_3d(smem_u32(smem_b + st * BLK_BYTES), map_b, 0, hb.c1(row), hb.c2(row), smem_u32(&ctl->full_b[st]));
        ++issued;
    }
    ctl->nload[p] = issued;  // drained at teardown if the CTA aborts (drain_half)
}

// Teardown after an abort (past the CTA's teardown barrier), streamed tile, pipeline p: the producer
// thread waits for the A tile (pipeline 0) and its last two K loads; the MMA thread for its last
// commit, which covers every MMA it issued.
__device__ __noinline__ void drain_half(PipeCtl* ctl, int p, bool mma_thread) {
    if (mma_thread) {
        const int m = ctl->nmma[p] - 1;
        if (m >= 0) wait_drain(smem_u32(&ctl->s_full[p + 2 * (m & 1)]), (uint32_t)(m >> 1) & 1u);
        return;
    }
    if (p == 0) wait_drain(smem_u32(&ctl->full_a), 0);
    const int n = ctl->nload[p];
    for (int m = max(0, n - 2); m < n; ++m)
        wait_drain(smem_u32(&ctl->full_b[2 * p + (m & 1)]), (uint32_t)(m >> 1) & 1u);
}

__device__ __noinline__ void mma_half(PipeCtl* ctl, const WaitCfg& wc, const uint8_t* smem_a, const uint8_t* smem_b,
                                      int p, int njobs) {
    constexpr uint32_t idesc = umma_idesc_bf16_f32(TILE, BLK);
    int issued = 0;
    if (wait_bounded(smem_u32(&ctl->full_a), 0, &ctl->abort_flag, wc)) {
        tc_fence_after();
        const uint64_t da = umma_desc_kmajor_sw128(smem_u32(smem_a));
        for (int m = 0; m < njobs; ++m) {
            const int st = 2 * p + (m & 1), buf = p + 2 * (m & 1);
            const uint32_t ph = (uint32_t)(m >> 1) & 1u;
            if (!wait_bounded(smem_u32(&ctl->full_b[st]), ph, &ctl->abort_flag, wc)) break;
            if (!wait_bounded(smem_u32(&ctl->s_empty[buf]), ph ^ 1u, &ctl->abort_flag, wc)) break;
            tc_fence_after();
            const uint64_t db = umma_desc_kmajor_sw128(smem_u32(smem_b + st * BLK_BYTES));
            const uint32_t d_tmem = ctl->tmem_base + (uint32_t)(buf * BLK);
#pragma unroll
            for (int k = 0; k < HEAD_DIM / 16; ++k)  // 16 bf16 = 32 B = 2 descriptor units per step
                tc_mma_bf16(d_tmem, da + 2u * k, db + 2u * k, idesc, k > 0 ? 1u : 0u);
            tc_commit(smem_u32(&ctl->empty_b[st]));
            tc_commit(smem_u32(&ctl->s_full[buf]));
            ++issued;
        }
    }
    ctl->nmma[p] = issued;  // drained at teardown if the CTA aborts (drain_half)
}

template <bool GEN, bool XT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
entmax_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, const AttnArgs args, const FwdOut out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smem_a = smem + OFF_A;
    uint8_t* smem_b = smem + OFF_B;
    float* cv = reinterpret_cast<float*>(smem + OFF_CV);
    uint16_t* cj = reinterpret_cast<uint16_t*>(smem + OFF_CJ);
    float* stage = reinterpret_cast<float*>(smem + OFF_STAGE);
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + OFF_BITS);
    uint16_t* blk_list = reinterpret_cast<uint16_t*>(smem + OFF_BLK);
    uint8_t* vslot = smem + OFF_VSLOT;
    int* supp_cnt = reinterpret_cast<int*>(smem + OFF_SUPP);
    RowOut* rows = reinterpret_cast<RowOut*>(smem + OFF_ROWS);
    float* red = reinterpret_cast<float*>(smem + OFF_RED);
    uint32_t* redo = reinterpret_cast<uint32_t*>(smem + OFF_FLAGS);
    uint64_t* vbar = reinterpret_cast<uint64_t*>(smem + OFF_VBAR);
    float* scratch = reinterpret_cast<float*>(smem + OFF_SCRATCH);
    PipeCtl* ctl = reinterpret_cast<PipeCtl*>(smem + OFF_CTL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = args.L;
    const int tile = blockIdx.x, bh = blockIdx.y;
    const int b = bh / args.H;
    const int bhk = kv_head_of(bh, args.H, args.Hkv);  // K/V head (b * Hkv + index)
    const HeadRef hq{args.layout, b, bh - b * args.H, args.H, L};          // rows of Q and O
    const HeadRef hkv{args.layout, b, bhk - b * args.Hkv, args.Hkv, L};    // rows of K and V
    const int i0 = tile * TILE;
    const WaitCfg wc{args.status, args.timeout_ns};
    // V row j of this head at Vh + j * vstep
    const __nv_bfloat16* Vh = reinterpret_cast<const __nv_bfloat16*>(args.V) + hkv.row(0) * HEAD_DIM;
    const size_t vstep = hkv.step() * HEAD_DIM;

    if (tid == 0) {
        mbar_init(smem_u32(vbar), 1);
        P::init(ctl);  // ends with the barrier-init fence
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
    }
    if (tid < TILE / 32) redo[tid] = 0u;
    if (warp == WARP_PRODUCER) {
        tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    build_key_bitmap(bits, args.key_mask, b, L);
    __syncthreads();
    if (warp == 0) {
        // key blocks that hold at least one key some row of this tile may attend to
        const int i_last = min(i0 + TILE - 1, L - 1);
        const int klo = args.window > 0 ? max(0, i0 - args.window + 1) : 0;
        const int khi = args.causal ? i_last : L - 1;
        const int nb = P::build_block_list(blk_list, bits, klo, khi, i0, i_last, args.causal, args.window);
        __syncwarp();
        if (nb <= NBUF && lane < nb) vslot[blk_list[lane] & ~FULL_BLOCK] = (uint8_t)lane;
        if (lane == 0) ctl->nblk = nb;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const float scale = args.scale;
    const float two_over_scale = 2.f / scale;
    const float c4 = 4.f / (scale * scale);
    // general alpha: am1 = alpha - 1, p = (y - t)^ex with y = am1 (scaled score - row max);
    // wk[k] = (k+1)^(-am1) / (am1 scale), the lower-bound offsets of gen_bound
    const float am1 = args.am1, ex = 1.f / am1;
    float wk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) wk[k] = GEN ? exp2f(-am1 * log2f((float)(k + 1))) / (am1 * scale) : 0.f;
    const int nblk = ctl->nblk;
    const bool resident = nblk <= NBUF;
    // Streamed tiles run pass A on every other listed block only (any subset of a row bounds tau
    // from below); pass B visits them all.  Extraction runs pass B alone.
    const int nA = XT ? 0 : resident ? nblk : (nblk + 1) / 2;
    const int njobs = resident ? nblk : nA + nblk;

    // per-warpgroup job counts of a streamed tile: pass-A blocks 2k (k < nA, k = g mod 2), then
    // pass-B blocks k = g mod 2
    const int mA0 = (nA + 1) >> 1, mA1 = nA >> 1, mB0 = (nblk + 1) >> 1, mB1 = nblk >> 1;
    if (warp == WARP_PRODUCER || warp == WARP_PRODUCER2) {
        const int p = warp == WARP_PRODUCER ? 0 : 1;
        if (lane == 0) {
            if (resident) {
                if (p == 0) P::producer(ctl, wc, &map_q, &map_k, hq, i0, blk_list, smem_a, smem_b, njobs, hkv);
            } else {
                produce_half(ctl, wc, &map_q, &map_k, hq, hkv, i0, blk_list, smem_a, smem_b, p, p ? mA1 : mA0, p ? mB1 : mB0);
            }
        }
        __syncwarp();
    } else if (warp == WARP_MMA || warp == WARP_MMA2) {
        const int p = warp == WARP_MMA ? 0 : 1;
        if (lane == 0) {
            if (resident) {
                if (p == 0) P::mma(ctl, wc, smem_a, smem_b, njobs);
            } else {
                mma_half(ctl, wc, smem_a, smem_b, p, p ? mA1 + mB1 : mA0 + mB0);
            }
        }
        __syncwarp();
    } else {
        // thread (g, r): query row i0 + r; warpgroup g takes half g of every block (resident) or
        // every other block (streamed)
        const int r = tid & (TILE - 1), g = tid >> 7;
        const int i = i0 + r;
        int rlo, rhi;
        row_key_range(i, L, args.causal, args.window, rlo, rhi);
        auto allowed = [&](int n, int jc) -> uint32_t {
            const bool full = (blk_list[n] & FULL_BLOCK) && i < L;
            return full ? 0xffffffffu : (jc < L && i < L) ? (bits[jc >> 5] & range_bits(jc, rlo, rhi)) : 0u;
        };
        bool live = true;

        // ---------------- pass A: the four largest 32-key chunk maxima (of every block, or of every
        // other block on a streamed tile).  Branch-free: a chunk costs a tree of three-input maxima
        // and a min/max insertion network.  The chunk maxima are scores of the row, so the exact
        // threshold of the four largest is a lower bound of tau (a subset's threshold never exceeds
        // the row's).
        float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
        int nallow = 0;
        const int slot = threadIdx.x % NUM_EPI;
        auto pass_a = [&](int n) {
            const int j0 = (int)(blk_list[n] & ~FULL_BLOCK) * BLK;
            return [&, n, j0](const float (&cur)[32], int c) {
                const uint32_t vm = allowed(n, j0 + c * 32);
                const float cm = vm == 0xffffffffu ? max32(cur) : masked_max(cur, vm);
                a3 = fmaxf(a3, fminf(a2, cm));
                a2 = fmaxf(a2, fminf(a1, cm));
                a1 = fmaxf(a1, fminf(a0, cm));
                a0 = fmaxf(a0, cm);
            };
        };
        if (XT) {
        } else if (resident) {
            for (int n = 0; n < nblk; ++n) {
                if (live) live = warp_wait(smem_u32(&ctl->s_full[n]), 0u, &ctl->abort_flag, wc);
                tc_fence_after();
                if (live) for_half_block(ctl, n, g, pass_a(n));
            }
        } else {
            // this warpgroup's pipeline: local job m in TMEM buffer g + 2 (m & 1), parity (m >> 1) & 1
            const int mA = g ? mA1 : mA0;
            for (int m = 0; m < mA; ++m) {
                const int buf = g + 2 * (m & 1);
                if (live) live = warp_wait(smem_u32(&ctl->s_full[buf]), (uint32_t)(m >> 1) & 1u, &ctl->abort_flag, wc);
                tc_fence_after();
                if (live) P::for_each_chunk(ctl, buf, pass_a(half_block(g, m, mA)));
            }
        }
        if (!XT) {
            {
                RowOut& mine = rows[g * TILE + r];
                mine.a0 = a0;
                mine.a1 = a1;
                mine.a2 = a2;
                mine.a3 = a3;
            }
            epi_sync();
            const RowOut& other = rows[(g ^ 1) * TILE + r];
            top4_insert(other.a0, a0, a1, a2, a3);
            top4_insert(other.a1, a0, a1, a2, a3);
            top4_insert(other.a2, a0, a1, a2, a3);
            top4_insert(other.a3, a0, a1, a2, a3);
        }
        // scores at or below t are outside the support: the largest chunk maximum seen minus 2
        // (scaled), raised to the exact threshold of the four largest chunk maxima seen (any
        // subset's threshold is at most tau).  Extraction: the given tau_i over the scale, lowered
        // by 2^-20 of itself so that no raw score whose scaled value exceeds tau_i is cut (the
        // exact test S_ij > tau_i follows on the listed candidates); an infinite tau_i (a row with
        // no allowed key) cuts everything.
        float t;
        if (XT) {
            t = i < L ? out.tau[(size_t)bh * L + i] / scale : INFINITY;
            if (isfinite(t)) t -= fabsf(t) * 0x1p-20f;
        } else {
            t = GEN ? gen_bound(a0, a1, a2, a3, wk, am1, ex, scale)
                    : fmaxf(a0 - two_over_scale, top4_bound(a0, a1, a2, a3, c4));
        }

        // ---------------- pass B: candidates s > m - 2 (scaled) into this warpgroup's partition
        float* pcv = cv + g * CAPW * TILE;
        uint16_t* pcj = cj + g * CAPW * TILE;
        int nc = 0;
        auto pass_b = [&](int e) {
            const uint16_t ent = blk_list[e];
            const int j0 = (int)(ent & ~FULL_BLOCK) * BLK;
            const bool full = (ent & FULL_BLOCK) && i < L;
            return [&, j0, full](const float (&cur)[32], int c) {
                const int jc = j0 + c * 32;
                const uint32_t vm = full ? 0xffffffffu
                                         : (jc < L && i < L) ? (bits[jc >> 5] & range_bits(jc, rlo, rhi)) : 0u;
                if (!XT) nallow += __popc(vm);  // extraction: a row with no allowed key has no hit
                uint32_t hits = hit_bits(cur, t) & __brev(vm);
                if (XT) {
                    // the support is sparse (about one hit per chunk that has one): each hit's score
                    // is picked from registers, with no staging of the chunk through shared memory
                    while (hits) {
                        const int q = __clz(hits);
                        hits &= ~(0x80000000u >> q);
                        if (nc < CAPW) {
                            pcv[nc * TILE + r] = pick32(cur, q);
                            pcj[nc * TILE + r] = (uint16_t)(jc + q);
                        }
                        ++nc;
                    }
                } else if (hits) {
                    stage_chunk(stage, slot, cur);
                    do {
                        const int q = __clz(hits);
                        hits &= ~(0x80000000u >> q);
                        if (nc < CAPW) {
                            pcv[nc * TILE + r] = staged(stage, slot, q);
                            pcj[nc * TILE + r] = (uint16_t)(jc + q);
                            if (!XT && !resident) prefetch_l2(Vh + (size_t)(jc + q) * vstep);
                        }
                        ++nc;
                    } while (hits);
                }
            };
        };
        if (resident) {
            tc_fence_after();
            for (int n = 0; n < nblk && live; ++n) {
                if (XT) {  // no pass A waited on the blocks
                    live = warp_wait(smem_u32(&ctl->s_full[n]), 0u, &ctl->abort_flag, wc);
                    tc_fence_after();
                    if (!live) break;
                }
                for_half_block(ctl, n, g, pass_b(n));
            }
        } else {
            const int mA = g ? mA1 : mA0, mB = g ? mB1 : mB0;
            for (int m = mA; m < mA + mB; ++m) {
                const int buf = g + 2 * (m & 1);
                if (live) live = warp_wait(smem_u32(&ctl->s_full[buf]), (uint32_t)(m >> 1) & 1u, &ctl->abort_flag, wc);
                tc_fence_after();
                if (live) P::for_each_chunk(ctl, buf, pass_b(half_block(g, m, mA)));
            }
        }
        rows[g * TILE + r].nallow = nallow;
        rows[g * TILE + r].n = min(nc, CAPW);
        rows[g * TILE + r].ovf = nc > CAPW ? 1 : 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool aborted = P::aborted(ctl);
    const bool v_staged = !XT && resident && !aborted;

    // V blocks of a resident tile into the (now idle) ring, overlapping phase 2
    if (warp == WARP_PRODUCER && lane == 0 && v_staged) {
        mbar_arrive_expect_tx(smem_u32(vbar), (uint32_t)(nblk * BLK_BYTES));
        for (int s = 0; s < nblk; ++s) {
            const int row = (int)(blk_list[s] & ~FULL_BLOCK) * BLK;
            tma_load_3d(smem_u32(smem_b + s * BLK_BYTES), &map_v, 0, hkv.c1(row), hkv.c2(row), smem_u32(vbar));
        }
    }

    // ---------------- extraction: the support is every candidate with S_ij > tau_i; written as
    // phase 2 writes it (a row past a partition's list is marked unsaved), two threads per row
    if (XT && !aborted && tid < NUM_EPI) {
        const int r = (warp << 4) | (lane >> 1), h = lane & 1;
        const int i = i0 + r;
        const RowOut s0 = rows[r], s1 = rows[TILE + r];
        int mode = 0;  // 0: listed (none when no key is allowed), 2: unsaved (a partition overflowed), 3: no row
        if (i >= L) mode = 3;
        else if (s0.ovf | s1.ovf) mode = 2;
        const int nh = mode == 0 ? (h == 0 ? s0.n : s1.n) : 0;
        float* pcv = cv + h * CAPW * TILE;
        uint16_t* pcj = cj + h * CAPW * TILE;
        const float tau_i = nh > 0 ? out.tau[(size_t)bh * L + i] : 0.f;
        int sn = 0;
        for (int k = 0; k < nh; ++k) {
            const float d = fmaf(scale, pcv[k * TILE + r], -tau_i);  // S_ij - tau_i (scaled)
            const uint16_t j = pcj[k * TILE + r];
            if (d > 0.f) {
                // h_ij = sqrt(p_ij) (alpha 1.5) or b_ij = am1 (S_ij - tau_i) (general alpha)
                pcv[sn * TILE + r] = GEN ? am1 * d : 0.5f * d;
                pcj[sn * TILE + r] = j;
                ++sn;
            }
        }
        supp_cnt[h * TILE + r] = sn;
        __syncwarp();
        save_row_support<GEN>(out.save, cv, cj, supp_cnt, r, h, mode, (size_t)bh * L, (size_t)bhk * L, i, L);
    }

    // ---------------- phase 2: tau per row, two threads per row (one per partition)
    if (!XT && !aborted && tid < NUM_EPI) {
        const int r = (warp << 4) | (lane >> 1), h = lane & 1;
        const int i = i0 + r;
        const RowOut s0 = rows[r], s1 = rows[TILE + r];
        const int nallow = s0.nallow + s1.nallow;
        int mode = 0;  // 0: solved here, 2: fallback, 3: no key
        if (i >= L || nallow == 0) mode = 3;
        else if (s0.ovf | s1.ovf) mode = 2;
        const int nh = mode == 0 ? (h == 0 ? s0.n : s1.n) : 0;
        float* pcv = cv + h * CAPW * TILE;
        uint16_t* pcj = cj + h * CAPW * TILE;
        // Row max: pass A saw every block of a resident tile, so its largest chunk maximum is the max;
        // on a streamed tile take the largest candidate (the max exceeds every lower bound of tau, so
        // it is always listed).
        float cmax = fmaxf(s0.a0, s1.a0);
        if (!resident) {
            cmax = -INFINITY;
            for (int k = 0; k < nh; ++k) cmax = fmaxf(cmax, pcv[k * TILE + r]);
            cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
        }
        const float ms = scale * cmax;  // scaled row max
        // every lane takes part in the pair shuffles (rows of one warp may differ in mode)
        // Bracket (shifted scaled units, row max = 0): lo = the bound the candidates were cut at (the
        // exact threshold of the four largest chunk maxima, or max - 2), g(lo) >= g(tau) = 1; hi =
        // -2/sqrt(k) with k = the candidates listed, a superset of the support, so
        // g(hi) <= k (1/sqrt k)^2 = 1.  Both lie inside the pages' bracket [-2, -2/sqrt(n)].
        float b0 = s0.a0, b1 = s0.a1, b2 = s0.a2, b3 = s0.a3;
        top4_insert(s1.a0, b0, b1, b2, b3);
        top4_insert(s1.a1, b0, b1, b2, b3);
        top4_insert(s1.a2, b0, b1, b2, b3);
        top4_insert(s1.a3, b0, b1, b2, b3);
        const float t_cut = GEN ? gen_bound(b0, b1, b2, b3, wk, am1, ex, scale)
                                : fmaxf(b0 - two_over_scale, top4_bound(b0, b1, b2, b3, c4));
        // general alpha, in y units: g(-1) >= 1 from the max alone, g(-k^(-am1)) <= 1 over k candidates
        const float hi = GEN ? -pow_pos((float)max(s0.n + s1.n, 1), -am1) : -2.f / sqrtf((float)max(s0.n + s1.n, 1));
        const float lo = GEN ? fminf(fmaxf(-1.f, am1 * fmaf(scale, t_cut, -ms)), hi)
                             : fminf(fmaxf(-2.f, fmaf(scale, t_cut, -ms)), hi);
        // the row's candidates split evenly over its two threads; registers: the warp's largest share
        // rounded up to a multiple of eight
        const int ns = mode == 0 ? (s0.n + s1.n + 1 - h) >> 1 : 0;
        const int nmax = __reduce_max_sync(0xffffffffu, ns);
        float tau_x;  // alpha 1.5: scaled units (row max 0); general alpha: y units
        if (GEN) {
            switch ((nmax + 7) >> 3) {
                case 0:
                case 1: tau_x = solve_tau_gen<8>(cv, r, h, ns, s0.n, scale, ms, am1, ex, lo, hi); break;
                case 2: tau_x = solve_tau_gen<16>(cv, r, h, ns, s0.n, scale, ms, am1, ex, lo, hi); break;
                case 3: tau_x = solve_tau_gen<24>(cv, r, h, ns, s0.n, scale, ms, am1, ex, lo, hi); break;
                case 4: tau_x = solve_tau_gen<32>(cv, r, h, ns, s0.n, scale, ms, am1, ex, lo, hi); break;
                case 5: tau_x = solve_tau_gen<40>(cv, r, h, ns, s0.n, scale, ms, am1, ex, lo, hi); break;
                case 6: tau_x = solve_tau_gen<48>(cv, r, h, ns, s0.n, scale, ms, am1, ex, lo, hi); break;
                case 7: tau_x = solve_tau_gen<56>(cv, r, h, ns, s0.n, scale, ms, am1, ex, lo, hi); break;
                default: tau_x = solve_tau_gen<CAPW>(cv, r, h, ns, s0.n, scale, ms, am1, ex, lo, hi); break;
            }
        } else {
            switch ((nmax + 7) >> 3) {
                case 0:
                case 1: tau_x = solve_tau<8, CAPW>(cv, r, h, ns, s0.n, scale, ms, lo, hi); break;
                case 2: tau_x = solve_tau<16, CAPW>(cv, r, h, ns, s0.n, scale, ms, lo, hi); break;
                case 3: tau_x = solve_tau<24, CAPW>(cv, r, h, ns, s0.n, scale, ms, lo, hi); break;
                case 4: tau_x = solve_tau<32, CAPW>(cv, r, h, ns, s0.n, scale, ms, lo, hi); break;
                case 5: tau_x = solve_tau<40, CAPW>(cv, r, h, ns, s0.n, scale, ms, lo, hi); break;
                case 6: tau_x = solve_tau<48, CAPW>(cv, r, h, ns, s0.n, scale, ms, lo, hi); break;
                case 7: tau_x = solve_tau<56, CAPW>(cv, r, h, ns, s0.n, scale, ms, lo, hi); break;
                default: tau_x = solve_tau<CAPW, CAPW>(cv, r, h, ns, s0.n, scale, ms, lo, hi); break;
            }
        }
        if (mode == 0) {
            // this thread's partition of the support: cv <- h_ij = sqrt(p_ij) (alpha 1.5) or
            // b_ij = y - t (general alpha; p = b^ex), cj <- j (in place)
            int sn = 0;
            auto keep = [&](float c, uint16_t j) {
                const float xv = fmaf(scale, c, -ms);
                if (GEN) {
                    const float b = am1 * xv - tau_x;
                    if (b > 0.f) {
                        pcv[sn * TILE + r] = b;
                        pcj[sn * TILE + r] = j;
                        ++sn;
                    }
                } else if (xv > tau_x) {
                    const float hh = 0.5f * (xv - tau_x);
                    pcv[sn * TILE + r] = hh;  // h = sqrt(p)
                    pcj[sn * TILE + r] = j;
                    ++sn;
                }
            };
            // two entries per step, both read before either is written back (writes go to slots
            // sn <= k, never past the entries still to be read)
            for (int k = 0; k < nh; k += 2) {
                const bool two = k + 1 < nh;
                const float c0 = pcv[k * TILE + r], c1 = two ? pcv[(k + 1) * TILE + r] : -INFINITY;
                const uint16_t j0 = pcj[k * TILE + r], j1 = two ? pcj[(k + 1) * TILE + r] : (uint16_t)0;
                keep(c0, j0);
                keep(c1, j1);
            }
            supp_cnt[h * TILE + r] = sn;
            if (h == 0) out.tau[(size_t)bh * L + i] = GEN ? ms + tau_x * ex : ms + tau_x;
        } else if (mode == 2) {
            if (h == 0) atomicOr(&redo[r >> 5], 1u << (r & 31));
            supp_cnt[h * TILE + r] = 0;
        } else {
            supp_cnt[h * TILE + r] = 0;
            if (h == 0 && i < L) out.tau[(size_t)bh * L + i] = INFINITY;  // no allowed key: O_i = 0
        }
        __syncwarp();
        if (out.save.row_cnt)
            save_row_support<GEN>(out.save, cv, cj, supp_cnt, r, h, mode, (size_t)bh * L, (size_t)bhk * L, i, L);

        // ---------------- phase 3: O_i = sum_j p_ij V_j over the row's whole support (both
        // partitions); thread h of the pair accumulates dimensions [32 h, 32 h + 32) in registers
        const bool v_ok = !v_staged || warp_wait(smem_u32(vbar), 0u, &ctl->abort_flag, wc);
        if (v_ok && mode != 2 && i < L) {
            const int n0 = supp_cnt[r], n1 = supp_cnt[TILE + r];
            float acc[4][8];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[c][k] = 0.f;
            const int ns = n0 + n1;
            if (v_staged) {
                // two support entries per step (their shared-memory reads overlap; a missing second
                // entry repeats the first with weight 0)
                for (int e = 0; e < ns; e += 2) {
                    uint4 x[2][4];
                    float pw[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int ee = e + u < ns ? e + u : e;
                        const int sl = ee < n0 ? ee : CAPW + (ee - n0);
                        const int j = cj[sl * TILE + r];
                        const float c = cv[sl * TILE + r];
                        pw[u] = e + u < ns ? (GEN ? pow_pos(c, ex) : c * c) : 0.f;
                        // 128-byte swizzled V block in ring slot vslot[j / BLK]: 16-byte chunk q of
                        // row `row` sits at chunk position q ^ (row & 7)
                        const uint32_t row = (uint32_t)j & (BLK - 1);
                        const uint8_t* base = smem_b + vslot[j / BLK] * BLK_BYTES + row * 128u;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            x[u][q] = *reinterpret_cast<const uint4*>(base + ((((uint32_t)(4 * h + q)) ^ (row & 7u)) << 4));
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int q = 0; q < 4; ++q) fma_bf16x8(acc[q], pw[u], x[u][q]);
                }
            } else {
                // V rows from L2, two support entries per step (eight 16-byte loads in flight; a missing
                // second entry repeats the first with weight 0)
                for (int e = 0; e < ns; e += 2) {
                    uint4 x[2][4];
                    float pw[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int ee = e + u < ns ? e + u : e;
                        const int sl = ee < n0 ? ee : CAPW + (ee - n0);
                        const uint4* src = reinterpret_cast<const uint4*>(Vh + (size_t)cj[sl * TILE + r] * vstep) + 4 * h;
                        const float c = cv[sl * TILE + r];
                        pw[u] = e + u < ns ? (GEN ? pow_pos(c, ex) : c * c) : 0.f;
#pragma unroll
                        for (int c = 0; c < 4; ++c) x[u][c] = __ldg(src + c);
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int c = 0; c < 4; ++c) fma_bf16x8(acc[c], pw[u], x[u][c]);
                }
            }
            const size_t oi = hq.row(i) * HEAD_DIM + 32 * h;
            if (out.out_f32) {
                float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out.O) + oi);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    dst[2 * c] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
                    dst[2 * c + 1] = make_float4(acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
                }
            } else {
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out.O) + oi);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    __nv_bfloat162 hv[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) hv[k] = __floats2bfloat162_rn(acc[c][2 * k], acc[c][2 * k + 1]);
                    dst[c] = *reinterpret_cast<const uint4*>(hv);
                }
            }
            if (!GEN && out.otil) {
                // auxiliary row (alpha 1.5): Otil_i = sum_j h_ij V_j and r_i = sum_j h_ij over the same
                // support, in a second walk over it (the V rows are hot)
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int k = 0; k < 8; ++k) acc[c][k] = 0.f;
                float rs = 0.f;
                for (int e = 0; e < ns; ++e) {
                    const int sl = e < n0 ? e : CAPW + (e - n0);
                    const int j = cj[sl * TILE + r];
                    const float w = cv[sl * TILE + r];
                    rs += w;
                    uint4 x[4];
                    if (v_staged) {
                        const uint32_t row = (uint32_t)j & (BLK - 1);
                        const uint8_t* base = smem_b + vslot[j / BLK] * BLK_BYTES + row * 128u;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            x[q] = *reinterpret_cast<const uint4*>(base + ((((uint32_t)(4 * h + q)) ^ (row & 7u)) << 4));
                    } else {
                        const uint4* src = reinterpret_cast<const uint4*>(Vh + (size_t)j * vstep) + 4 * h;
#pragma unroll
                        for (int q = 0; q < 4; ++q) x[q] = __ldg(src + q);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) fma_bf16x8(acc[q], w, x[q]);
                }
                const size_t row = (size_t)bh * L + i;
                float4* dst = reinterpret_cast<float4*>(out.otil + row * HEAD_DIM + 32 * h);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    dst[2 * c] = make_float4(acc[c][0], acc[c][1], acc[c][2], acc[c][3]);
                    dst[2 * c + 1] = make_float4(acc[c][4], acc[c][5], acc[c][6], acc[c][7]);
                }
                if (h == 0) out.rsum[row] = rs;
            }
        }
    }
    __syncthreads();
    // a V wait that gave up raised the abort flag: the staged copies must land before exit
    if (v_staged && warp == WARP_PRODUCER && lane == 0 && P::aborted(ctl)) wait_drain(smem_u32(vbar), 0u);

    // ---------------- phase 4: exact redo of overflowed rows
    if (!XT && !P::aborted(ctl)) {
        for (int wd = 0; wd < TILE / 32; ++wd) {
            uint32_t mask = redo[wd];  // uniform across the CTA
            while (mask) {
                const int rr = wd * 32 + __ffs(mask) - 1;
                mask &= mask - 1;
                fallback_row<GEN>(reinterpret_cast<const __nv_bfloat16*>(args.Q),
                                  reinterpret_cast<const __nv_bfloat16*>(args.K),
                                  reinterpret_cast<const __nv_bfloat16*>(args.V), bits, scratch, red, hq, hkv, bh,
                                  i0 + rr, L, args.causal, args.window, scale, am1,
                                  rows[rr].nallow + rows[TILE + rr].nallow, out.O, out.out_f32, out.tau,
                                  out.otil, out.rsum);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // Past this barrier no thread waits, so the abort flag is final (uniform).  After an abort every
    // TMA load and MMA issued must complete before the CTA frees TMEM and its shared memory.
    if (P::aborted(ctl)) {
        if (lane == 0) {
            if (resident) {
                if (warp == WARP_PRODUCER) P::drain_loads(ctl);
                if (warp == WARP_MMA) P::drain_mma(ctl);
            } else if (warp == WARP_PRODUCER || warp == WARP_PRODUCER2) {
                drain_half(ctl, warp == WARP_PRODUCER ? 0 : 1, false);
            } else if (warp == WARP_MMA || warp == WARP_MMA2) {
                drain_half(ctl, warp == WARP_MMA ? 0 : 1, true);
            }
        }
        tc_fence_before();
        __syncthreads();
    }
    if (warp == WARP_PRODUCER) {
        tc_fence_after();
        tmem_dealloc(ctl->tmem_base, TMEM_COLS);
    }
}

}  // namespace

size_t fwd_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_fwd(const AttnArgs& a, const FwdOut& o, cudaStream_t stream, bool extract) {
    CUtensorMap mq, mk, mv;
    cudaError_t e = make_tile_map(&mq, a.Q, a.layout, a.B, a.H, a.L, TILE);
    if (e != cudaSuccess) return e;
    e = make_tile_map(&mk, a.K, a.layout, a.B, a.Hkv, a.L, BLK);
    if (e != cudaSuccess) return e;
    e = make_tile_map(&mv, a.V, a.layout, a.B, a.Hkv, a.L, BLK);
    if (e != cudaSuccess) return e;
    using Fn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const AttnArgs, const FwdOut);
    // [extract][generic alpha]; shared-memory attribute slots 0, 4 (forward), 12, 14 (extraction)
    static const Fn fns[2][2] = {{entmax_fwd_kernel<false, false>, entmax_fwd_kernel<true, false>},
                                 {entmax_fwd_kernel<false, true>, entmax_fwd_kernel<true, true>}};
    static const int slots[2][2] = {{0, 4}, {12, 14}};
    const bool gen = generic_alpha(a);
    const Fn f = fns[extract][gen];
    e = ensure_smem_attr(reinterpret_cast<const void*>(f), SMEM_BYTES, slots[extract][gen]);
    if (e != cudaSuccess) return e;
    dim3 grid((a.L + TILE - 1) / TILE, a.B * a.H);
    f<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(mq, mk, mv, a, o);
    return cudaGetLastError();
}

}  // namespace entmax
