// fwd.cu -- forward pass of 1.5-entmax attention on sm_100a.
//
// Computes, for every query row i of every (b, h) (page "svd-sst2-roberta-adasplash",
// sections 2.2-2.3 and 3; model cards "roberta-base-adasplash" / "distilbert-sst2-adasplash"):
//   S_ij = scale * Q_i . K_j over the allowed keys (key padding, causal, window),
//   tau_i with sum_j max(0, (S_ij - tau_i)/2)^2 = 1, by bisection on [max-2, max-2/sqrt(n)],
//   O_i = sum_j max(0, (S_ij - tau_i)/2)^2 V_j.
//
// One CTA per 128-query tile.  Phases:
//  1. S pass (common.cuh): QK^T on tcgen05, 128 keys per block, fp32 scores in TMEM.  Each
//     epilogue thread owns one query row and keeps only *candidates*: scores above a running
//     lower bound t of tau (max - 2, tightened to the exact threshold of the row's top four
//     scores whenever the list fills).  A score at or below any lower bound of tau is outside
//     the support, so the support is a subset of the candidates.
//  2. tau solve per row on the candidate list: the pages' 25 halvings of the bracket
//     [max - 2, max - 2/sqrt(n)], with g(mid) summed over the candidates (held in registers by two
//     threads per row), then the root of sum_S (S_ij - tau)^2 = 4 in closed form on the support
//     S = {S_ij > final midpoint}, kept if it lies in the final bracket (else the midpoint).
//  3. O_i = sum p_ij V_j over the support (typically 5-40 keys) with one warp per row: lane l
//     accumulates dimensions 2l, 2l+1 from V rows gathered out of L2 (prefetched into L2 when the
//     candidate was listed).
//  4. Rows whose candidates exceed the list capacity are redone exactly by the whole CTA on
//     CUDA cores (scores into shared memory, bisection with block reductions).
#include <cuda_bf16.h>
#include <math.h>
#include "common.cuh"
#include "internal.h"

namespace entmax {
namespace {

using P = Pipe<128, 4, 4, 2>;  // 128-key blocks, 4-deep ring, 4 TMEM buffers, 2 epilogue warpgroups
using PipeCtl = P::Ctl;
constexpr int BLK = P::BLK, NSTAGE = P::NSTAGE, NUM_EPI_WG = P::NUM_EPI_WG;
constexpr int NUM_EPI = P::NUM_EPI, NUM_THREADS = P::NUM_THREADS, NUM_WARPS = P::NUM_WARPS;
constexpr int WARP_PRODUCER = P::WARP_PRODUCER, WARP_MMA = P::WARP_MMA;
constexpr int BLK_BYTES = P::BLK_BYTES, TMEM_COLS = P::TMEM_COLS, MAX_BLOCKS = P::MAX_BLOCKS;
constexpr int STAGE_FLOATS = NUM_EPI * 32;  // per-thread staging of one 32-value chunk

constexpr int CAP = 128;              // candidates per row, split between the two warpgroups
constexpr int CAPW = CAP / NUM_EPI_WG;
constexpr int REG_CAND = 32;          // candidates per thread held in registers by the tau solve

// shared-memory layout (bytes from the 1024-aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + TILE_BYTES;
constexpr int OFF_CV = OFF_B + NSTAGE * BLK_BYTES;     // float [CAP][TILE]
constexpr int OFF_CJ = OFF_CV + CAP * TILE * 4;        // u16   [CAP][TILE]
constexpr int OFF_STAGE = OFF_CJ + CAP * TILE * 2;     // float [NUM_EPI][32]
constexpr int OFF_BITS = OFF_STAGE + STAGE_FLOATS * 4; // u32   [MASK_WORDS]
constexpr int OFF_BLK = OFF_BITS + MASK_WORDS * 4;     // u16   [MAX_BLOCKS]
constexpr int OFF_SUPP = OFF_BLK + MAX_BLOCKS * 2;     // int   [2][TILE] support size per partition
constexpr int OFF_ROWS = OFF_SUPP + 2 * TILE * 4;      // RowOut[2][TILE] per-warpgroup row state
constexpr int OFF_RED = OFF_ROWS + 2 * TILE * 32;      // float [NUM_THREADS]
constexpr int OFF_FLAGS = OFF_RED + NUM_THREADS * 4;   // u32   [TILE/32] rows redone by the fallback
constexpr int OFF_TSHARE = OFF_FLAGS + 16;             // float [2][2][TILE] bounds exchanged per block pair
constexpr int OFF_CTL = OFF_TSHARE + 4 * TILE * 4;
constexpr int SMEM_USED = OFF_CTL + (int)sizeof(PipeCtl);
constexpr int SMEM_BYTES = SMEM_USED + 1024;
// scratch reused after the S pass: per-row undecided candidates, then fallback score rows
constexpr int OFF_SCRATCH = 0;
constexpr int SCRATCH_BYTES = OFF_CV;
static_assert(CAP * TILE * 4 <= SCRATCH_BYTES, "undecided-candidate scratch must fit the S-pass buffers");
static_assert(MAX_L * 4 <= SCRATCH_BYTES, "fallback score row must fit the S-pass buffers");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct RowState {
    float t;                 // raw-score lower bound of tau (scores <= t are never in the support)
    float a0, a1, a2, a3;    // four largest raw scores seen by this warpgroup (a0 = running max)
    int n;                   // candidates stored in this warpgroup's partition
    int nallow;              // allowed keys seen
    int ovf;                 // partition overflowed: row is redone by the fallback
};

struct __align__(16) RowOut {
    float a0, a1, a2, a3;
    float t;
    int n, nallow, ovf;
};

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

// Drops the partition's candidates at or below the bound t; returns the new count.
__device__ __noinline__ int compact_list(float t, int n, float* cv, uint16_t* cj, int r) {
    int w = 0;
    for (int c = 0; c < n; ++c) {
        const float v = cv[c * TILE + r];
        if (v > t) {
            cv[w * TILE + r] = v;
            cj[w * TILE + r] = cj[c * TILE + r];
            ++w;
        }
    }
    return w;
}

// Append candidate v (key j) to this warpgroup's partition (cv/cj already offset to it), prefetch
// its V row into L2 for the output gather, and keep the warpgroup's four largest scores.  Returns
// true when v entered the top four (the caller then tightens the bound once per chunk).
__device__ __forceinline__ bool push_candidate(RowState& st, float v, int j, float* cv, uint16_t* cj, int r,
                                               const __nv_bfloat16* Vh) {
    if (!(v > st.t)) return false;  // the bound rose since the chunk was filtered
    if (st.n == CAPW) {
        st.n = compact_list(st.t, st.n, cv, cj, r);
        if (st.n == CAPW) {
            st.ovf = 1;
            st.t = INFINITY;
            return false;
        }
    }
    cv[st.n * TILE + r] = v;
    cj[st.n * TILE + r] = (uint16_t)j;
    ++st.n;
    prefetch_l2(Vh + (size_t)j * HEAD_DIM);
    if (v > st.a3) {
        top4_insert(v, st.a0, st.a1, st.a2, st.a3);
        return true;
    }
    return false;
}

// Writes row r's support (both partitions, p_ij in cv) to the saved lists as (j, sqrt(p_ij)) and
// counts each key once per row that holds it.  Run by the row's two threads (h = 0, 1) after phase 2;
// rows redone on CUDA cores (mode 2) or with more than SAVE_CAP entries are marked unsaved.
__device__ __forceinline__ void save_row_support(const SavedSupport& sv, const float* cv, const uint16_t* cj,
                                                 const int* supp_cnt, int r, int h, int mode, size_t head_row0,
                                                 int i, int L) {
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
        sv.row_sp[row * SAVE_CAP + base + e] = sqrtf(cv[(slot0 + e) * TILE + r]);
        atomicAdd(sv.key_cnt + head_row0 + j, 1);
    }
}

// Named barrier over the 8 epilogue warps (id 3; 0 is __syncthreads).
__device__ __forceinline__ void epi_pair_sync() {
    asm volatile("bar.sync 3, %0;" ::"n"(NUM_EPI) : "memory");
}

// Slow path of phase 2 (a partition keeps more than REG_CAND candidates above the bound): the same
// bisection by one thread over the candidate list in shared memory, with candidates already known
// to be in the support folded into running moments and those below the bracket dropped.  Writes the
// support compactly from slot 0: cv <- p_ij, cj <- j.  Returns tau_x; *supp = support size.
__device__ __noinline__ float solve_row_smem(float* cv, uint16_t* cj, float* U, int r, int n0, int n1, float scale,
                                             float ms, int nallow, int* supp) {
    float lo = -2.f, hi = -2.f / sqrtf((float)nallow);
    float K = 0.f, S1 = 0.f, S2 = 0.f;
    int u = 0;
    for (int q = 0; q < NUM_EPI_WG; ++q) {
        const int n = q == 0 ? n0 : n1;
        for (int c = q * CAPW; c < q * CAPW + n; ++c) {
            const float x = fmaf(scale, cv[c * TILE + r], -ms);
            if (x >= hi) {
                K += 1.f;
                S1 += x;
                S2 = fmaf(x, x, S2);
            } else if (x > lo) {
                U[u * TILE + r] = x;
                ++u;
            }
        }
    }
    for (int it = 0; it < 25 && u > 0; ++it) {
        const float mid = 0.5f * (lo + hi);
        float g = 0.25f * fmaf(mid * K, mid, fmaf(-2.f * mid, S1, S2));
        float ka = 0.f, s1a = 0.f, s2a = 0.f;
        for (int e = 0; e < u; ++e) {
            const float x = U[e * TILE + r];
            if (x >= mid) {
                const float d = x - mid;
                g = fmaf(0.25f * d, d, g);
                ka += 1.f;
                s1a += x;
                s2a = fmaf(x, x, s2a);
            }
        }
        int w = 0;
        if (g > 1.f) {
            lo = mid;
            for (int e = 0; e < u; ++e) {
                const float x = U[e * TILE + r];
                if (x > mid) U[w++ * TILE + r] = x;
            }
        } else {
            hi = mid;
            K += ka;
            S1 += s1a;
            S2 += s2a;
            for (int e = 0; e < u; ++e) {
                const float x = U[e * TILE + r];
                if (x < mid) U[w++ * TILE + r] = x;
            }
        }
        u = w;
    }
    float tau_x;
    if (u == 0 && K > 0.f) {
        const float mu = S1 / K;
        const float var = fmaxf(S2 / K - mu * mu, 0.f);
        tau_x = mu - sqrtf(fmaxf(4.f / K - var, 0.f));
        tau_x = fminf(fmaxf(tau_x, lo), hi);
    } else {
        tau_x = 0.5f * (lo + hi);
    }
    int s = 0;
    for (int q = 0; q < NUM_EPI_WG; ++q) {
        const int n = q == 0 ? n0 : n1;
        for (int c = q * CAPW; c < q * CAPW + n; ++c) {
            const float x = fmaf(scale, cv[c * TILE + r], -ms);
            if (x > tau_x) {
                const float h = 0.5f * (x - tau_x);
                cv[s * TILE + r] = h * h;
                cj[s * TILE + r] = cj[c * TILE + r];
                ++s;
            }
        }
    }
    *supp = s;
    return tau_x;
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

// Phase 4: the whole CTA recomputes one row exactly on CUDA cores.
__device__ __noinline__ void fallback_row(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                                          const __nv_bfloat16* __restrict__ V, const uint32_t* bits, float* sbuf,
                                          float* red, int bh, int i, int L, int causal, int window, float scale,
                                          int nallow, void* O, int out_f32, float* tau) {
    const int tid = threadIdx.x;
    float* qf = red + 64;  // 64 floats (red[0..63] holds reduction partials)
    const size_t head = (size_t)bh * L * HEAD_DIM;
    __syncthreads();
    if (tid < HEAD_DIM) qf[tid] = __bfloat162float(Q[head + (size_t)i * HEAD_DIM + tid]);
    __syncthreads();
    int lo, hi;
    row_key_range(i, L, causal, window, lo, hi);
    const int span = hi - lo + 1;
    float mloc = -INFINITY;
    for (int e = tid; e < span; e += NUM_THREADS) {
        const int j = lo + e;
        float s = -INFINITY;
        if ((bits[j >> 5] >> (j & 31)) & 1u) {
            const uint4* kr = reinterpret_cast<const uint4*>(K + head + (size_t)j * HEAD_DIM);
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
    float blo = m - 2.f, bhi = m - 2.f / sqrtf((float)nallow);
    bool resolved = false;
    for (int it = 0; it < 25; ++it) {
        const float mid = 0.5f * (blo + bhi);
        float gl = 0.f, inside = 0.f;
        for (int e = tid; e < span; e += NUM_THREADS) {
            const float s = sbuf[e];
            if (s > mid) {
                const float d = 0.5f * (s - mid);
                gl = fmaf(d, d, gl);
            }
            if (s > blo && s < bhi) inside += 1.f;
        }
        const float2 r2 = block_sum2(gl, inside, red);
        if (r2.y == 0.f) {
            resolved = true;
            break;
        }
        if (r2.x > 1.f) blo = mid;
        else bhi = mid;
    }
    float t;
    if (!resolved) {
        // one more count: the last halving may have emptied the bracket
        float inside = 0.f;
        for (int e = tid; e < span; e += NUM_THREADS) {
            const float s = sbuf[e];
            if (s > blo && s < bhi) inside += 1.f;
        }
        resolved = block_sum2(inside, 0.f, red).x == 0.f;
    }
    if (resolved) {
        float k = 0.f, s1 = 0.f, s2 = 0.f;
        for (int e = tid; e < span; e += NUM_THREADS) {
            const float s = sbuf[e];
            if (s >= bhi) {
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
    // O_i: thread -> (dimension d, key phase ph)
    constexpr int PH = NUM_THREADS / HEAD_DIM;
    const int d = tid % HEAD_DIM, ph = tid / HEAD_DIM;
    float acc = 0.f;
    for (int e = ph; e < span; e += PH) {
        const float s = sbuf[e];
        if (s > t) {
            const float h = 0.5f * (s - t);
            acc = fmaf(h * h, __bfloat162float(V[head + (size_t)(lo + e) * HEAD_DIM + d]), acc);
        }
    }
    __syncthreads();
    red[tid] = acc;
    __syncthreads();
    if (tid < HEAD_DIM) {
        float o = 0.f;
#pragma unroll
        for (int p = 0; p < PH; ++p) o += red[tid + p * HEAD_DIM];
        const size_t oi = head + (size_t)i * HEAD_DIM + tid;
        if (out_f32) reinterpret_cast<float*>(O)[oi] = o;
        else reinterpret_cast<__nv_bfloat16*>(O)[oi] = __float2bfloat16_rn(o);
        if (tid == 0) tau[(size_t)bh * L + i] = t;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
entmax_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  const AttnArgs args, const FwdOut out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smem_a = smem + OFF_A;
    uint8_t* smem_b = smem + OFF_B;
    float* cv = reinterpret_cast<float*>(smem + OFF_CV);
    uint16_t* cj = reinterpret_cast<uint16_t*>(smem + OFF_CJ);
    float* stage = reinterpret_cast<float*>(smem + OFF_STAGE);
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + OFF_BITS);
    uint16_t* blk_list = reinterpret_cast<uint16_t*>(smem + OFF_BLK);
    int* supp_cnt = reinterpret_cast<int*>(smem + OFF_SUPP);
    RowOut* rows = reinterpret_cast<RowOut*>(smem + OFF_ROWS);
    float* red = reinterpret_cast<float*>(smem + OFF_RED);
    uint32_t* redo = reinterpret_cast<uint32_t*>(smem + OFF_FLAGS);
    float* tshare = reinterpret_cast<float*>(smem + OFF_TSHARE);
    float* scratch = reinterpret_cast<float*>(smem + OFF_SCRATCH);
    PipeCtl* ctl = reinterpret_cast<PipeCtl*>(smem + OFF_CTL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = args.L;
    const int tile = blockIdx.x, bh = blockIdx.y;
    const int b = bh / args.H;
    const int i0 = tile * TILE;
    const WaitCfg wc{args.status, args.timeout_ns};
    const __nv_bfloat16* Vh = reinterpret_cast<const __nv_bfloat16*>(args.V) + (size_t)bh * L * HEAD_DIM;

    if (tid == 0) {
        P::init(ctl);
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_k);
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
        if (lane == 0) ctl->nblk = nb;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const float scale = args.scale;
    const float c4 = 4.f / (scale * scale);
    const float two_over_scale = 2.f / scale;

    if (warp == WARP_PRODUCER) {
        if (lane == 0) P::producer(ctl, wc, &map_q, &map_k, bh, i0, blk_list, smem_a, smem_b);
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0) P::mma(ctl, wc, smem_a, smem_b);
        __syncwarp();
    } else {
        // ---------------- phase 1: candidate filter (thread (g, r): row i0 + r, blocks n = g mod 2)
        const int r = tid & (TILE - 1), g = tid >> 7;
        RowState st{-INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, 0, 0, 0};
        const int i = i0 + r;
        int rlo, rhi;
        row_key_range(i, L, args.causal, args.window, rlo, rhi);
        float* pcv = cv + g * CAPW * TILE;
        uint16_t* pcj = cj + g * CAPW * TILE;
        const int nblk = ctl->nblk;
        bool live = true;
        // the two warpgroups take blocks 2k and 2k+1, then swap bounds: the other warpgroup's bound
        // is a lower bound of tau as well (any subset of a row), and exchanging it at fixed points
        // keeps the candidate sets, hence the results, independent of timing
        for (int k = 0; 2 * k < nblk; ++k) {
            const int n = 2 * k + g;
            if (n < nblk && live) live = P::wait_scores(ctl, wc, n);
            if (n < nblk && live) {
                const int j0 = (int)(blk_list[n] & ~FULL_BLOCK) * BLK;
                const bool full = (blk_list[n] & FULL_BLOCK) && i < L;
                P::for_each_chunk(ctl, n, [&](const float (&cur)[32], int c) {
                    const int jc = j0 + c * 32;
                    const uint32_t vm = full ? 0xffffffffu
                                             : (jc < L && i < L) ? (bits[jc >> 5] & range_bits(jc, rlo, rhi)) : 0u;
                    st.nallow += __popc(vm);
                    if (st.t == -INFINITY && vm != 0u) {
                        // first allowed scores of this row: start from (max - 2) of the chunk
                        float mx = -INFINITY;
#pragma unroll
                        for (int q = 0; q < 32; ++q) mx = fmaxf(mx, ((vm >> q) & 1u) ? cur[q] : -INFINITY);
                        st.t = mx - two_over_scale;
                    }
                    uint32_t hits = hit_bits(cur, st.t) & __brev(vm);
                    if (hits) {
                        stage_chunk(stage, threadIdx.x % NUM_EPI, cur);
                        bool grew = false;
                        do {
                            const int q = __clz(hits);
                            hits &= ~(0x80000000u >> q);
                            grew |= push_candidate(st, staged(stage, threadIdx.x % NUM_EPI, q), jc + q, pcv, pcj, r, Vh);
                        } while (hits);
                        // early in the row the bound moves fast: tighten it after every chunk of the
                        // first block, later once per block pair (below)
                        if (grew && k == 0) st.t = fmaxf(st.t, top4_bound(st.a0, st.a1, st.a2, st.a3, c4));
                    }
                });
            }
            if (k > 0) st.t = fmaxf(st.t, top4_bound(st.a0, st.a1, st.a2, st.a3, c4));
            float* tx = tshare + (k & 1) * 2 * TILE;
            tx[g * TILE + r] = st.t;
            epi_pair_sync();
            st.t = fmaxf(st.t, tx[(g ^ 1) * TILE + r]);
        }
        rows[g * TILE + r] = RowOut{st.a0, st.a1, st.a2, st.a3, st.t, st.n, st.nallow, st.ovf};
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool aborted = P::aborted(ctl);

    // ---------------- phase 2: tau per row, two threads per row (one per partition)
    if (!aborted && tid < NUM_EPI) {
        const int r = (warp << 4) | (lane >> 1), h = lane & 1;
        const int i = i0 + r;
        const RowOut s0 = rows[r], s1 = rows[TILE + r];
        const int nallow = s0.nallow + s1.nallow;
        const int ovf = s0.ovf | s1.ovf;
        // merged bound: the four largest scores of the whole row
        float a0 = s0.a0, a1 = s0.a1, a2 = s0.a2, a3 = s0.a3;
        top4_insert(s1.a0, a0, a1, a2, a3);
        top4_insert(s1.a1, a0, a1, a2, a3);
        top4_insert(s1.a2, a0, a1, a2, a3);
        top4_insert(s1.a3, a0, a1, a2, a3);
        const float tf = fmaxf(fmaxf(s0.t, s1.t), top4_bound(a0, a1, a2, a3, c4));
        const float ms = scale * a0;  // scaled row max
        int mode = 0;                 // 0: registers, 1: slow path, 2: fallback, 3: no key
        if (i >= L || nallow == 0) mode = 3;
        else if (ovf) mode = 2;
        int nh = h == 0 ? s0.n : s1.n;
        float* pcv = cv + h * CAPW * TILE;
        uint16_t* pcj = cj + h * CAPW * TILE;
        if (mode == 0 && nh > REG_CAND) nh = compact_list(tf, nh, pcv, pcj, r);
        // every lane takes part in the pair shuffles below (rows of one warp may differ in mode)
        const int nh_other = __shfl_xor_sync(0xffffffffu, nh, 1);
        if (mode == 0 && (nh > REG_CAND || nh_other > REG_CAND)) mode = 1;
        float x[REG_CAND];
#pragma unroll
        for (int k = 0; k < REG_CAND; ++k) {
            const float v = (mode == 0 && k < nh) ? pcv[k * TILE + r] : -INFINITY;
            x[k] = v > tf ? fmaf(scale, v, -ms) : -INFINITY;
        }
        float lo = -2.f, hi = -2.f / sqrtf((float)max(nallow, 1));
        for (int it = 0; it < 25; ++it) {
            const float mid = 0.5f * (lo + hi);
            float g0 = 0.f, g1 = 0.f, g2 = 0.f, g3 = 0.f;
#pragma unroll
            for (int k = 0; k < REG_CAND; k += 4) {
                const float d0 = fmaxf(x[k] - mid, 0.f), d1 = fmaxf(x[k + 1] - mid, 0.f);
                const float d2 = fmaxf(x[k + 2] - mid, 0.f), d3 = fmaxf(x[k + 3] - mid, 0.f);
                g0 = fmaf(d0, d0, g0);
                g1 = fmaf(d1, d1, g1);
                g2 = fmaf(d2, d2, g2);
                g3 = fmaf(d3, d3, g3);
            }
            float gs = (g0 + g1) + (g2 + g3);
            gs += __shfl_xor_sync(0xffffffffu, gs, 1);
            if (0.25f * gs > 1.f) lo = mid;
            else hi = mid;
        }
        // support fixed by the final bracket: closed-form root of sum_S (x - tau)^2 = 4
        const float mid = 0.5f * (lo + hi);
        float K = 0.f, S1 = 0.f, S2 = 0.f;
#pragma unroll
        for (int k = 0; k < REG_CAND; ++k) {
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
            if (tc >= lo && tc <= hi) tau_x = tc;
        }
        if (mode == 0) {
            // this thread's partition of the support: cv <- p_ij, cj <- j (in place)
            int sn = 0;
            for (int k = 0; k < nh; ++k) {
                const float xv = fmaf(scale, pcv[k * TILE + r], -ms);
                if (xv > tau_x) {
                    const float hh = 0.5f * (xv - tau_x);
                    pcv[sn * TILE + r] = hh * hh;
                    pcj[sn * TILE + r] = pcj[k * TILE + r];
                    ++sn;
                }
            }
            supp_cnt[h * TILE + r] = sn;
            if (h == 0) out.tau[(size_t)bh * L + i] = ms + tau_x;
        } else if (mode == 1) {
            if (h == 0) {
                int sn = 0;
                // counts after this pair's compaction (h = 0 holds partition 0, its partner partition 1)
                const float tx = solve_row_smem(cv, cj, scratch, r, nh, nh_other, scale, ms, nallow, &sn);
                supp_cnt[r] = sn;
                supp_cnt[TILE + r] = 0;
                out.tau[(size_t)bh * L + i] = ms + tx;
            }
        } else if (mode == 2) {
            if (h == 0) atomicOr(&redo[r >> 5], 1u << (r & 31));
            supp_cnt[h * TILE + r] = 0;
        } else {
            supp_cnt[h * TILE + r] = 0;
            if (h == 0 && i < L) out.tau[(size_t)bh * L + i] = INFINITY;  // no allowed key: O_i = 0
        }
        __syncwarp();  // the slow path's counts (written by h = 0) are read by both threads of the pair
        if (out.save.row_cnt) save_row_support(out.save, cv, cj, supp_cnt, r, h, mode, (size_t)bh * L, i, L);
    }
    __syncthreads();

    // ---------------- phase 3: O_i = sum_j p_ij V_j, one warp per row, two rows in flight
    if (!aborted) {
        for (int ra = warp; ra < TILE; ra += 2 * NUM_WARPS) {
            const int rb = ra + NUM_WARPS;
            const bool okb = rb < TILE;
            float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
            const int na0 = supp_cnt[ra], na1 = supp_cnt[TILE + ra];
            const int nb0 = okb ? supp_cnt[rb] : 0, nb1 = okb ? supp_cnt[TILE + rb] : 0;
            gather_accumulate2(Vh, cj, cv, ra, 0, na0, okb ? rb : ra, 0, nb0, lane, a0, a1, b0, b1);
            gather_accumulate2(Vh, cj, cv, ra, CAPW, CAPW + na1, okb ? rb : ra, CAPW, CAPW + nb1, lane, a0, a1, b0, b1);
            for (int q = 0; q < 2; ++q) {
                const int rr = q == 0 ? ra : rb;
                const int i = i0 + rr;
                if ((q == 1 && !okb) || i >= L || ((redo[rr >> 5] >> (rr & 31)) & 1u)) continue;
                const float o0 = q == 0 ? a0 : b0, o1 = q == 0 ? a1 : b1;
                const size_t oi = ((size_t)bh * L + i) * HEAD_DIM + 2 * lane;
                if (out.out_f32) {
                    *reinterpret_cast<float2*>(reinterpret_cast<float*>(out.O) + oi) = make_float2(o0, o1);
                } else {
                    *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(out.O) + oi) =
                        __floats2bfloat162_rn(o0, o1);
                }
            }
        }
    }
    __syncthreads();

    // ---------------- phase 4: exact redo of overflowed rows
    if (!aborted) {
        for (int wd = 0; wd < TILE / 32; ++wd) {
            uint32_t mask = redo[wd];  // uniform across the CTA
            while (mask) {
                const int rr = wd * 32 + __ffs(mask) - 1;
                mask &= mask - 1;
                fallback_row(reinterpret_cast<const __nv_bfloat16*>(args.Q), reinterpret_cast<const __nv_bfloat16*>(args.K),
                             reinterpret_cast<const __nv_bfloat16*>(args.V), bits, scratch, red, bh, i0 + rr, L,
                             args.causal, args.window, scale, rows[rr].nallow + rows[TILE + rr].nallow, out.O,
                             out.out_f32, out.tau);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_PRODUCER) {
        tc_fence_after();
        tmem_dealloc(ctl->tmem_base, TMEM_COLS);
    }
}

}  // namespace

size_t fwd_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_fwd(const AttnArgs& a, const FwdOut& o, cudaStream_t stream) {
    CUtensorMap mq, mk;
    cudaError_t e = make_tile_map(&mq, a.Q, a.B * a.H, a.L, TILE);
    if (e != cudaSuccess) return e;
    e = make_tile_map(&mk, a.K, a.B * a.H, a.L, BLK);
    if (e != cudaSuccess) return e;
    e = ensure_smem_attr(reinterpret_cast<const void*>(entmax_fwd_kernel), SMEM_BYTES, 0);
    if (e != cudaSuccess) return e;
    dim3 grid((a.L + TILE - 1) / TILE, a.B * a.H);
    entmax_fwd_kernel<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(mq, mk, a, o);
    return cudaGetLastError();
}

}  // namespace entmax
