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
//  2. tau solve per row on the candidate list: the pages' bisection, where candidates already
//     known to lie above the bracket are folded into running moments and those below it are
//     dropped; once no candidate lies strictly inside the bracket the support is fixed and the
//     root of the now-quadratic constraint is taken in closed form.  If 25 halvings leave the
//     support undecided the final midpoint is used, as on the pages.
//  3. O_i = sum p_ij V_j over the support (typically 5-40 keys) with one warp per row: lane l
//     accumulates dimensions 2l, 2l+1 from V rows gathered out of L2.
//  4. Rows whose candidates exceed the list capacity are redone exactly by the whole CTA on
//     CUDA cores (scores into shared memory, bisection with block reductions).
#include <cuda_bf16.h>
#include <math.h>
#include "common.cuh"
#include "internal.h"

namespace entmax {
namespace {

constexpr int CAP = 128;  // candidates per row

// shared-memory layout (bytes from the 1024-aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + TILE_BYTES;
constexpr int OFF_CV = OFF_B + NSTAGE * BLK_BYTES;     // float [CAP][TILE]
constexpr int OFF_CJ = OFF_CV + CAP * TILE * 4;        // u16   [CAP][TILE]
constexpr int OFF_BITS = OFF_CJ + CAP * TILE * 2;      // u32   [MASK_WORDS]
constexpr int OFF_BLK = OFF_BITS + MASK_WORDS * 4;     // u16   [MAX_BLOCKS]
constexpr int OFF_SUPP = OFF_BLK + MAX_BLOCKS * 2;     // int   [TILE]  support size (or -1: redo)
constexpr int OFF_NALLOW = OFF_SUPP + TILE * 4;        // int   [TILE]
constexpr int OFF_RED = OFF_NALLOW + TILE * 4;         // float [256]   reductions / fallback q
constexpr int OFF_CTL = OFF_RED + 256 * 4;
constexpr int SMEM_USED = OFF_CTL + (int)sizeof(PipeCtl);
constexpr int SMEM_BYTES = SMEM_USED + 1024;
// scratch reused after the S pass: per-row undecided candidates, then fallback score rows
constexpr int OFF_SCRATCH = 0;
constexpr int SCRATCH_BYTES = OFF_CV;
static_assert(CAP * TILE * 4 <= SCRATCH_BYTES, "undecided-candidate scratch must fit the S-pass buffers");
static_assert(MAX_L * 4 <= SCRATCH_BYTES, "fallback score row must fit the S-pass buffers");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct RowState {
    float t;        // raw-score lower bound of tau (scores <= t are never in the support)
    float m;        // running max raw score
    int n;          // candidates stored
    int nallow;     // allowed keys seen
    int ovf;        // list overflowed: row is redone by the fallback
};

// Exact threshold (raw units, constraint sum (v - t)^2 = c4) of the four largest candidates:
// a valid lower bound of the row's tau, used to prune a full list.
__device__ __noinline__ void prune_list(RowState& st, float* cv, uint16_t* cj, int r, float c4) {
    float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
    for (int c = 0; c < st.n; ++c) {
        const float v = cv[c * TILE + r];
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
    const float z[4] = {a0, a1, a2, a3};
    float sum = 0.f, sq = 0.f, bound = a0 - sqrtf(c4);
#pragma unroll
    for (int k = 1; k <= 4; ++k) {
        sum += z[k - 1];
        sq = fmaf(z[k - 1], z[k - 1], sq);
        const float mu = sum / k;
        const float delta = c4 / k - (sq / k - mu * mu);
        if (delta >= 0.f) {
            const float tk = mu - sqrtf(delta);
            if (tk <= z[k - 1]) bound = tk;
        }
    }
    st.t = fmaxf(st.t, bound);
    int w = 0;
    for (int c = 0; c < st.n; ++c) {
        const float v = cv[c * TILE + r];
        if (v > st.t) {
            cv[w * TILE + r] = v;
            cj[w * TILE + r] = cj[c * TILE + r];
            ++w;
        }
    }
    st.n = w;
}

__device__ __forceinline__ void push_candidate(RowState& st, float v, int j, float* cv, uint16_t* cj, int r,
                                               float c4, float two_over_scale) {
    if (st.n == CAP) {
        prune_list(st, cv, cj, r, c4);
        if (st.n == CAP) {
            st.ovf = 1;
            st.t = INFINITY;
            return;
        }
        if (!(v > st.t)) return;
    }
    cv[st.n * TILE + r] = v;
    cj[st.n * TILE + r] = (uint16_t)j;
    ++st.n;
    if (v > st.m) {
        st.m = v;
        st.t = fmaxf(st.t, v - two_over_scale);
    }
}

// Phase 2: tau of one row from its candidate list.  Works in shifted, scaled units
// x = scale * v - ms (ms = scale * max), bracket [-2, -2/sqrt(nallow)].  Rewrites the list
// in place as the support: cv <- p_ij, cj <- j.  Returns tau_x; *supp = support size.
__device__ float solve_row(float* cv, uint16_t* cj, float* U, int r, int n, float scale, float ms, int nallow,
                           int* supp) {
    float lo = -2.f, hi = -2.f / sqrtf((float)nallow);
    float K = 0.f, S1 = 0.f, S2 = 0.f;  // moments of candidates known to be in the support
    int u = 0;                          // undecided candidates (strictly inside the bracket)
    for (int c = 0; c < n; ++c) {
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
    for (int it = 0; it < 25 && u > 0; ++it) {
        const float mid = 0.5f * (lo + hi);
        // g(mid) = sum over the support side of ((x - mid)/2)^2
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
        if (g > 1.f) {  // root lies right of mid
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
        // support fixed: sum_S (x - tau)^2 = 4, smaller root
        const float mu = S1 / K;
        const float var = fmaxf(S2 / K - mu * mu, 0.f);
        tau_x = mu - sqrtf(fmaxf(4.f / K - var, 0.f));
        tau_x = fminf(fmaxf(tau_x, lo), hi);
    } else {
        tau_x = 0.5f * (lo + hi);
    }
    int s = 0;
    for (int c = 0; c < n; ++c) {
        const float x = fmaf(scale, cv[c * TILE + r], -ms);
        if (x > tau_x) {
            const float h = 0.5f * (x - tau_x);
            cv[s * TILE + r] = h * h;
            cj[s * TILE + r] = cj[c * TILE + r];
            ++s;
        }
    }
    *supp = s;
    return tau_x;
}

// Block-wide sum of two floats (all NUM_THREADS threads call it).
__device__ __forceinline__ float2 block_sum2(float a, float b, float* red) {
    a = warp_sum(a);
    b = warp_sum(b);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) {
        red[warp] = a;
        red[8 + warp] = b;
    }
    __syncthreads();
    float sa = 0.f, sb = 0.f;
#pragma unroll
    for (int w = 0; w < NUM_THREADS / 32; ++w) {
        sa += red[w];
        sb += red[8 + w];
    }
    return make_float2(sa, sb);
}

__device__ __forceinline__ float block_max(float a, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[16 + warp] = a;
    __syncthreads();
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < NUM_THREADS / 32; ++w) m = fmaxf(m, red[16 + w]);
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
    const int d = tid & (HEAD_DIM - 1), ph = tid >> 6;
    float acc = 0.f;
    for (int e = ph; e < span; e += NUM_THREADS / HEAD_DIM) {
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
        const float o = red[tid] + red[tid + 64] + red[tid + 128] + red[tid + 192];
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
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + OFF_BITS);
    uint16_t* blk_list = reinterpret_cast<uint16_t*>(smem + OFF_BLK);
    int* supp_cnt = reinterpret_cast<int*>(smem + OFF_SUPP);
    int* nallow_s = reinterpret_cast<int*>(smem + OFF_NALLOW);
    float* red = reinterpret_cast<float*>(smem + OFF_RED);
    float* scratch = reinterpret_cast<float*>(smem + OFF_SCRATCH);
    PipeCtl* ctl = reinterpret_cast<PipeCtl*>(smem + OFF_CTL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = args.L;
    const int tile = blockIdx.x, bh = blockIdx.y;
    const int b = bh / args.H;
    const int i0 = tile * TILE;
    const WaitCfg wc{args.status, args.timeout_ns};

    if (tid == 0) {
        init_pipe(ctl);
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_k);
    }
    if (warp == 4) {
        tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    build_key_bitmap(bits, args.key_mask, b, L);
    __syncthreads();
    if (tid == 0) {
        // key blocks that hold at least one key some row of this tile may attend to
        const int i_last = min(i0 + TILE - 1, L - 1);
        int klo = 0, khi = L - 1;
        if (args.window > 0) klo = max(0, i0 - args.window + 1);
        if (args.causal) khi = i_last;
        int nb = 0;
        for (int kb = klo / BLK; kb <= khi / BLK; ++kb) {
            bool any = false;
            for (int w = kb * (BLK / 32); w < (kb + 1) * (BLK / 32) && w * 32 <= khi; ++w)
                any |= (bits[w] & range_bits(w * 32, klo, khi)) != 0u;
            if (any) blk_list[nb++] = (uint16_t)kb;
        }
        ctl->nblk = nb;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const float scale = args.scale;
    const float two_over_scale = 2.f / scale;
    const float c4 = 4.f / (scale * scale);
    RowState st{-INFINITY, -INFINITY, 0, 0, 0};

    if (warp == 4) {
        if (lane == 0) role_producer(ctl, wc, &map_q, &map_k, bh, i0, blk_list, smem_a, smem_b);
        __syncwarp();
    } else if (warp == 5) {
        if (lane == 0) role_mma(ctl, wc, smem_a, smem_b);
        __syncwarp();
    } else if (warp < 4) {
        // ---------------- phase 1: candidate filter (thread r = query row i0 + r)
        const int r = tid;
        const int i = i0 + r;
        int rlo, rhi;
        row_key_range(i, L, args.causal, args.window, rlo, rhi);
        const uint32_t lane_base = ctl->tmem_base + ((uint32_t)(warp * 32) << 16);
        const int nblk = ctl->nblk;
        for (int n = 0; n < nblk; ++n) {
            if (!epi_wait_scores(ctl, wc, n)) break;
            const int j0 = (int)blk_list[n] * BLK;
#pragma unroll 1
            for (int c = 0; c < BLK / 32; ++c) {
                float v[32];
                tmem_ld32(lane_base + (uint32_t)((n & 1) * BLK + c * 32), v);
                tmem_wait_ld();
                if (c == BLK / 32 - 1) epi_release_scores(ctl, n);
                const int jc = j0 + c * 32;
                const uint32_t vm = (jc < L) ? (bits[jc >> 5] & range_bits(jc, rlo, rhi)) : 0u;
                if (i >= L) continue;
                st.nallow += __popc(vm);
                if (vm == 0xffffffffu) {
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (v[k] > st.t) push_candidate(st, v[k], jc + k, cv, cj, r, c4, two_over_scale);
                } else if (vm != 0u) {
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (((vm >> k) & 1u) && v[k] > st.t) push_candidate(st, v[k], jc + k, cv, cj, r, c4, two_over_scale);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool aborted = cta_aborted(ctl);

    // ---------------- phase 2: tau per row (scratch reuses the S-pass buffers)
    if (!aborted && warp < 4) {
        const int r = tid, i = i0 + r;
        int supp = 0;
        if (i < L) {
            if (st.nallow == 0) {
                out.tau[(size_t)bh * L + i] = INFINITY;  // no allowed key: O_i = 0
            } else if (st.ovf) {
                supp = -1;
            } else {
                const float ms = scale * st.m;
                const float tau_x = solve_row(cv, cj, scratch, r, st.n, scale, ms, st.nallow, &supp);
                out.tau[(size_t)bh * L + i] = ms + tau_x;
            }
        }
        supp_cnt[r] = supp;
        nallow_s[r] = st.nallow;
    }
    __syncthreads();

    // ---------------- phase 3: O_i = sum_j p_ij V_j, one warp per row
    if (!aborted) {
        const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(args.V);
        const size_t head = (size_t)bh * L * HEAD_DIM;
        for (int r = warp; r < TILE; r += NUM_THREADS / 32) {
            const int i = i0 + r;
            const int k = supp_cnt[r];
            if (i >= L || k < 0) continue;
            float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
            int e = 0;
            for (; e + 2 <= k; e += 2) {
                const int j0 = cj[e * TILE + r], j1 = cj[(e + 1) * TILE + r];
                const float p0 = cv[e * TILE + r], p1 = cv[(e + 1) * TILE + r];
                const uint32_t w0 = reinterpret_cast<const uint32_t*>(V + head + (size_t)j0 * HEAD_DIM)[lane];
                const uint32_t w1 = reinterpret_cast<const uint32_t*>(V + head + (size_t)j1 * HEAD_DIM)[lane];
                a0 = fmaf(p0, bf16lo(w0), a0);
                a1 = fmaf(p0, bf16hi(w0), a1);
                b0 = fmaf(p1, bf16lo(w1), b0);
                b1 = fmaf(p1, bf16hi(w1), b1);
            }
            if (e < k) {
                const int j0 = cj[e * TILE + r];
                const float p0 = cv[e * TILE + r];
                const uint32_t w0 = reinterpret_cast<const uint32_t*>(V + head + (size_t)j0 * HEAD_DIM)[lane];
                a0 = fmaf(p0, bf16lo(w0), a0);
                a1 = fmaf(p0, bf16hi(w0), a1);
            }
            a0 += b0;
            a1 += b1;
            const size_t oi = head + (size_t)i * HEAD_DIM + 2 * lane;
            if (out.out_f32) {
                *reinterpret_cast<float2*>(reinterpret_cast<float*>(out.O) + oi) = make_float2(a0, a1);
            } else {
                __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
                *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(out.O) + oi) = h;
            }
        }
    }
    __syncthreads();

    // ---------------- phase 4: exact redo of overflowed rows
    if (!aborted) {
        for (int r = 0; r < TILE; ++r) {
            if (supp_cnt[r] >= 0) continue;  // uniform across the CTA
            fallback_row(reinterpret_cast<const __nv_bfloat16*>(args.Q), reinterpret_cast<const __nv_bfloat16*>(args.K),
                         reinterpret_cast<const __nv_bfloat16*>(args.V), bits, scratch, red, bh, i0 + r, L,
                         args.causal, args.window, scale, nallow_s[r], out.O, out.out_f32, out.tau);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(ctl->tmem_base, TMEM_COLS);
    }
}

}  // namespace

size_t fwd_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_fwd(const AttnArgs& a, const FwdOut& o, cudaStream_t stream) {
    CUtensorMap mq, mk;
    cudaError_t e = make_tile_map(&mq, a.Q, a.B * a.H, a.L);
    if (e != cudaSuccess) return e;
    e = make_tile_map(&mk, a.K, a.B * a.H, a.L);
    if (e != cudaSuccess) return e;
    e = ensure_smem_attr(reinterpret_cast<const void*>(entmax_fwd_kernel), SMEM_BYTES, 0);
    if (e != cudaSuccess) return e;
    dim3 grid((a.L + TILE - 1) / TILE, a.B * a.H);
    entmax_fwd_kernel<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(mq, mk, a, o);
    return cudaGetLastError();
}

}  // namespace entmax
