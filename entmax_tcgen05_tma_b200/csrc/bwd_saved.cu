// bwd_saved.cu -- backward pass of alpha-entmax attention from the forward's saved supports.
//
// Same closed-form Jacobian as bwd.cu (page "svd-sst2-roberta-adasplash", section 2.4):
//   dA_ij = dO_i . V_j,  sp_ij = sqrt(p_ij),  u_i = sum_j sp_ij dA_ij / sum_j sp_ij,
//   dS_ij = sp_ij (dA_ij - u_i),  dQ_i = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i,
//   dV_j = sum_i p_ij dO_i.
// General alpha (p = b^(1/am1), b = am1 (S - tau), am1 = alpha - 1; the pages' entmax_bisect
// routine): the Jacobian has the same form with the weight w_ij = p_ij^(2 - alpha) = b^(1/am1 - 1) in
// place of sp_ij (at alpha 1.5, w = b = sqrt(p)).  The saved lists hold b_ij in both cases.
// The supports {(j, b_ij)} come from the training forward (or, for a backward given tau alone, from
// the support extraction of fwd.cu), so these kernels form no QK^T: their work is proportional to
// the number of support entries.
//
//  1. key_scan:   per head, exclusive scan of the per-key support counts -> bucket offsets.
//  2. rows:       four query rows per warp, eight lanes per row (each lane owns eight dimensions, so
//                 a gathered row is one 16-byte load per lane): dA_ij, u_i, dS_ij, dQ_i, and the
//                 entries (i, sp_ij, dS_ij) scattered into per-key buckets.
//  3. keys:       four keys per warp, eight lanes per key: dK_j and dV_j from its bucket (gathered
//                 Q_i, dO_i rows).
//  4. unsaved:    rows whose support was not saved (redone on CUDA cores in the forward, or with more
//                 than SAVE_CAP entries) are recomputed exactly by a whole CTA each; their dK/dV terms
//                 are added with atomics after step 3.
// Summation order inside a bucket follows the fill order, so dK and dV may differ in the last bits
// from run to run; dQ does not.
#include <cuda_bf16.h>
#include <math.h>
#include "common.cuh"
#include "internal.h"

namespace entmax {
namespace {

constexpr int ROW_WARPS = 8;  // warps per CTA of the rows / keys kernels

// Whether the support-list backward must do nothing: the forward that wrote its lists in the same
// call gave up (a recorded device error), so the lists may hold anything.
__device__ __forceinline__ bool guarded(const int* guard) { return guard && *(volatile const int*)guard != 0; }

__global__ void __launch_bounds__(1024) key_scan_kernel(const int* __restrict__ key_cnt, int* __restrict__ key_off,
                                                        int* __restrict__ key_cur, int L, const int* guard) {
    if (guarded(guard)) return;
    __shared__ int wsum[32];
    const size_t base = (size_t)blockIdx.x * L;
    const int per = (L + 1023) / 1024;
    const int begin = min(L, (int)threadIdx.x * per), end = min(L, begin + per);
    int sum = 0;
    for (int j = begin; j < end; ++j) sum += key_cnt[base + j];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = wsum[lane];
        int inc = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        wsum[lane] = inc - v;
    }
    __syncthreads();
    int run = wsum[warp] + incl - sum;
    for (int j = begin; j < end; ++j) {
        key_off[base + j] = run;
        run += key_cnt[base + j];
        key_cur[base + j] = 0;
    }
}

constexpr int RPW = 4;  // rows (keys) per warp: eight lanes each, lane s of a group owns dimensions 8s .. 8s+7

__device__ __forceinline__ void unpack8(const uint4& x, float (&v)[8]) {
    const uint32_t u[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = bf16lo(u[k]);
        v[2 * k + 1] = bf16hi(u[k]);
    }
}

// Sum over the eight lanes of a group (lanes 8q .. 8q + 7).
__device__ __forceinline__ float group8_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    return v;
}

// Gathered 128-byte rows: lane sd's 16-byte piece of row j, at x + j * step elements.
struct GlobalRows {
    const __nv_bfloat16* x;  // row 0
    size_t step;             // elements from one row to the next
    __device__ __forceinline__ uint4 get(size_t j, int sd) const {
        return __ldg(reinterpret_cast<const uint4*>(x + j * step) + sd);
    }
};
// The same with consecutive rows (step 64, a shift).
struct DenseRows {
    const __nv_bfloat16* x;
    __device__ __forceinline__ uint4 get(size_t j, int sd) const {
        return __ldg(reinterpret_cast<const uint4*>(x + j * HEAD_DIM) + sd);
    }
};
// One query row per group of eight lanes (lane sd owns dimensions 8 sd .. 8 sd + 7), row list
// staged in shared memory (mj, msp; mds holds dA, then dS).  dA_e = dO_i . V_je with one 16-byte
// piece of V_je per lane and a three-step group reduction, two entries in flight; then u_i, dS_e,
// the bucket entries, and dQ_i (one 16-byte piece of K_je per lane per entry).  cnt < 0: no row, or
// a row the exact pass handles.
// GEN: general alpha, weights w = b^em1 (em1 = 1/am1 - 1) and p = w b; the buckets then hold p
// instead of b.
// qmem: memory row of query row `row` in Q, dO and dQ (layout); bucket entries name it by qmem.
// PLAIN (layout 0): qmem is row itself and is not used.
template <bool GEN, bool PLAIN, class Rows>
__device__ __forceinline__ void rows_group(const AttnArgs& a, const BwdIO& io, const SavedSupport& sv,
                                           const SavedBwdWs& ws, long long row, size_t qmem_, int cnt, int bhk,
                                           const Rows& Vr, const Rows& Kr, uint16_t* mj, float* msp, float* mds,
                                           int sd, float em1) {
    const size_t qmem = PLAIN ? (size_t)row : qmem_;
    const int L = a.L;
    const size_t cap = (size_t)(a.H / a.Hkv) * L * SAVE_CAP;  // bucket entries of one KV head
    const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
    for (int e = sd; e < cnt; e += 8) {
        mj[e] = sv.row_j[(size_t)row * SAVE_CAP + e];
        msp[e] = sv.row_sp[(size_t)row * SAVE_CAP + e];
    }
    float g[8];
    {
        const uint4 x = cnt >= 0 ? __ldg(reinterpret_cast<const uint4*>(dO + qmem * HEAD_DIM) + sd)
                                 : make_uint4(0u, 0u, 0u, 0u);
        unpack8(x, g);
    }
    const int maxc = __reduce_max_sync(0xffffffffu, max(cnt, 0));
    __syncwarp();
    // dA_e, two entries in flight
    for (int e = 0; e < maxc; e += 2) {
        uint4 x[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const bool ok = e + u < cnt;
            x[u] = ok ? Vr.get(mj[e + u], sd) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float v[8];
            unpack8(x[u], v);
            float part = 0.f;
#pragma unroll
            for (int d = 0; d < 8; ++d) part = fmaf(g[d], v[d], part);
            part = group8_sum(part);
            if (sd == 0 && e + u < cnt) mds[e + u] = part;
        }
    }
    __syncwarp();
    // u_i = sum w dA / sum w over the row's entries (w = sp at alpha 1.5)
    float r1 = 0.f, w1 = 0.f;
    for (int e = sd; e < cnt; e += 8) {
        const float w = GEN ? pow_pos(msp[e], em1) : msp[e];
        r1 += w;
        w1 = fmaf(w, mds[e], w1);
    }
    r1 = group8_sum(r1);
    w1 = group8_sum(w1);
    const float uu = r1 > 0.f ? w1 / r1 : 0.f;
    __syncwarp();
    // dS_e, and (i, sp, dS) into key j's bucket
    for (int e = sd; e < cnt; e += 8) {
        const float sp = msp[e];
        const float w = GEN ? pow_pos(sp, em1) : sp;
        const float ds = w * (mds[e] - uu);
        mds[e] = ds;
        const size_t key = (size_t)bhk * L + mj[e];
        const size_t at = (size_t)bhk * cap + (size_t)ws.key_off[key] + (size_t)atomicAdd(ws.key_cur + key, 1);
        ws.bucket_i[at] = (uint32_t)qmem;
        ws.bucket_sp[at] = GEN ? w * sp : sp;
        ws.bucket_ds[at] = ds;
    }
    __syncwarp();
    // dQ_i = scale sum_e dS_e K_je, two entries in flight
    float acc[8];
#pragma unroll
    for (int d = 0; d < 8; ++d) acc[d] = 0.f;
    for (int e = 0; e < maxc; e += 2) {
        uint4 x[2];
        float dsv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const bool ok = e + u < cnt;
            dsv[u] = ok ? mds[e + u] : 0.f;
            x[u] = ok ? Kr.get(mj[e + u], sd) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float v[8];
            unpack8(x[u], v);
#pragma unroll
            for (int d = 0; d < 8; ++d) acc[d] = fmaf(dsv[u], v[d], acc[d]);
        }
    }
    if (cnt >= 0) {
        float4* dst = reinterpret_cast<float4*>(io.dQ + qmem * HEAD_DIM + 8 * sd);
        dst[0] = make_float4(a.scale * acc[0], a.scale * acc[1], a.scale * acc[2], a.scale * acc[3]);
        dst[1] = make_float4(a.scale * acc[4], a.scale * acc[5], a.scale * acc[6], a.scale * acc[7]);
    }
    __syncwarp();  // the lists are rewritten for the next rows
}

// One key per group of eight lanes: dK_j = scale sum dS Q_i and dV_j = sum p dO_i over key j's bucket,
// lane sd of the group loading entry e0 + sd and the group sharing it by shuffles; two entries (two
// 16-byte pieces each per lane) in flight.  valid = false: no key (the group still takes part).
// key: logical key row (bhk * L + j); kmem: its memory row in K, V, dK and dV (layout; PLAIN, i.e.
// layout 0: key).
// SPLIT groups of eight lanes share one key (grouped-query heads make its bucket SPLIT-fold longer):
// group `sub` takes every SPLIT-th run of eight entries, and the partial sums are added across the
// groups (lane groups 8q .. 8q + 7 with q = key slot * SPLIT + sub) before group 0 writes.
template <bool GEN, bool PLAIN, int SPLIT, class Rows>
__device__ __forceinline__ void keys_group(const AttnArgs& a, const BwdIO& io, const SavedSupport& sv,
                                           const SavedBwdWs& ws, long long key, size_t kmem_, bool valid, int bhk,
                                           const Rows& Qr, const Rows& Gr, int sd, int g0, int sub) {
    const size_t kmem = PLAIN ? (size_t)key : kmem_;
    const int L = a.L;
    const size_t cap = (size_t)(a.H / a.Hkv) * L * SAVE_CAP;  // bucket entries of one KV head
    const int n = valid ? sv.key_cnt[key] : 0;
    const size_t b0 = (size_t)bhk * cap + (size_t)(valid ? ws.key_off[key] : 0);
    const int maxn = __reduce_max_sync(0xffffffffu, n);
    float ak[8], av[8];
#pragma unroll
    for (int d = 0; d < 8; ++d) ak[d] = av[d] = 0.f;
    // every group runs the same number of steps (the shuffles below take all 32 lanes); group sub
    // reads entries e0 + 8 sub .. e0 + 8 sub + 7 of each step
    for (int e00 = 0; e00 < maxn; e00 += 8 * SPLIT) {
        const int e0 = e00 + 8 * sub;
        const bool mine = e0 + sd < n;
        const uint32_t ei = mine ? ws.bucket_i[b0 + e0 + sd] : 0u;
        const float esp = mine ? ws.bucket_sp[b0 + e0 + sd] : 0.f;
        const float eds = mine ? ws.bucket_ds[b0 + e0 + sd] : 0.f;
#pragma unroll
        for (int t = 0; t < 8; t += 2) {
            uint4 xg[2], xq[2];
            float pv[2], dv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int src = g0 | (t + u);
                const uint32_t it = __shfl_sync(0xffffffffu, ei, src);
                const float st = __shfl_sync(0xffffffffu, esp, src);
                const float dt = __shfl_sync(0xffffffffu, eds, src);
                const bool ok = e0 + t + u < n;
                pv[u] = ok ? (GEN ? st : st * st) : 0.f;  // p_ij
                dv[u] = ok ? dt : 0.f;
                xg[u] = ok ? Gr.get(it, sd) : make_uint4(0u, 0u, 0u, 0u);
                xq[u] = ok ? Qr.get(it, sd) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float vg[8], vq[8];
                unpack8(xg[u], vg);
                unpack8(xq[u], vq);
#pragma unroll
                for (int d = 0; d < 8; ++d) {
                    av[d] = fmaf(pv[u], vg[d], av[d]);
                    ak[d] = fmaf(dv[u], vq[d], ak[d]);
                }
            }
        }
    }
#pragma unroll
    for (int o = 8; o < 8 * SPLIT; o <<= 1) {
#pragma unroll
        for (int d = 0; d < 8; ++d) {
            ak[d] += __shfl_xor_sync(0xffffffffu, ak[d], o);
            av[d] += __shfl_xor_sync(0xffffffffu, av[d], o);
        }
    }
    if (valid && sub == 0) {
        float4* dk = reinterpret_cast<float4*>(io.dK + kmem * HEAD_DIM + 8 * sd);
        float4* dv4 = reinterpret_cast<float4*>(io.dV + kmem * HEAD_DIM + 8 * sd);
        dk[0] = make_float4(a.scale * ak[0], a.scale * ak[1], a.scale * ak[2], a.scale * ak[3]);
        dk[1] = make_float4(a.scale * ak[4], a.scale * ak[5], a.scale * ak[6], a.scale * ak[7]);
        dv4[0] = make_float4(av[0], av[1], av[2], av[3]);
        dv4[1] = make_float4(av[4], av[5], av[6], av[7]);
    }
}

// Four query rows per warp (eight lanes each), rows of K and V gathered from L2.  PLAIN: layout 0,
// where memory rows are the logical row ids and rows of one head are consecutive.
template <bool GEN, bool PLAIN>
__global__ void __launch_bounds__(ROW_WARPS * 32) saved_rows_kernel(const AttnArgs a, const BwdIO io,
                                                                    const SavedSupport sv, const SavedBwdWs ws) {
    if (guarded(io.guard)) return;
    __shared__ uint16_t lj[ROW_WARPS][RPW][SAVE_CAP];
    __shared__ float lsp[ROW_WARPS][RPW][SAVE_CAP];
    __shared__ float lds[ROW_WARPS][RPW][SAVE_CAP];  // dA, then dS
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = lane >> 3, sd = lane & 7;
    const int L = a.L;
    const long long R = (long long)a.B * a.H * L;
    const float em1 = 1.f / a.am1 - 1.f;
    for (long long grp = (long long)blockIdx.x * ROW_WARPS + warp; grp * RPW < R; grp += (long long)gridDim.x * ROW_WARPS) {
        const long long row = grp * RPW + q;
        const int cnt = row < R ? sv.row_cnt[row] : -1;
        const int bh = row < R ? (int)(row / L) : 0;
        if (PLAIN) {
            const int bhk = kv_head_of(bh, a.H, a.Hkv);
            const size_t head = (size_t)bhk * L * HEAD_DIM;
            const DenseRows Vr{reinterpret_cast<const __nv_bfloat16*>(a.V) + head};
            const DenseRows Kr{reinterpret_cast<const __nv_bfloat16*>(a.K) + head};
            rows_group<GEN, true>(a, io, sv, ws, row, 0, cnt, bhk, Vr, Kr, lj[warp][q], lsp[warp][q], lds[warp][q],
                                  sd, em1);
        } else {
            const int b = bh / a.H, i = (int)(row - (long long)bh * L);
            const int bhk = kv_head_of(bh, a.H, a.Hkv);
            const HeadRef hq{a.layout, b, bh - b * a.H, a.H, L}, hkv{a.layout, b, bhk - b * a.Hkv, a.Hkv, L};
            const size_t head = hkv.row(0) * HEAD_DIM, step = hkv.step() * HEAD_DIM;
            const GlobalRows Vr{reinterpret_cast<const __nv_bfloat16*>(a.V) + head, step};
            const GlobalRows Kr{reinterpret_cast<const __nv_bfloat16*>(a.K) + head, step};
            rows_group<GEN, false>(a, io, sv, ws, row, hq.row(i), cnt, bhk, Vr, Kr, lj[warp][q], lsp[warp][q],
                                   lds[warp][q], sd, em1);
        }
    }
}

// 4 / SPLIT keys per warp (8 SPLIT lanes each), rows of Q and dO gathered from L2.  PLAIN as for
// the rows.
template <bool GEN, bool PLAIN, int SPLIT>
__global__ void __launch_bounds__(ROW_WARPS * 32) saved_keys_kernel(const AttnArgs a, const BwdIO io,
                                                                    const SavedSupport sv, const SavedBwdWs ws) {
    static_assert(SPLIT == 1 || SPLIT == 2 || SPLIT == 4, "lane groups per key");
    if (guarded(io.guard)) return;
    constexpr int KPW = RPW / SPLIT;  // keys per warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = lane >> 3, sd = lane & 7, g0 = lane & ~7;
    const int kq = q / SPLIT, sub = q % SPLIT;
    const int L = a.L;
    const long long Rk = (long long)a.B * a.Hkv * L;  // keys
    // bucket entries name their query row by its memory row, so Q and dO are read from the base
    const DenseRows Qr{reinterpret_cast<const __nv_bfloat16*>(a.Q)};
    const DenseRows Gr{reinterpret_cast<const __nv_bfloat16*>(io.dO)};
    for (long long grp = (long long)blockIdx.x * ROW_WARPS + warp; grp * KPW < Rk; grp += (long long)gridDim.x * ROW_WARPS) {
        const long long key = grp * KPW + kq;
        const bool kv = key < Rk;
        const int bhk = kv ? (int)(key / L) : 0;
        size_t kmem = 0;
        if (!PLAIN) {
            const int b = bhk / a.Hkv;
            const HeadRef hkv{a.layout, b, bhk - b * a.Hkv, a.Hkv, L};
            kmem = hkv.row((int)(key - (long long)bhk * L));
        }
        keys_group<GEN, PLAIN, SPLIT>(a, io, sv, ws, key, kmem, kv, bhk, Qr, Gr, sd, g0, sub);
    }
}

constexpr int UNSAVED_THREADS = 256;

__device__ __forceinline__ float block_sum256(float v, float* red) {
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < UNSAVED_THREADS / 32; ++w) s += red[w];
    return s;
}

__device__ __forceinline__ float dot64_f32(const float* a, const __nv_bfloat16* row) {
    const uint4* p = reinterpret_cast<const uint4*>(row);
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 w = __ldg(p + c);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            acc = fmaf(a[c * 8 + 2 * t], bf16lo(ws[t]), acc);
            acc = fmaf(a[c * 8 + 2 * t + 1], bf16hi(ws[t]), acc);
        }
    }
    return acc;
}

// Rows whose support was not saved: recomputed exactly by one CTA each (scores on CUDA cores), dQ_i
// stored, dK/dV contributions added with atomics (this kernel runs after saved_keys_kernel).
template <bool GEN>
__global__ void __launch_bounds__(UNSAVED_THREADS) unsaved_rows_kernel(const AttnArgs a, const BwdIO io,
                                                                      const SavedSupport sv) {
    if (guarded(io.guard)) return;
    extern __shared__ float sbuf[];  // [L]: b_ij = am1 (S_ij - tau_i) (sqrt(p_ij) at alpha 1.5); [L, 2L): dA_ij
    const float am1 = a.am1, em1 = 1.f / am1 - 1.f;
    __shared__ float red[UNSAVED_THREADS];
    __shared__ float qf[HEAD_DIM], gf[HEAD_DIM];
    const int tid = threadIdx.x;
    const int L = a.L;
    const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
    const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
    const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.V);
    const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
    const int n_unsaved = *sv.unsaved_cnt;
    for (int idx = blockIdx.x; idx < n_unsaved; idx += gridDim.x) {
        const long long row = sv.unsaved_rows[idx];
        const long long bh = row / L;
        const int i = (int)(row - bh * L);
        const int b = (int)(bh / a.H);
        const int bhk = kv_head_of((int)bh, a.H, a.Hkv);
        const HeadRef hq{a.layout, b, (int)bh - b * a.H, a.H, L};            // rows of Q, dO, dQ
        const HeadRef hkv{a.layout, b, bhk - b * a.Hkv, a.Hkv, L};          // rows of K, V, dK, dV
        const size_t qmem = hq.row(i);
        __syncthreads();
        if (tid < HEAD_DIM) {
            qf[tid] = __bfloat162float(Q[qmem * HEAD_DIM + tid]);
            gf[tid] = __bfloat162float(dO[qmem * HEAD_DIM + tid]);
        }
        __syncthreads();
        const float tau = io.tau[row];
        int lo, hi;
        row_key_range(i, L, a.causal, a.window, lo, hi);
        const int span = hi - lo + 1;
        float r = 0.f, w = 0.f;
        for (int e = tid; e < span; e += UNSAVED_THREADS) {
            const int j = lo + e;
            float sp = 0.f;
            if (!a.key_mask || a.key_mask[(size_t)b * L + j]) {
                const float s = a.scale * dot64_f32(qf, K + hkv.row(j) * HEAD_DIM);
                sp = fmaxf((GEN ? am1 : 0.5f) * (s - tau), 0.f);
            }
            float dA = 0.f;
            if (sp > 0.f) {
                dA = dot64_f32(gf, V + hkv.row(j) * HEAD_DIM);
                const float wt = GEN ? pow_pos(sp, em1) : sp;
                r += wt;
                w = fmaf(wt, dA, w);
            }
            sbuf[e] = sp;
            sbuf[L + e] = dA;
        }
        const float rs = block_sum256(r, red);
        const float ws = block_sum256(w, red);
        const float u = rs > 0.f ? ws / rs : 0.f;
        __syncthreads();
        constexpr int PH = UNSAVED_THREADS / HEAD_DIM;
        const int d = tid % HEAD_DIM, ph = tid / HEAD_DIM;
        float acc = 0.f;
        for (int e = ph; e < span; e += PH) {
            const float sp = sbuf[e];
            if (sp > 0.f) {
                const size_t key = hkv.row(lo + e);  // memory row of K, V, dK, dV
                const float wt = GEN ? pow_pos(sp, em1) : sp;
                const float ds = wt * (sbuf[L + e] - u);
                acc = fmaf(ds, __bfloat162float(K[key * HEAD_DIM + d]), acc);
                atomicAdd(io.dK + key * HEAD_DIM + d, a.scale * ds * qf[d]);
                atomicAdd(io.dV + key * HEAD_DIM + d, wt * sp * gf[d]);
            }
        }
        __syncthreads();
        red[tid] = acc;
        __syncthreads();
        if (tid < HEAD_DIM) {
            float q = 0.f;
#pragma unroll
            for (int p = 0; p < PH; ++p) q += red[tid + p * HEAD_DIM];
            io.dQ[qmem * HEAD_DIM + tid] = a.scale * q;
        }
    }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t saved_support_bytes(long long R) {
    return align256(R * 4) + align256(R * SAVE_CAP * 2) + align256(R * SAVE_CAP * 4) + align256(R * 4) + 256 +
           align256(R * 4);
}

SavedSupport carve_saved(void* base, long long R) {
    uint8_t* p = static_cast<uint8_t*>(base);
    SavedSupport s;
    s.row_cnt = reinterpret_cast<int*>(p);
    p += align256(R * 4);
    s.row_j = reinterpret_cast<uint16_t*>(p);
    p += align256(R * SAVE_CAP * 2);
    s.row_sp = reinterpret_cast<float*>(p);
    p += align256(R * SAVE_CAP * 4);
    s.key_cnt = reinterpret_cast<int*>(p);
    p += align256(R * 4);
    s.unsaved_cnt = reinterpret_cast<int*>(p);
    p += 256;
    s.unsaved_rows = reinterpret_cast<int*>(p);
    return s;
}

size_t saved_bwd_ws_bytes(long long R) {
    return 2 * align256(R * 4) + align256(R * SAVE_CAP * 4) * 3;
}

SavedBwdWs carve_saved_bwd_ws(void* base, long long R) {
    uint8_t* p = static_cast<uint8_t*>(base);
    SavedBwdWs w;
    w.key_off = reinterpret_cast<int*>(p);
    p += align256(R * 4);
    w.key_cur = reinterpret_cast<int*>(p);
    p += align256(R * 4);
    w.bucket_i = reinterpret_cast<uint32_t*>(p);
    p += align256(R * SAVE_CAP * 4);
    w.bucket_sp = reinterpret_cast<float*>(p);
    p += align256(R * SAVE_CAP * 4);
    w.bucket_ds = reinterpret_cast<float*>(p);
    return w;
}

cudaError_t launch_bwd_saved(const AttnArgs& a, const BwdIO& io, const SavedSupport& sv, const SavedBwdWs& ws,
                             cudaStream_t stream) {
    const long long R = (long long)a.B * a.H * a.L;
    key_scan_kernel<<<a.B * a.Hkv, 1024, 0, stream>>>(sv.key_cnt, ws.key_off, ws.key_cur, a.L, io.guard);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>((R + ROW_WARPS - 1) / ROW_WARPS, (long long)sms * 8));
    const bool gen = generic_alpha(a);
    const bool plain = a.layout == 0;  // memory rows = logical row ids
    if (gen) {
        if (plain) saved_rows_kernel<true, true><<<grid, ROW_WARPS * 32, 0, stream>>>(a, io, sv, ws);
        else saved_rows_kernel<true, false><<<grid, ROW_WARPS * 32, 0, stream>>>(a, io, sv, ws);
    } else {
        if (plain) saved_rows_kernel<false, true><<<grid, ROW_WARPS * 32, 0, stream>>>(a, io, sv, ws);
        else saved_rows_kernel<false, false><<<grid, ROW_WARPS * 32, 0, stream>>>(a, io, sv, ws);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long Rk = (long long)a.B * a.Hkv * a.L;
    // lane groups per key: grouped-query buckets hold H / H_kv query heads' entries
    const int rep_heads = a.H / a.Hkv, split = rep_heads >= 4 ? 4 : rep_heads >= 2 ? 2 : 1;
    const long long kwarps = (Rk * split + RPW - 1) / RPW;
    const unsigned kgrid = (unsigned)std::max<long long>(1, std::min<long long>((kwarps + ROW_WARPS - 1) / ROW_WARPS, (long long)sms * 8));
    // one instantiation per (generic alpha, layout 0, lane groups per key)
    using KeysFn = void (*)(const AttnArgs, const BwdIO, const SavedSupport, const SavedBwdWs);
    static const KeysFn keys_fns[2][2][3] = {
        {{saved_keys_kernel<false, false, 1>, saved_keys_kernel<false, false, 2>, saved_keys_kernel<false, false, 4>},
         {saved_keys_kernel<false, true, 1>, saved_keys_kernel<false, true, 2>, saved_keys_kernel<false, true, 4>}},
        {{saved_keys_kernel<true, false, 1>, saved_keys_kernel<true, false, 2>, saved_keys_kernel<true, false, 4>},
         {saved_keys_kernel<true, true, 1>, saved_keys_kernel<true, true, 2>, saved_keys_kernel<true, true, 4>}}};
    keys_fns[gen][plain][split == 4 ? 2 : split - 1]<<<kgrid, ROW_WARPS * 32, 0, stream>>>(a, io, sv, ws);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int smem = 2 * a.L * (int)sizeof(float);
    const void* ufn = gen ? reinterpret_cast<const void*>(unsaved_rows_kernel<true>)
                          : reinterpret_cast<const void*>(unsaved_rows_kernel<false>);
    e = ensure_smem_attr(ufn, 2 * MAX_L * (int)sizeof(float), gen ? 5 : 3);
    if (e != cudaSuccess) return e;
    if (gen) unsaved_rows_kernel<true><<<(unsigned)sms, UNSAVED_THREADS, smem, stream>>>(a, io, sv);
    else unsaved_rows_kernel<false><<<(unsigned)sms, UNSAVED_THREADS, smem, stream>>>(a, io, sv);
    return cudaGetLastError();
}

}  // namespace entmax
