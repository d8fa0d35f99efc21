// bwd.cu -- backward pass of 1.5-entmax attention on sm_100a.
//
// Closed-form Jacobian of page "svd-sst2-roberta-adasplash", section 2.4 (restated in the
// model card "roberta-base-adasplash", section 2): with sp_ij = sqrt(p_ij) = [(S_ij - tau_i)/2]_+
// and the upstream gradient dA_ij = dL/dp_ij = dO_i . V_j,
//   dS_ij = sp_ij (dA_ij - u_i),    u_i = sum_j sp_ij dA_ij / sum_j sp_ij,
//   dQ_i = scale sum_j dS_ij K_j,   dK_j = scale sum_i dS_ij Q_i,   dV_j = sum_i p_ij dO_i.
// Zero gradient off the support.
//
// Two kernels, no atomics:
//  * rows kernel  (one CTA per 128 queries): S = Q K^T recomputed on tcgen05 with the forward's
//    exact MMA order, so {S_ij > tau_i} is the forward's support bit for bit.  Each epilogue
//    thread lists its row's support; then one warp per row forms dA by gathered dot products,
//    u_i, dS and dQ_i.  u_i goes to the workspace.
//  * keys kernel  (one CTA per 128 keys): S^T = K Q^T on tcgen05 (TMEM lane = key), each thread
//    lists the queries whose support holds its key (threshold tau_i per column), then one warp
//    per key accumulates dK_j and dV_j from gathered Q_i, dO_i rows.
// A row (or key) with more than CAP support entries is redone by the whole CTA on CUDA cores.
#include <cuda_bf16.h>
#include <math.h>
#include "common.cuh"
#include "internal.h"

namespace entmax {
namespace {

constexpr int CAP = 128;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + TILE_BYTES;
constexpr int OFF_CV = OFF_B + NSTAGE * BLK_BYTES;     // float [CAP][TILE]: sp
constexpr int OFF_CJ = OFF_CV + CAP * TILE * 4;        // u16   [CAP][TILE]: partner index
constexpr int OFF_BITS = OFF_CJ + CAP * TILE * 2;      // u32   [MASK_WORDS]
constexpr int OFF_BLK = OFF_BITS + MASK_WORDS * 4;     // u16   [MAX_BLOCKS]
constexpr int OFF_CNT = OFF_BLK + MAX_BLOCKS * 2;      // int   [TILE]: entries (-1: redo)
constexpr int OFF_TBUF = OFF_CNT + TILE * 4;           // float [2][TILE]: column thresholds
constexpr int OFF_RED = OFF_TBUF + 2 * TILE * 4;       // float [256]
constexpr int OFF_CTL = OFF_RED + 256 * 4;
constexpr int SMEM_USED = OFF_CTL + (int)sizeof(PipeCtl);
constexpr int SMEM_BYTES = SMEM_USED + 1024;
constexpr int OFF_SCRATCH = 0;                          // reused after the S pass
constexpr int SCRATCH_FLOATS = OFF_CV / 4;
static_assert(CAP * TILE <= SCRATCH_FLOATS, "dA scratch must fit the S-pass buffers");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

constexpr int EPI_BARRIER = 1;  // named barrier among the 4 epilogue warps

__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(EPI_BARRIER), "n"(128) : "memory");
}

struct ListState {
    int n;
    int ovf;
};

__device__ __forceinline__ void push_entry(ListState& st, float sp, int idx, float* cv, uint16_t* cj, int r) {
    if (st.n == CAP) {
        st.ovf = 1;
        return;
    }
    cv[st.n * TILE + r] = sp;
    cj[st.n * TILE + r] = (uint16_t)idx;
    ++st.n;
}

__device__ __forceinline__ float block_sum(float a, float* red) {
    a = warp_sum(a);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = a;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < NUM_THREADS / 32; ++w) s += red[w];
    return s;
}

__device__ __forceinline__ void load_row_f32(const __nv_bfloat16* src, float* dst) {
    // 64 bf16 -> 64 floats, by threads 0..63 of the CTA
    if (threadIdx.x < HEAD_DIM) dst[threadIdx.x] = __bfloat162float(src[threadIdx.x]);
}

__device__ __forceinline__ float dot64_f32_bf16(const float* a, const __nv_bfloat16* row) {
    const uint4* p = reinterpret_cast<const uint4*>(row);
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 w = p[c];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            acc = fmaf(a[c * 8 + 2 * t], bf16lo(ws[t]), acc);
            acc = fmaf(a[c * 8 + 2 * t + 1], bf16hi(ws[t]), acc);
        }
    }
    return acc;
}

// Whole-CTA exact redo of one query row: dQ_i and u_i on CUDA cores.
__device__ __noinline__ void rows_fallback(const AttnArgs& a, const BwdIO& io, const uint32_t* bits, float* sbuf,
                                           float* red, int bh, int i) {
    const int tid = threadIdx.x;
    const int L = a.L;
    const size_t head = (size_t)bh * L * HEAD_DIM;
    const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
    const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
    const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.V);
    const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
    float* qf = red + 64;
    float* gf = red + 128;
    __syncthreads();
    load_row_f32(Q + head + (size_t)i * HEAD_DIM, qf);
    if (tid >= 64 && tid < 128) gf[tid - 64] = __bfloat162float(dO[head + (size_t)i * HEAD_DIM + tid - 64]);
    __syncthreads();
    const float tau = io.tau[(size_t)bh * L + i];
    int lo, hi;
    row_key_range(i, L, a.causal, a.window, lo, hi);
    const int span = hi - lo + 1;
    float r = 0.f, w = 0.f;
    for (int e = tid; e < span; e += NUM_THREADS) {
        const int j = lo + e;
        float sp = 0.f;
        if ((bits[j >> 5] >> (j & 31)) & 1u) {
            const float s = a.scale * dot64_f32_bf16(qf, K + head + (size_t)j * HEAD_DIM);
            sp = fmaxf(0.5f * (s - tau), 0.f);
        }
        if (sp > 0.f) {
            const float dA = dot64_f32_bf16(gf, V + head + (size_t)j * HEAD_DIM);
            r += sp;
            w = fmaf(sp, dA, w);
        }
        sbuf[e] = sp;
    }
    const float rs = block_sum(r, red);
    const float ws = block_sum(w, red);
    const float u = rs > 0.f ? ws / rs : 0.f;
    for (int e = tid; e < span; e += NUM_THREADS) {
        const float sp = sbuf[e];
        if (sp > 0.f) sbuf[e] = sp * (dot64_f32_bf16(gf, V + head + (size_t)(lo + e) * HEAD_DIM) - u);
    }
    __syncthreads();
    const int d = tid & (HEAD_DIM - 1), ph = tid >> 6;
    float acc = 0.f;
    for (int e = ph; e < span; e += NUM_THREADS / HEAD_DIM) {
        const float ds = sbuf[e];
        if (ds != 0.f) acc = fmaf(ds, __bfloat162float(K[head + (size_t)(lo + e) * HEAD_DIM + d]), acc);
    }
    __syncthreads();
    red[tid] = acc;
    __syncthreads();
    if (tid < HEAD_DIM) {
        io.dQ[head + (size_t)i * HEAD_DIM + tid] = a.scale * (red[tid] + red[tid + 64] + red[tid + 128] + red[tid + 192]);
        if (tid == 0) io.u[(size_t)bh * L + i] = u;
    }
    __syncthreads();
}

// Whole-CTA exact redo of one key: dK_j and dV_j on CUDA cores, queries in chunks.
__device__ __noinline__ void keys_fallback(const AttnArgs& a, const BwdIO& io, float* sbuf, float* red, int bh,
                                           int j) {
    const int tid = threadIdx.x;
    const int L = a.L;
    const size_t head = (size_t)bh * L * HEAD_DIM;
    const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
    const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
    const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.V);
    const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
    float* kf = red + 64;
    float* vf = red + 128;
    __syncthreads();
    load_row_f32(K + head + (size_t)j * HEAD_DIM, kf);
    if (tid >= 64 && tid < 128) vf[tid - 64] = __bfloat162float(V[head + (size_t)j * HEAD_DIM + tid - 64]);
    __syncthreads();
    int qlo, qhi;
    col_query_range(j, L, a.causal, a.window, qlo, qhi);
    const int d = tid & (HEAD_DIM - 1), ph = tid >> 6;
    float accK = 0.f, accV = 0.f;
    constexpr int CHUNK = SCRATCH_FLOATS / 2;
    float* pbuf = sbuf;           // p_ij
    float* dsbuf = sbuf + CHUNK;  // dS_ij
    for (int c0 = qlo; c0 <= qhi; c0 += CHUNK) {
        const int cn = min(CHUNK, qhi - c0 + 1);
        for (int e = tid; e < cn; e += NUM_THREADS) {
            const int i = c0 + e;
            const float s = a.scale * dot64_f32_bf16(kf, Q + head + (size_t)i * HEAD_DIM);
            const float sp = fmaxf(0.5f * (s - io.tau[(size_t)bh * L + i]), 0.f);
            float ds = 0.f;
            if (sp > 0.f) ds = sp * (dot64_f32_bf16(vf, dO + head + (size_t)i * HEAD_DIM) - io.u[(size_t)bh * L + i]);
            pbuf[e] = sp * sp;
            dsbuf[e] = ds;
        }
        __syncthreads();
        for (int e = ph; e < cn; e += NUM_THREADS / HEAD_DIM) {
            const float p = pbuf[e];
            if (p > 0.f) {
                const size_t row = head + (size_t)(c0 + e) * HEAD_DIM + d;
                accV = fmaf(p, __bfloat162float(dO[row]), accV);
                accK = fmaf(dsbuf[e], __bfloat162float(Q[row]), accK);
            }
        }
        __syncthreads();
    }
    red[tid] = accK;
    __syncthreads();
    float k_out = 0.f;
    if (tid < HEAD_DIM) k_out = red[tid] + red[tid + 64] + red[tid + 128] + red[tid + 192];
    __syncthreads();
    red[tid] = accV;
    __syncthreads();
    if (tid < HEAD_DIM) {
        io.dK[head + (size_t)j * HEAD_DIM + tid] = a.scale * k_out;
        io.dV[head + (size_t)j * HEAD_DIM + tid] = red[tid] + red[tid + 64] + red[tid + 128] + red[tid + 192];
    }
    __syncthreads();
}

struct Smem {
    uint8_t* a;
    uint8_t* b;
    float* cv;
    uint16_t* cj;
    uint32_t* bits;
    uint16_t* blk;
    int* cnt;
    float* tbuf;
    float* red;
    float* scratch;
    PipeCtl* ctl;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
    uint8_t* s = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    Smem m;
    m.a = s + OFF_A;
    m.b = s + OFF_B;
    m.cv = reinterpret_cast<float*>(s + OFF_CV);
    m.cj = reinterpret_cast<uint16_t*>(s + OFF_CJ);
    m.bits = reinterpret_cast<uint32_t*>(s + OFF_BITS);
    m.blk = reinterpret_cast<uint16_t*>(s + OFF_BLK);
    m.cnt = reinterpret_cast<int*>(s + OFF_CNT);
    m.tbuf = reinterpret_cast<float*>(s + OFF_TBUF);
    m.red = reinterpret_cast<float*>(s + OFF_RED);
    m.scratch = reinterpret_cast<float*>(s + OFF_SCRATCH);
    m.ctl = reinterpret_cast<PipeCtl*>(s + OFF_CTL);
    return m;
}

__device__ __forceinline__ void setup_cta(const Smem& sm, const CUtensorMap* ma, const CUtensorMap* mb) {
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        init_pipe(sm.ctl);
        prefetch_tmap(ma);
        prefetch_tmap(mb);
    }
    if (warp == 4) {
        tmem_alloc(smem_u32(&sm.ctl->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
}

__device__ __forceinline__ void finish_cta(const Smem& sm) {
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 4) {
        tc_fence_after();
        tmem_dealloc(sm.ctl->tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ rows kernel
__global__ void __launch_bounds__(NUM_THREADS, 1)
entmax_bwd_rows_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                       const AttnArgs a, const BwdIO io) {
    extern __shared__ uint8_t smem_raw[];
    const Smem sm = carve(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.L, tile = blockIdx.x, bh = blockIdx.y, b = bh / a.H;
    const int i0 = tile * TILE;
    const WaitCfg wc{a.status, a.timeout_ns};
    PipeCtl* ctl = sm.ctl;

    setup_cta(sm, &map_q, &map_k);
    build_key_bitmap(sm.bits, a.key_mask, b, L);
    __syncthreads();
    if (tid == 0) {
        const int i_last = min(i0 + TILE - 1, L - 1);
        int klo = 0, khi = L - 1;
        if (a.window > 0) klo = max(0, i0 - a.window + 1);
        if (a.causal) khi = i_last;
        int nb = 0;
        for (int kb = klo / BLK; kb <= khi / BLK; ++kb) {
            bool any = false;
            for (int w = kb * (BLK / 32); w < (kb + 1) * (BLK / 32) && w * 32 <= khi; ++w)
                any |= (sm.bits[w] & range_bits(w * 32, klo, khi)) != 0u;
            if (any) sm.blk[nb++] = (uint16_t)kb;
        }
        ctl->nblk = nb;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const float scale = a.scale;
    ListState st{0, 0};
    if (warp == 4) {
        if (lane == 0) role_producer(ctl, wc, &map_q, &map_k, bh, i0, sm.blk, sm.a, sm.b);
        __syncwarp();
    } else if (warp == 5) {
        if (lane == 0) role_mma(ctl, wc, sm.a, sm.b);
        __syncwarp();
    } else if (warp < 4) {
        const int r = tid, i = i0 + r;
        int rlo, rhi;
        row_key_range(i, L, a.causal, a.window, rlo, rhi);
        const float tau = i < L ? io.tau[(size_t)bh * L + i] : INFINITY;
        const float t = tau / scale;  // raw-score threshold
        const float half_scale = 0.5f * scale;
        const uint32_t lane_base = ctl->tmem_base + ((uint32_t)(warp * 32) << 16);
        const int nblk = ctl->nblk;
        for (int n = 0; n < nblk; ++n) {
            if (!epi_wait_scores(ctl, wc, n)) break;
            const int j0 = (int)sm.blk[n] * BLK;
#pragma unroll 1
            for (int c = 0; c < BLK / 32; ++c) {
                float v[32];
                tmem_ld32(lane_base + (uint32_t)((n & 1) * BLK + c * 32), v);
                tmem_wait_ld();
                if (c == BLK / 32 - 1) epi_release_scores(ctl, n);
                const int jc = j0 + c * 32;
                const uint32_t vm = (jc < L && i < L) ? (sm.bits[jc >> 5] & range_bits(jc, rlo, rhi)) : 0u;
                if (vm == 0xffffffffu) {
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (v[k] > t) push_entry(st, half_scale * (v[k] - t), jc + k, sm.cv, sm.cj, r);
                } else if (vm != 0u) {
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (((vm >> k) & 1u) && v[k] > t) push_entry(st, half_scale * (v[k] - t), jc + k, sm.cv, sm.cj, r);
                }
            }
        }
        sm.cnt[r] = st.ovf ? -1 : st.n;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool aborted = cta_aborted(ctl);

    if (!aborted) {
        const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
        const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.V);
        const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
        const size_t head = (size_t)bh * L * HEAD_DIM;
        float* dAbuf = sm.scratch;  // [CAP][TILE]
        for (int r = warp; r < TILE; r += NUM_THREADS / 32) {
            const int i = i0 + r;
            const int k = sm.cnt[r];
            if (i >= L || k < 0) continue;
            const uint32_t gw = reinterpret_cast<const uint32_t*>(dO + head + (size_t)i * HEAD_DIM)[lane];
            const float g0 = bf16lo(gw), g1 = bf16hi(gw);
            float rs = 0.f, ws = 0.f;
            int e = 0;
            for (; e + 2 <= k; e += 2) {
                const int ja = sm.cj[e * TILE + r], jb = sm.cj[(e + 1) * TILE + r];
                const uint32_t va = reinterpret_cast<const uint32_t*>(V + head + (size_t)ja * HEAD_DIM)[lane];
                const uint32_t vb = reinterpret_cast<const uint32_t*>(V + head + (size_t)jb * HEAD_DIM)[lane];
                float da = fmaf(g0, bf16lo(va), g1 * bf16hi(va));
                float db = fmaf(g0, bf16lo(vb), g1 * bf16hi(vb));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    da += __shfl_xor_sync(0xffffffffu, da, o);
                    db += __shfl_xor_sync(0xffffffffu, db, o);
                }
                const float spa = sm.cv[e * TILE + r], spb = sm.cv[(e + 1) * TILE + r];
                rs += spa + spb;
                ws = fmaf(spa, da, fmaf(spb, db, ws));
                if (lane == 0) {
                    dAbuf[e * TILE + r] = da;
                    dAbuf[(e + 1) * TILE + r] = db;
                }
            }
            if (e < k) {
                const int ja = sm.cj[e * TILE + r];
                const uint32_t va = reinterpret_cast<const uint32_t*>(V + head + (size_t)ja * HEAD_DIM)[lane];
                const float da = warp_sum(fmaf(g0, bf16lo(va), g1 * bf16hi(va)));
                const float spa = sm.cv[e * TILE + r];
                rs += spa;
                ws = fmaf(spa, da, ws);
                if (lane == 0) dAbuf[e * TILE + r] = da;
            }
            const float u = rs > 0.f ? ws / rs : 0.f;
            __syncwarp();
            float q0 = 0.f, q1 = 0.f;
            for (e = 0; e < k; ++e) {
                const int j = sm.cj[e * TILE + r];
                const float ds = sm.cv[e * TILE + r] * (dAbuf[e * TILE + r] - u);
                const uint32_t kw = reinterpret_cast<const uint32_t*>(K + head + (size_t)j * HEAD_DIM)[lane];
                q0 = fmaf(ds, bf16lo(kw), q0);
                q1 = fmaf(ds, bf16hi(kw), q1);
            }
            *reinterpret_cast<float2*>(io.dQ + head + (size_t)i * HEAD_DIM + 2 * lane) =
                make_float2(scale * q0, scale * q1);
            if (lane == 0) io.u[(size_t)bh * L + i] = u;
        }
    }
    __syncthreads();
    if (!aborted) {
        for (int r = 0; r < TILE; ++r) {
            if (sm.cnt[r] >= 0) continue;
            rows_fallback(a, io, sm.bits, sm.scratch, sm.red, bh, i0 + r);
        }
    }
    finish_cta(sm);
}

// ------------------------------------------------------------------ keys kernel
__global__ void __launch_bounds__(NUM_THREADS, 1)
entmax_bwd_keys_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                       const AttnArgs a, const BwdIO io) {
    extern __shared__ uint8_t smem_raw[];
    const Smem sm = carve(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.L, tile = blockIdx.x, bh = blockIdx.y, b = bh / a.H;
    const int j0 = tile * TILE;
    const WaitCfg wc{a.status, a.timeout_ns};
    PipeCtl* ctl = sm.ctl;

    setup_cta(sm, &map_k, &map_q);
    build_key_bitmap(sm.bits, a.key_mask, b, L);
    __syncthreads();
    if (tid == 0) {
        const int j_last = min(j0 + TILE - 1, L - 1);
        bool any_key = false;
        for (int w = j0 / 32; w <= j_last / 32; ++w) any_key |= (sm.bits[w] & range_bits(w * 32, j0, j_last)) != 0u;
        int nb = 0;
        if (any_key) {
            const int qlo = a.causal ? j0 : 0;
            const int qhi = a.window > 0 ? min(L - 1, j_last + a.window - 1) : L - 1;
            for (int qb = qlo / BLK; qb <= qhi / BLK; ++qb) sm.blk[nb++] = (uint16_t)qb;
        }
        ctl->nblk = nb;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const float scale = a.scale;
    ListState st{0, 0};
    if (warp == 4) {
        if (lane == 0) role_producer(ctl, wc, &map_k, &map_q, bh, j0, sm.blk, sm.a, sm.b);
        __syncwarp();
    } else if (warp == 5) {
        if (lane == 0) role_mma(ctl, wc, sm.a, sm.b);
        __syncwarp();
    } else if (warp < 4) {
        const int r = tid, j = j0 + r;
        const bool key_ok = j < L && ((sm.bits[j >> 5] >> (j & 31)) & 1u);
        int qlo, qhi;
        col_query_range(j, L, a.causal, a.window, qlo, qhi);
        const float half_scale = 0.5f * scale;
        const uint32_t lane_base = ctl->tmem_base + ((uint32_t)(warp * 32) << 16);
        const int nblk = ctl->nblk;
        bool live = true;  // every epilogue warp runs all nblk iterations: the named barrier counts match
        for (int n = 0; n < nblk; ++n) {
            const int q0 = (int)sm.blk[n] * BLK;
            float* tb = sm.tbuf + (n & 1) * TILE;
            {
                const int i = q0 + r;
                tb[r] = i < L ? io.tau[(size_t)bh * L + i] / scale : INFINITY;
            }
            epi_sync();
            if (live) live = epi_wait_scores(ctl, wc, n);
            if (!live) continue;
#pragma unroll 1
            for (int c = 0; c < BLK / 32; ++c) {
                float v[32];
                tmem_ld32(lane_base + (uint32_t)((n & 1) * BLK + c * 32), v);
                tmem_wait_ld();
                if (c == BLK / 32 - 1) epi_release_scores(ctl, n);
                const int qc = q0 + c * 32;
                const uint32_t vm = key_ok ? range_bits(qc, qlo, qhi) : 0u;
                if (vm == 0u) continue;
                float t[32];
#pragma unroll
                for (int k4 = 0; k4 < 8; ++k4) {
                    const float4 t4 = reinterpret_cast<const float4*>(tb + c * 32)[k4];
                    t[4 * k4] = t4.x;
                    t[4 * k4 + 1] = t4.y;
                    t[4 * k4 + 2] = t4.z;
                    t[4 * k4 + 3] = t4.w;
                }
#pragma unroll
                for (int k = 0; k < 32; ++k)
                    if (((vm >> k) & 1u) && v[k] > t[k]) push_entry(st, half_scale * (v[k] - t[k]), qc + k, sm.cv, sm.cj, r);
            }
        }
        sm.cnt[r] = st.ovf ? -1 : st.n;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool aborted = cta_aborted(ctl);

    if (!aborted) {
        const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
        const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.V);
        const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
        const size_t head = (size_t)bh * L * HEAD_DIM;
        for (int r = warp; r < TILE; r += NUM_THREADS / 32) {
            const int j = j0 + r;
            const int k = sm.cnt[r];
            if (j >= L || k < 0) continue;
            const uint32_t vw = reinterpret_cast<const uint32_t*>(V + head + (size_t)j * HEAD_DIM)[lane];
            const float v0 = bf16lo(vw), v1 = bf16hi(vw);
            float k0 = 0.f, k1 = 0.f, w0 = 0.f, w1 = 0.f;
            for (int e = 0; e < k; ++e) {
                const int i = sm.cj[e * TILE + r];
                const float sp = sm.cv[e * TILE + r];
                const uint32_t gw = reinterpret_cast<const uint32_t*>(dO + head + (size_t)i * HEAD_DIM)[lane];
                const uint32_t qw = reinterpret_cast<const uint32_t*>(Q + head + (size_t)i * HEAD_DIM)[lane];
                const float g0 = bf16lo(gw), g1 = bf16hi(gw);
                const float dA = warp_sum(fmaf(g0, v0, g1 * v1));
                const float ds = sp * (dA - io.u[(size_t)bh * L + i]);
                const float p = sp * sp;
                w0 = fmaf(p, g0, w0);
                w1 = fmaf(p, g1, w1);
                k0 = fmaf(ds, bf16lo(qw), k0);
                k1 = fmaf(ds, bf16hi(qw), k1);
            }
            *reinterpret_cast<float2*>(io.dK + head + (size_t)j * HEAD_DIM + 2 * lane) = make_float2(scale * k0, scale * k1);
            *reinterpret_cast<float2*>(io.dV + head + (size_t)j * HEAD_DIM + 2 * lane) = make_float2(w0, w1);
        }
    }
    __syncthreads();
    if (!aborted) {
        for (int r = 0; r < TILE; ++r) {
            if (sm.cnt[r] >= 0) continue;
            keys_fallback(a, io, sm.scratch, sm.red, bh, j0 + r);
        }
    }
    finish_cta(sm);
}

}  // namespace

size_t bwd_rows_smem_bytes() { return SMEM_BYTES; }
size_t bwd_keys_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_bwd(const AttnArgs& a, const BwdIO& io, cudaStream_t stream) {
    CUtensorMap mq, mk;
    cudaError_t e = make_tile_map(&mq, a.Q, a.B * a.H, a.L);
    if (e != cudaSuccess) return e;
    e = make_tile_map(&mk, a.K, a.B * a.H, a.L);
    if (e != cudaSuccess) return e;
    e = ensure_smem_attr(reinterpret_cast<const void*>(entmax_bwd_rows_kernel), SMEM_BYTES, 1);
    if (e != cudaSuccess) return e;
    e = ensure_smem_attr(reinterpret_cast<const void*>(entmax_bwd_keys_kernel), SMEM_BYTES, 2);
    if (e != cudaSuccess) return e;
    dim3 grid((a.L + TILE - 1) / TILE, a.B * a.H);
    entmax_bwd_rows_kernel<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(mq, mk, a, io);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    entmax_bwd_keys_kernel<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(mk, mq, a, io);
    return cudaGetLastError();
}

}  // namespace entmax
