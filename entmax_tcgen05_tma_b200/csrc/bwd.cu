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

using P = Pipe<128, 4, 4, 2>;  // 128-key blocks, 4-deep ring, 4 TMEM buffers, 2 epilogue warpgroups
using PipeCtl = P::Ctl;
constexpr int BLK = P::BLK, NSTAGE = P::NSTAGE, NBUF = P::NBUF, NUM_EPI_WG = P::NUM_EPI_WG;
constexpr int NUM_EPI = P::NUM_EPI, NUM_THREADS = P::NUM_THREADS, NUM_WARPS = P::NUM_WARPS;
constexpr int WARP_PRODUCER = P::WARP_PRODUCER, WARP_MMA = P::WARP_MMA;
constexpr int BLK_BYTES = P::BLK_BYTES, TMEM_COLS = P::TMEM_COLS, MAX_BLOCKS = P::MAX_BLOCKS;
constexpr int STAGE_FLOATS = NUM_EPI * 32;  // per-thread staging of one 32-value chunk

constexpr int CAP = 128;              // support entries per row (or key), split between the warpgroups
constexpr int CAPW = CAP / NUM_EPI_WG;

constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + TILE_BYTES;
constexpr int OFF_CV = OFF_B + NSTAGE * BLK_BYTES;     // float [CAP][TILE]: sp
constexpr int OFF_CJ = OFF_CV + CAP * TILE * 4;        // u16   [CAP][TILE]: partner index
constexpr int OFF_STAGE = OFF_CJ + CAP * TILE * 2;     // float [NUM_EPI][32]
constexpr int OFF_BITS = OFF_STAGE + STAGE_FLOATS * 4; // u32   [MASK_WORDS]
constexpr int OFF_BLK = OFF_BITS + MASK_WORDS * 4;     // u16   [MAX_BLOCKS]
constexpr int OFF_CNT = OFF_BLK + MAX_BLOCKS * 2;      // int   [NUM_EPI_WG][TILE]: entries (-1: redo)
constexpr int OFF_TBUF = OFF_CNT + NUM_EPI_WG * TILE * 4;  // float [NBUF][TILE]: column thresholds
constexpr int OFF_RED = OFF_TBUF + NBUF * TILE * 4;    // float [NUM_THREADS]
constexpr int OFF_FLAGS = OFF_RED + NUM_THREADS * 4;   // u32   [TILE/32] rows (keys) redone on CUDA cores
constexpr int OFF_CTL = OFF_FLAGS + 16;
constexpr int SMEM_USED = OFF_CTL + (int)sizeof(PipeCtl);
constexpr int SMEM_BYTES = SMEM_USED + 1024;
constexpr int OFF_SCRATCH = 0;                          // reused after the S pass
constexpr int SCRATCH_FLOATS = OFF_CV / 4;
static_assert(CAP * TILE <= SCRATCH_FLOATS, "dA scratch must fit the S-pass buffers");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// Named barrier among the 4 warps of epilogue warpgroup g (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void wg_sync(int g) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(128) : "memory");
}

struct ListState {
    int n;
    int ovf;
};

// Lists support entry (partner idx, sp) and prefetches into L2 the two rows its gather will read.
__device__ __forceinline__ void push_entry(ListState& st, float sp, int idx, float* cv, uint16_t* cj, int r,
                                           const __nv_bfloat16* X1, const __nv_bfloat16* X2) {
    if (st.n == CAPW) {
        st.ovf = 1;
        return;
    }
    cv[st.n * TILE + r] = sp;
    cj[st.n * TILE + r] = (uint16_t)idx;
    ++st.n;
    prefetch_l2(X1 + (size_t)idx * HEAD_DIM);
    prefetch_l2(X2 + (size_t)idx * HEAD_DIM);
}

__device__ __forceinline__ float block_sum(float a, float* red) {
    a = warp_sum(a);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = a;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < NUM_WARPS; ++w) s += red[w];
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
    constexpr int PH = NUM_THREADS / HEAD_DIM;
    const int d = tid % HEAD_DIM, ph = tid / HEAD_DIM;
    float acc = 0.f;
    for (int e = ph; e < span; e += PH) {
        const float ds = sbuf[e];
        if (ds != 0.f) acc = fmaf(ds, __bfloat162float(K[head + (size_t)(lo + e) * HEAD_DIM + d]), acc);
    }
    __syncthreads();
    red[tid] = acc;
    __syncthreads();
    if (tid < HEAD_DIM) {
        float q = 0.f;
#pragma unroll
        for (int p = 0; p < PH; ++p) q += red[tid + p * HEAD_DIM];
        io.dQ[head + (size_t)i * HEAD_DIM + tid] = a.scale * q;
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
    constexpr int PH = NUM_THREADS / HEAD_DIM;
    const int d = tid % HEAD_DIM, ph = tid / HEAD_DIM;
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
        for (int e = ph; e < cn; e += PH) {
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
    if (tid < HEAD_DIM) {
#pragma unroll
        for (int p = 0; p < PH; ++p) k_out += red[tid + p * HEAD_DIM];
    }
    __syncthreads();
    red[tid] = accV;
    __syncthreads();
    if (tid < HEAD_DIM) {
        float v_out = 0.f;
#pragma unroll
        for (int p = 0; p < PH; ++p) v_out += red[tid + p * HEAD_DIM];
        io.dK[head + (size_t)j * HEAD_DIM + tid] = a.scale * k_out;
        io.dV[head + (size_t)j * HEAD_DIM + tid] = v_out;
    }
    __syncthreads();
}

struct Smem {
    uint8_t* a;
    uint8_t* b;
    float* cv;
    uint16_t* cj;
    float* stage;
    uint32_t* bits;
    uint16_t* blk;
    int* cnt;
    float* tbuf;
    float* red;
    uint32_t* redo;
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
    m.stage = reinterpret_cast<float*>(s + OFF_STAGE);
    m.bits = reinterpret_cast<uint32_t*>(s + OFF_BITS);
    m.blk = reinterpret_cast<uint16_t*>(s + OFF_BLK);
    m.cnt = reinterpret_cast<int*>(s + OFF_CNT);
    m.tbuf = reinterpret_cast<float*>(s + OFF_TBUF);
    m.red = reinterpret_cast<float*>(s + OFF_RED);
    m.redo = reinterpret_cast<uint32_t*>(s + OFF_FLAGS);
    m.scratch = reinterpret_cast<float*>(s + OFF_SCRATCH);
    m.ctl = reinterpret_cast<PipeCtl*>(s + OFF_CTL);
    return m;
}

__device__ __forceinline__ void setup_cta(const Smem& sm, const CUtensorMap* ma, const CUtensorMap* mb) {
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        P::init(sm.ctl);
        prefetch_tmap(ma);
        prefetch_tmap(mb);
    }
    if (tid < TILE / 32) sm.redo[tid] = 0u;
    if (warp == WARP_PRODUCER) {
        tmem_alloc(smem_u32(&sm.ctl->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
}

__device__ __forceinline__ void finish_cta(const Smem& sm) {
    tc_fence_before();
    __syncthreads();
    // Past this barrier no thread waits, so the abort flag is final (uniform).  After an abort every
    // TMA load and MMA issued must complete before the CTA frees TMEM and its shared memory.
    if (P::aborted(sm.ctl)) {
        const int warp = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) {
            if (warp == WARP_PRODUCER) P::drain_loads(sm.ctl);
            if (warp == WARP_MMA) P::drain_mma(sm.ctl);
        }
        tc_fence_before();
        __syncthreads();
    }
    if ((threadIdx.x >> 5) == WARP_PRODUCER) {
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
    if (warp == 0) {
        const int i_last = min(i0 + TILE - 1, L - 1);
        const int klo = a.window > 0 ? max(0, i0 - a.window + 1) : 0;
        const int khi = a.causal ? i_last : L - 1;
        const int nb = P::build_block_list(sm.blk, sm.bits, klo, khi, i0, i_last, a.causal, a.window);
        if (lane == 0) ctl->nblk = nb;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const float scale = a.scale;
    const int r = tid & (TILE - 1), g = tid >> 7;  // epilogue row and warpgroup
    ListState st{0, 0};
    if (warp == WARP_PRODUCER) {
        // [B, H, L, 64] tensors (this path takes layout 0 only)
        const HeadRef hr{0, bh / a.H, bh % a.H, a.H, a.L};
        if (lane == 0) P::producer(ctl, wc, &map_q, &map_k, hr, i0, sm.blk, sm.a, sm.b, ctl->nblk, hr);
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0) P::mma(ctl, wc, sm.a, sm.b, ctl->nblk);
        __syncwarp();
    } else {
        const int i = i0 + r;
        int rlo, rhi;
        row_key_range(i, L, a.causal, a.window, rlo, rhi);
        const float tau = i < L ? io.tau[(size_t)bh * L + i] : INFINITY;
        const float t = tau / scale;  // raw-score threshold: support iff raw score > t
        const float half_scale = 0.5f * scale;
        const __nv_bfloat16* Vh = reinterpret_cast<const __nv_bfloat16*>(a.V) + (size_t)bh * L * HEAD_DIM;
        const __nv_bfloat16* Kh = reinterpret_cast<const __nv_bfloat16*>(a.K) + (size_t)bh * L * HEAD_DIM;
        float* pcv = sm.cv + g * CAPW * TILE;
        uint16_t* pcj = sm.cj + g * CAPW * TILE;
        const int nblk = ctl->nblk;
        for (int n = g; n < nblk; n += NUM_EPI_WG) {
            if (!P::wait_scores(ctl, wc, n)) break;
            const int j0 = (int)(sm.blk[n] & ~FULL_BLOCK) * BLK;
            const bool full = (sm.blk[n] & FULL_BLOCK) && i < L;
            P::for_each_chunk(ctl, n, [&](const float (&cur)[32], int c) {
                const int jc = j0 + c * 32;
                const uint32_t vm = full ? 0xffffffffu
                                         : (jc < L && i < L) ? (sm.bits[jc >> 5] & range_bits(jc, rlo, rhi)) : 0u;
                uint32_t hits = hit_bits(cur, t) & __brev(vm);
                if (hits) {
                    stage_chunk(sm.stage, threadIdx.x % NUM_EPI, cur);
                    do {
                        const int k = __clz(hits);
                        hits &= ~(0x80000000u >> k);
                        push_entry(st, half_scale * (staged(sm.stage, threadIdx.x % NUM_EPI, k) - t), jc + k, pcv, pcj, r, Vh, Kh);
                    } while (hits);
                }
            });
        }
        sm.cnt[g * TILE + r] = st.ovf ? 0 : st.n;
        if (st.ovf) atomicOr(&sm.redo[r >> 5], 1u << (r & 31));
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool aborted = P::aborted(ctl);

    if (!aborted) {
        const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
        const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.V);
        const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
        const size_t head = (size_t)bh * L * HEAD_DIM;
        float* dAbuf = sm.scratch;  // [CAP][TILE], same slots as the entry lists
        for (int rr = warp; rr < TILE; rr += NUM_WARPS) {
            const int i = i0 + rr;
            const int k0 = sm.cnt[rr], k1 = sm.cnt[TILE + rr];
            if (i >= L || ((sm.redo[rr >> 5] >> (rr & 31)) & 1u)) continue;
            const uint32_t gw = reinterpret_cast<const uint32_t*>(dO + head + (size_t)i * HEAD_DIM)[lane];
            const float g0 = bf16lo(gw), g1 = bf16hi(gw);
            // dA_e = <dO_i, V_j> for every entry, eight gathered rows in flight
            float rs = 0.f, ws = 0.f;
            for (int q = 0; q < NUM_EPI_WG; ++q) {
                const int base = q * CAPW, end = base + (q == 0 ? k0 : k1);
                for (int e = base; e < end; e += 8) {
                    uint32_t x[8];
                    float pd[8];
#pragma unroll
                    for (int u8 = 0; u8 < 8; ++u8) {
                        const bool ok = e + u8 < end;
                        const int j = ok ? (int)sm.cj[(e + u8) * TILE + rr] : 0;
                        x[u8] = ok ? __ldg(reinterpret_cast<const uint32_t*>(V + head + (size_t)j * HEAD_DIM) + lane) : 0u;
                    }
#pragma unroll
                    for (int u8 = 0; u8 < 8; ++u8) pd[u8] = fmaf(g0, bf16lo(x[u8]), g1 * bf16hi(x[u8]));
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                        for (int u8 = 0; u8 < 8; ++u8) pd[u8] += __shfl_xor_sync(0xffffffffu, pd[u8], o);
                    }
#pragma unroll
                    for (int u8 = 0; u8 < 8; ++u8) {
                        if (e + u8 < end) {
                            const float sp = sm.cv[(e + u8) * TILE + rr];
                            rs += sp;
                            ws = fmaf(sp, pd[u8], ws);
                            if (lane == 0) dAbuf[(e + u8) * TILE + rr] = pd[u8];
                        }
                    }
                }
            }
            const float u = rs > 0.f ? ws / rs : 0.f;
            __syncwarp();
            // dS_e = sp_e (dA_e - u), written over dA, then dQ_i = scale sum_e dS_e K_j
            for (int q = 0; q < NUM_EPI_WG; ++q) {
                const int base = q * CAPW, end = base + (q == 0 ? k0 : k1);
                for (int e = base + lane; e < end; e += 32)
                    dAbuf[e * TILE + rr] = sm.cv[e * TILE + rr] * (dAbuf[e * TILE + rr] - u);
            }
            __syncwarp();
            float q0 = 0.f, q1 = 0.f, q2 = 0.f, q3 = 0.f;
            gather_accumulate2(K + head, sm.cj, dAbuf, rr, 0, k0, rr, CAPW, CAPW + k1, lane, q0, q1, q2, q3);
            q0 += q2;
            q1 += q3;
            *reinterpret_cast<float2*>(io.dQ + head + (size_t)i * HEAD_DIM + 2 * lane) =
                make_float2(scale * q0, scale * q1);
            if (lane == 0) io.u[(size_t)bh * L + i] = u;
        }
    }
    __syncthreads();
    if (!aborted) {
        for (int wd = 0; wd < TILE / 32; ++wd) {
            uint32_t mask = sm.redo[wd];  // uniform across the CTA
            while (mask) {
                const int rr = wd * 32 + __ffs(mask) - 1;
                mask &= mask - 1;
                rows_fallback(a, io, sm.bits, sm.scratch, sm.red, bh, i0 + rr);
            }
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
    const int r = tid & (TILE - 1), g = tid >> 7;  // epilogue key and warpgroup
    ListState st{0, 0};
    if (warp == WARP_PRODUCER) {
        const HeadRef hr{0, bh / a.H, bh % a.H, a.H, a.L};
        if (lane == 0) P::producer(ctl, wc, &map_k, &map_q, hr, j0, sm.blk, sm.a, sm.b, ctl->nblk, hr);
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0) P::mma(ctl, wc, sm.a, sm.b, ctl->nblk);
        __syncwarp();
    } else {
        const int j = j0 + r;
        const bool key_ok = j < L && ((sm.bits[j >> 5] >> (j & 31)) & 1u);
        int qlo, qhi;
        col_query_range(j, L, a.causal, a.window, qlo, qhi);
        const float half_scale = 0.5f * scale;
        const __nv_bfloat16* dOh = reinterpret_cast<const __nv_bfloat16*>(io.dO) + (size_t)bh * L * HEAD_DIM;
        const __nv_bfloat16* Qh = reinterpret_cast<const __nv_bfloat16*>(a.Q) + (size_t)bh * L * HEAD_DIM;
        float* pcv = sm.cv + g * CAPW * TILE;
        uint16_t* pcj = sm.cj + g * CAPW * TILE;
        const int nblk = ctl->nblk;
        bool live = true;  // each warpgroup runs all its iterations so its named-barrier counts match
        for (int n = g; n < nblk; n += NUM_EPI_WG) {
            const int q0 = (int)sm.blk[n] * BLK;
            float* tb = sm.tbuf + (n % NBUF) * TILE;
            {
                const int i = q0 + r;
                tb[r] = i < L ? io.tau[(size_t)bh * L + i] / scale : INFINITY;
            }
            wg_sync(g);
            if (live) live = P::wait_scores(ctl, wc, n);
            if (!live) continue;
            P::for_each_chunk(ctl, n, [&](const float (&cur)[32], int c) {
                const int qc = q0 + c * 32;
                const uint32_t vm = key_ok ? range_bits(qc, qlo, qhi) : 0u;
                float t[32];
#pragma unroll
                for (int k4 = 0; k4 < 8; ++k4) {
                    const float4 t4 = reinterpret_cast<const float4*>(tb + c * 32)[k4];
                    t[4 * k4] = t4.x;
                    t[4 * k4 + 1] = t4.y;
                    t[4 * k4 + 2] = t4.z;
                    t[4 * k4 + 3] = t4.w;
                }
                uint32_t hits = hit_bits(cur, t) & __brev(vm);
                if (hits) {
                    stage_chunk(sm.stage, threadIdx.x % NUM_EPI, cur);
                    do {
                        const int k = __clz(hits);
                        hits &= ~(0x80000000u >> k);
                        push_entry(st, half_scale * (staged(sm.stage, threadIdx.x % NUM_EPI, k) - tb[c * 32 + k]), qc + k, pcv, pcj, r, dOh, Qh);
                    } while (hits);
                }
            });
        }
        sm.cnt[g * TILE + r] = st.ovf ? 0 : st.n;
        if (st.ovf) atomicOr(&sm.redo[r >> 5], 1u << (r & 31));
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool aborted = P::aborted(ctl);

    if (!aborted) {
        const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
        const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.V);
        const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
        const size_t head = (size_t)bh * L * HEAD_DIM;
        for (int rr = warp; rr < TILE; rr += NUM_WARPS) {
            const int j = j0 + rr;
            const int k0 = sm.cnt[rr], k1 = sm.cnt[TILE + rr];
            if (j >= L || ((sm.redo[rr >> 5] >> (rr & 31)) & 1u)) continue;
            const uint32_t vw = reinterpret_cast<const uint32_t*>(V + head + (size_t)j * HEAD_DIM)[lane];
            const float v0 = bf16lo(vw), v1 = bf16hi(vw);
            float kk0 = 0.f, kk1 = 0.f, w0 = 0.f, w1 = 0.f;
            const float* ub = io.u + (size_t)bh * L;
            for (int q = 0; q < NUM_EPI_WG; ++q) {
                const int base = q * CAPW, end = base + (q == 0 ? k0 : k1);
                for (int e = base; e < end; e += 8) {
                    uint32_t gw[8], qw[8];
                    float uu[8], sp[8], pd[8];
#pragma unroll
                    for (int u8 = 0; u8 < 8; ++u8) {
                        const bool ok = e + u8 < end;
                        const int i = ok ? (int)sm.cj[(e + u8) * TILE + rr] : 0;
                        sp[u8] = ok ? sm.cv[(e + u8) * TILE + rr] : 0.f;
                        gw[u8] = ok ? __ldg(reinterpret_cast<const uint32_t*>(dO + head + (size_t)i * HEAD_DIM) + lane) : 0u;
                        qw[u8] = ok ? __ldg(reinterpret_cast<const uint32_t*>(Q + head + (size_t)i * HEAD_DIM) + lane) : 0u;
                        uu[u8] = ok ? __ldg(ub + i) : 0.f;
                    }
#pragma unroll
                    for (int u8 = 0; u8 < 8; ++u8) pd[u8] = fmaf(bf16lo(gw[u8]), v0, bf16hi(gw[u8]) * v1);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                        for (int u8 = 0; u8 < 8; ++u8) pd[u8] += __shfl_xor_sync(0xffffffffu, pd[u8], o);
                    }
#pragma unroll
                    for (int u8 = 0; u8 < 8; ++u8) {
                        const float ds = sp[u8] * (pd[u8] - uu[u8]);
                        const float p = sp[u8] * sp[u8];
                        w0 = fmaf(p, bf16lo(gw[u8]), w0);
                        w1 = fmaf(p, bf16hi(gw[u8]), w1);
                        kk0 = fmaf(ds, bf16lo(qw[u8]), kk0);
                        kk1 = fmaf(ds, bf16hi(qw[u8]), kk1);
                    }
                }
            }
            *reinterpret_cast<float2*>(io.dK + head + (size_t)j * HEAD_DIM + 2 * lane) = make_float2(scale * kk0, scale * kk1);
            *reinterpret_cast<float2*>(io.dV + head + (size_t)j * HEAD_DIM + 2 * lane) = make_float2(w0, w1);
        }
    }
    __syncthreads();
    if (!aborted) {
        for (int wd = 0; wd < TILE / 32; ++wd) {
            uint32_t mask = sm.redo[wd];  // uniform across the CTA
            while (mask) {
                const int rr = wd * 32 + __ffs(mask) - 1;
                mask &= mask - 1;
                keys_fallback(a, io, sm.scratch, sm.red, bh, j0 + rr);
            }
        }
    }
    finish_cta(sm);
}

}  // namespace

size_t bwd_rows_smem_bytes() { return SMEM_BYTES; }
size_t bwd_keys_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_bwd(const AttnArgs& a, const BwdIO& io, cudaStream_t stream) {
    CUtensorMap mq, mk;
    cudaError_t e = make_tile_map(&mq, a.Q, 0, a.B, a.H, a.L, TILE);
    if (e != cudaSuccess) return e;
    e = make_tile_map(&mk, a.K, 0, a.B, a.H, a.L, BLK);
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
