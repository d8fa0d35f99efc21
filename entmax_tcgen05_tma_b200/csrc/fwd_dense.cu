// fwd_dense.cu -- forward pass of 1.5-entmax attention with its products on tcgen05, for rows whose
// allowed keys span few 64-key blocks: sequences of at most 512 keys, causal windows of at most 128.
//
// Page "svd-sst2-roberta-adasplash", sections 2.2-2.3 and 3 (model cards "roberta-base-adasplash" /
// "distilbert-sst2-adasplash", the bracket [max - 2, max - 2/sqrt(n)]): S = scale Q K^T over the
// allowed keys, tau_i with sum_j [(S_ij - tau_i)/2]_+^2 = 1, P = [(S - tau)/2]_+^2, O = P V.
// On such rows a 128 x 64 tile of (query, key) pairs costs less as a tcgen05 product than as a
// gather over its support, and two CTAs share an SM where the gather forward (fwd.cu) runs one.
// One CTA per 128 queries walks the listed key blocks three times:
//   pass 1:  S = Q K^T; the epilogue takes each row's max m and the four largest maxima of its
//            32-key chunks, whose exact threshold is a lower bound of tau (a subset's threshold
//            never exceeds the row's);
//   pass 2:  S again; the scores above t = max(m - 2/scale, that bound) -- a superset of the
//            support -- go to the row's two candidate lists in shared memory (one per half row);
//   tau:     two lanes per row, candidates in registers (tau15.cuh: halvings of a sub-bracket of the
//            pages' bracket that still holds the root, stop once the support is fixed, exact
//            closed-form finish); candidates past a full list go to a spill area
//            shared by the CTA, and a row that used it is solved by a whole warp (the bisection over
//            32 lanes); only if the spill area overflows, tau comes from all of the row's scores,
//            recomputed on CUDA cores;
//   pass 3:  S again; P = [(S - tau)/2]_+^2 as bf16 hi + lo parts written back over the S columns
//            (tcgen05.st); O += P_hi V + P_lo V, A read from TMEM, the V block (M/N-major) from
//            shared memory;
//   end:     O (bf16 or fp32) and tau to HBM.
// Recomputing S costs 4 MMAs a block per pass; holding a row's scores instead would need more TMEM
// than two CTAs have.  P enters P V as two bf16 parts (P = hi + lo to about 16 significant bits), so
// O carries fp32-level accuracy.  Roles and the TMEM part layout: dense.cuh.  A row with no allowed
// key gets O = 0 and tau = +inf.  Every wait is bounded; an abort drains the CTA's own loads and
// MMAs at teardown.
#include <cuda_bf16.h>
#include <math.h>
#include "dense.cuh"
#include "internal.h"
#include "tau15.cuh"

namespace entmax {
namespace {

using namespace dense;

constexpr int NSD = 3;                               // input ring stages
constexpr int CAPD = 32;                             // candidates per row and half
constexpr int DO_Q = 0;                              // Q tile [128][64] bf16, SW128
constexpr int DO_RING = DO_Q + TILE_BYTES;           // NSD x (K block, V block)
constexpr int DO_CV = DO_RING + NSD * 2 * BLK_ROW_BYTES;  // float [2][CAPD + 1][TILE] candidate lists
constexpr int DO_BITS = DO_CV + 2 * (CAPD + 1) * TILE * 4;  // u32 [MASK_WORDS] valid keys
constexpr int DO_BLK = DO_BITS + MASK_WORDS * 4;     // u16 [MAX_L / BK] key blocks
constexpr int DO_TOP = DO_BLK + (MAX_L / BK) * 2;    // float4 [2][TILE] each half's four largest chunk maxima
constexpr int DO_CNT = DO_TOP + 2 * TILE * 16;       // int [2][TILE] each half's candidate count
constexpr int DO_ROW = DO_CNT + 2 * TILE * 4;        // float [2][TILE] the row's cut t; -tau/2
constexpr int DO_OVF = DO_ROW + 2 * TILE * 4;        // u32 [TILE / 32] rows whose lists overflowed
constexpr int NSP = 512;                             // spill entries: candidates past a full list
constexpr int DO_SPV = DO_OVF + 16;                  // float [NSP] spilled candidate values
constexpr int DO_SPR = DO_SPV + NSP * 4;             // u8 [NSP] their rows
constexpr int DO_CTL = DO_SPR + NSP;

struct FdCtl {
    uint64_t full_q;          // Q tile landed
    uint64_t full[NSD];       // K (passes 1, 2) or K, V (pass 3) block landed
    uint64_t empty[NSD];      // stage free (its last MMA completed)
    uint64_t s_full[2];       // S of a block in TMEM set 0 / 1
    uint64_t s_free[2];       // the set free again (MMA commit after its last product)
    uint64_t p_ready[2];      // epilogue done with the set: S read, P parts stored (8 warp arrivals)
    uint64_t acc_done;        // last O MMA completed
    uint32_t tmem_base;
    int abort_flag;
    int nblk;
    int nload;
    int nspill;               // spill entries claimed (may exceed NSP: then the spill area overflowed)
    uint32_t last_bar;
    uint32_t last_par;
};
constexpr int D_SMEM_BYTES = DO_CTL + (int)sizeof(FdCtl) + 1024;
static_assert(DO_RING % 1024 == 0 && BLK_ROW_BYTES % 1024 == 0, "operand alignment");
static_assert(DO_TOP % 16 == 0 && DO_CTL % 8 == 0, "alignment");
static_assert(D_SMEM_BYTES <= 113 * 1024, "two CTAs per SM");
constexpr int FB_NPL = 16;                           // a fallback row's scores per lane: 512 keys at most
static_assert(FB_NPL * 32 >= 512 && 3 * 64 >= 128 + 63, "a dense row has at most 512 allowed keys");

// The hits of a 32-value chunk (bit 31 - k <-> value k) past the first `skip` into the CTA's spill
// area, tagged with their row.  Out of line: it runs only when a row's list is full.
__device__ __noinline__ void spill_hits(const float (&v)[32], uint32_t hits, int skip, int r, int* nspill,
                                        float* spv, uint8_t* spr) {
    for (int k = 0; k < 32; ++k) {
        if (!((hits >> (31 - k)) & 1u)) continue;
        if (skip > 0) {
            --skip;
            continue;
        }
        const int q = atomicAdd(nspill, 1);
        if (q < NSP) {
            spv[q] = v[k];
            spr[q] = (uint8_t)r;
        }
    }
}

// tau (score units) of a row whose lists overflowed, from its candidates: the full lists plus its
// entries of the spill area, gathered into a warp's registers (lane l takes list entries l, l + 32
// and spill slots l + 32 q) and solved over 32 lanes.  t_cut: the cut the candidates passed.  Out
// of line: it runs only for such rows.
__device__ __noinline__ float solve_spilled_row(const float* cv, const int* cnt, const float* spv, const uint8_t* spr,
                                                int nsp, int rr, float t_cut, float scale, int lane) {
    const int m0 = min(cnt[rr], CAPD), m1 = min(cnt[TILE + rr], CAPD);
    float y[2 + NSP / 32];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int e = lane + 32 * c;
        y[c] = e < m0 ? cv[e * TILE + rr] : (e - m0 < m1 ? cv[(CAPD + 1 + e - m0) * TILE + rr] : -INFINITY);
    }
#pragma unroll
    for (int c = 0; c < NSP / 32; ++c) {
        const int q = lane + 32 * c;
        y[2 + c] = (q < nsp && spr[q] == rr) ? spv[q] : -INFINITY;
    }
    float mx = -INFINITY;
    int na = 0;
#pragma unroll
    for (int c = 0; c < 2 + NSP / 32; ++c) {
        mx = fmaxf(mx, y[c]);
        na += y[c] > -INFINITY ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        na += __shfl_xor_sync(0xffffffffu, na, o);
    }
    const float ms = scale * mx;
#pragma unroll
    for (int c = 0; c < 2 + NSP / 32; ++c) y[c] = fmaf(scale, y[c], -ms);  // -inf stays -inf
    // the candidates are the scores above the cut: a superset of the support
    const float hi = -2.f / sqrtf((float)max(na, 1));
    const float lo = fminf(fmaxf(-2.f, fmaf(scale, t_cut, -ms)), hi);
    return ms + solve_tau_warp<2 + NSP / 32>(y, lo, hi);
}

__device__ __forceinline__ float bfl(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bfh(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__global__ void __launch_bounds__(THREADS, 2)
entmax_dense_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v, const AttnArgs a, const FwdOut out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + DO_Q;
    uint8_t* ring = smem + DO_RING;
    float* cv = reinterpret_cast<float*>(smem + DO_CV);
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + DO_BITS);
    uint16_t* blk = reinterpret_cast<uint16_t*>(smem + DO_BLK);
    float4* top = reinterpret_cast<float4*>(smem + DO_TOP);
    int* cnt = reinterpret_cast<int*>(smem + DO_CNT);
    float* rowv = reinterpret_cast<float*>(smem + DO_ROW);
    uint32_t* ovf = reinterpret_cast<uint32_t*>(smem + DO_OVF);
    float* spv = reinterpret_cast<float*>(smem + DO_SPV);
    uint8_t* spr = smem + DO_SPR;
    FdCtl* ctl = reinterpret_cast<FdCtl*>(smem + DO_CTL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.L, tile = blockIdx.x, bh = blockIdx.y, b = bh / a.H;
    const int bhk = kv_head_of(bh, a.H, a.Hkv);
    const HeadRef hq{a.layout, b, bh - b * a.H, a.H, L};
    const HeadRef hkv{a.layout, b, bhk - b * a.Hkv, a.Hkv, L};
    const int i0 = tile * TILE;
    const WaitCfg wc{a.status, a.timeout_ns};

    if (tid == 0) {
        mbar_init(smem_u32(&ctl->full_q), 1);
        for (int s = 0; s < NSD; ++s) {
            mbar_init(smem_u32(&ctl->full[s]), 1);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_u32(&ctl->s_full[t]), 1);
            mbar_init(smem_u32(&ctl->s_free[t]), 1);
            mbar_init(smem_u32(&ctl->p_ready[t]), NUM_EPI / 32);
        }
        mbar_init(smem_u32(&ctl->acc_done), 1);
        ctl->abort_flag = 0;
        ctl->nload = 0;
        ctl->nspill = 0;
        ctl->last_bar = 0;
        ctl->last_par = 0;
        fence_barrier_init();
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
    }
    if (tid < TILE / 32) ovf[tid] = 0u;
    if (warp == W_PROD) {
        tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS_D);
        tmem_relinquish();
    }
    build_key_bitmap(bits, a.key_mask, b, L);
    __syncthreads();
    if (warp == 0) {
        const int i_last = min(i0 + TILE - 1, L - 1);
        const int klo = a.window > 0 ? max(0, i0 - a.window + 1) : 0;
        const int khi = a.causal ? i_last : L - 1;
        const int nb = BlockList::build_block_list(blk, bits, klo, khi, i0, i_last, a.causal, a.window);
        if (lane == 0) ctl->nblk = nb;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int nb = ctl->nblk;
    const int njobs = 3 * nb;  // job m: pass m / nb over listed block m % nb
    const uint32_t tmem = ctl->tmem_base;  // sets: S [0, 64) and [64, 128); O accumulator [128, 192)

    if (warp == W_PROD) {
        if (lane == 0) {
            mbar_arrive_expect_tx(smem_u32(&ctl->full_q), TILE_BYTES);
            tma_load_3d(smem_u32(sQ), &map_q, 0, hq.c1(i0), hq.c2(i0), smem_u32(&ctl->full_q));
            int issued = 0;
            for (int m = 0; m < njobs; ++m) {
                const int s = m % NSD;
                if (!wait_bounded(smem_u32(&ctl->empty[s]), ((uint32_t)(m / NSD) & 1u) ^ 1u, &ctl->abort_flag, wc))
                    break;
                const bool p3 = m >= 2 * nb;
                const int row = (int)(blk[m % nb] & ~FULL_BLOCK) * BK;
                uint8_t* st = ring + s * 2 * BLK_ROW_BYTES;
                mbar_arrive_expect_tx(smem_u32(&ctl->full[s]), (p3 ? 2 : 1) * BLK_ROW_BYTES);
                tma_load_3d(smem_u32(st), &map_k, 0, hkv.c1(row), hkv.c2(row), smem_u32(&ctl->full[s]));
                if (p3)
                    tma_load_3d(smem_u32(st + BLK_ROW_BYTES), &map_v, 0, hkv.c1(row), hkv.c2(row),
                                smem_u32(&ctl->full[s]));
                ++issued;
            }
            ctl->nload = issued;
        }
        __syncwarp();
    } else if (warp == W_MMA) {
        if (lane == 0) {
            constexpr uint32_t IDESC_S = umma_idesc_bf16_f32(TILE, BK);
            constexpr uint32_t IDESC_O = umma_idesc_bf16_f32_bmn(TILE, HEAD_DIM);
            uint32_t last_bar = 0, last_par = 0;
            bool ok = wait_bounded(smem_u32(&ctl->full_q), 0, &ctl->abort_flag, wc);
            const uint64_t dq = umma_desc_kmajor_sw128(smem_u32(sQ));
            if (ok) tc_fence_after();
            // job j's set is read (and, in pass 3, holds its P parts): O += P_hi V + P_lo V for a
            // pass-3 job, then release the stage and the set
            auto finish = [&](int j) -> bool {
                const int s = j % NSD, t = j & 1;
                if (!wait_bounded(smem_u32(&ctl->p_ready[t]), (uint32_t)(j >> 1) & 1u, &ctl->abort_flag, wc))
                    return false;
                tc_fence_after();
                if (j >= 2 * nb) {
                    const int n = j - 2 * nb;
                    const uint64_t vm = umma_desc_mnmajor_sw128(smem_u32(ring + s * 2 * BLK_ROW_BYTES + BLK_ROW_BYTES));
                    const uint32_t set = tmem + 64u * (uint32_t)t;
                    // 16 keys per step: hi part at column 16 k, lo part at 16 k + 8; two 8-row groups
                    // (2048 B) of the V block
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_bf16_ta(tmem + 128, set + 16 * k, vm + 128u * k, IDESC_O, (n > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_bf16_ta(tmem + 128, set + 16 * k + 8, vm + 128u * k, IDESC_O, 1u);
                }
                commit_to(&ctl->empty[s], (uint32_t)(j / NSD) & 1u, &last_bar, &last_par);
                commit_to(&ctl->s_free[t], (uint32_t)(j >> 1) & 1u, &last_bar, &last_par);
                return true;
            };
            for (int m = 0; m < njobs && ok; ++m) {
                const int s = m % NSD, t = m & 1;
                ok = wait_bounded(smem_u32(&ctl->full[s]), (uint32_t)(m / NSD) & 1u, &ctl->abort_flag, wc) &&
                     wait_bounded(smem_u32(&ctl->s_free[t]), ((uint32_t)(m >> 1) & 1u) ^ 1u, &ctl->abort_flag, wc);
                if (!ok) break;
                tc_fence_after();
                const uint64_t dk = umma_desc_kmajor_sw128(smem_u32(ring + s * 2 * BLK_ROW_BYTES));
#pragma unroll
                for (int k = 0; k < HEAD_DIM / 16; ++k)
                    tc_mma_bf16(tmem + 64u * (uint32_t)t, dq + 2u * k, dk + 2u * k, IDESC_S, k > 0 ? 1u : 0u);
                commit_to(&ctl->s_full[t], (uint32_t)(m >> 1) & 1u, &last_bar, &last_par);
                if (m > 0) ok = finish(m - 1);
            }
            if (ok && njobs > 0) ok = finish(njobs - 1);
            if (ok && nb > 0) commit_to(&ctl->acc_done, 0u, &last_bar, &last_par);
            ctl->last_bar = last_bar;
            ctl->last_par = last_par;
        }
        __syncwarp();
    } else {
        // epilogue: thread (g, r) <-> query row i0 + r <-> TMEM lane r, columns [32 g, 32 g + 32)
        const int r = tid & (TILE - 1), g = tid >> 7, i = i0 + r;
        int rlo, rhi;
        row_key_range(i, L, a.causal, a.window, rlo, rhi);
        const float scale = a.scale;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        auto trow = [&](int m) { return tmem + lane_base + 64u * (uint32_t)(m & 1) + (uint32_t)(HB * g); };
        auto allowed = [&](int e) -> uint32_t {  // bit k: key 32 g + k of listed block e allowed for row i
            const uint16_t ent = blk[e];
            const int jc = (int)(ent & ~FULL_BLOCK) * BK + HB * g;
            if ((ent & FULL_BLOCK) && i < L) return 0xffffffffu;
            return (jc < L && i < L) ? (bits[jc >> 5] & range_bits(jc, rlo, rhi)) : 0u;
        };
        auto release = [&](int m) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->p_ready[m & 1]));
        };
        // the scores of job m, this thread's 32 columns, in registers; the set goes back at once
        auto read_scores = [&](int m, float (&v)[32]) -> bool {
            if (!warp_wait_d(smem_u32(&ctl->s_full[m & 1]), (uint32_t)(m >> 1) & 1u, &ctl->abort_flag, wc)) return false;
            tc_fence_after();
            tmem_ld32(trow(m), v);
            tmem_wait_ld(v);
            release(m);
            return true;
        };
        bool live = true;

        // ---- pass 1: this half's four largest chunk maxima (a chunk = its 32 columns of a block)
        float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
        for (int n = 0; n < nb && live; ++n) {
            float v[32];
            live = read_scores(n, v);
            if (!live) break;
            const uint32_t vm = allowed(n);
            if (vm != 0xffffffffu) {
#pragma unroll
                for (int k = 0; k < 32; ++k) v[k] = ((vm >> k) & 1u) ? v[k] : -INFINITY;
            }
            const float cm = max32(v);
            a3 = fmaxf(a3, fminf(a2, cm));
            a2 = fmaxf(a2, fminf(a1, cm));
            a1 = fmaxf(a1, fminf(a0, cm));
            a0 = fmaxf(a0, cm);
        }
        top[g * TILE + r] = make_float4(a0, a1, a2, a3);
        epi_bar();
        {
            const float4 o = top[(g ^ 1) * TILE + r];
            top4_insert(o.x, a0, a1, a2, a3);
            top4_insert(o.y, a0, a1, a2, a3);
            top4_insert(o.z, a0, a1, a2, a3);
            top4_insert(o.w, a0, a1, a2, a3);
        }
        // scores at or below t are outside the support: the row max minus 2 (scaled), raised to the
        // exact threshold of the four largest chunk maxima (raw units).  t lies below the row max, so
        // a row with an allowed key has at least one candidate.
        const float t = fmaxf(a0 - 2.f / scale, top4_bound(a0, a1, a2, a3, 4.f / (scale * scale)));
        if (g == 0) rowv[r] = t;

        // ---- pass 2: candidates s > t into this half's list
        float* lst = cv + g * (CAPD + 1) * TILE + r;
        int nc = 0;
        for (int n = 0; n < nb && live; ++n) {
            float v[32];
            live = read_scores(nb + n, v);
            if (!live) break;
            const uint32_t hits = hit_bits(v, t) & __brev(allowed(n));  // bit 31 - k <-> value k
            if (__any_sync(0xffffffffu, hits != 0u)) {
                // branch-free append: every value goes to the next free slot (slot CAPD, past the
                // list, takes the writes of a full list) and the count moves on a hit only
                const int nc0 = nc;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    lst[min(nc, CAPD) * TILE] = v[k];
                    nc += (int)((hits >> (31 - k)) & 1u);
                }
                if (nc > CAPD) spill_hits(v, hits, max(0, CAPD - nc0), r, &ctl->nspill, spv, spr);  // rare
            }
        }
        cnt[g * TILE + r] = nc;
        if (nc > CAPD) atomicOr(&ovf[r >> 5], 1u << (r & 31));
        epi_bar();

        // ---- tau: two lanes per row (lane h holds the row's entries h, h + 2, ... of both lists)
        {
            const int rr = (warp << 4) | (lane >> 1), h = lane & 1;
            const int n0 = cnt[rr], n1 = cnt[TILE + rr];
            const int ii = i0 + rr;
            const bool over = (ovf[rr >> 5] >> (rr & 31)) & 1u;
            // the row max exceeds every lower bound of tau, so it is a candidate: the largest entry
            const bool solve = live && ii < L && !over && n0 + n1 > 0;
            const int ns = solve ? (n0 + n1 + 1 - h) >> 1 : 0;
            float cmax = -INFINITY;
            for (int k = 0; k < ns; ++k) {
                const int e = 2 * k + h;
                cmax = fmaxf(cmax, cv[(e < n0 ? e : CAPD + 1 + (e - n0)) * TILE + rr]);
            }
            cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
            const float ms = scale * cmax;
            const float tcut = rowv[rr];
            // bracket (scaled, shifted: row max 0): lo from the cut (g(lo) >= 1), hi = -2/sqrt(k) over
            // the k candidates, a superset of the support (g(hi) <= 1); both inside [-2, -2/sqrt(n)]
            const float hi = -2.f / sqrtf((float)max(n0 + n1, 1));
            const float lo = fminf(fmaxf(-2.f, fmaf(scale, tcut, -ms)), hi);
            const int nmax = __reduce_max_sync(0xffffffffu, ns);
            float tau_x;
            if (nmax <= 8) tau_x = solve_tau<8, CAPD + 1>(cv, rr, h, ns, n0, scale, ms, lo, hi);
            else if (nmax <= 16) tau_x = solve_tau<16, CAPD + 1>(cv, rr, h, ns, n0, scale, ms, lo, hi);
            else if (nmax <= 24) tau_x = solve_tau<24, CAPD + 1>(cv, rr, h, ns, n0, scale, ms, lo, hi);
            else tau_x = solve_tau<CAPD, CAPD + 1>(cv, rr, h, ns, n0, scale, ms, lo, hi);
            // a row with no allowed key (or past L): tau = +inf, so that every weight below is 0
            const float tau = solve ? ms + tau_x : INFINITY;
            if (h == 0 && !over) {
                rowv[TILE + rr] = -0.5f * tau;
                if (live && ii < L) out.tau[(size_t)bh * L + ii] = tau;
            }
        }

        // ---- rows whose lists overflowed, one warp per row.  Their candidates are the full lists plus
        // their entries of the spill area: gathered into the warp's registers (lane l takes list
        // entries l, l + 32 and spill slots l + 32 q), then solved as above over 32 lanes.  Only if the
        // spill area itself overflowed, tau comes from all of the row's scores, recomputed on CUDA cores.
        {
            uint32_t wm[TILE / 32];
#pragma unroll
            for (int q = 0; q < TILE / 32; ++q) wm[q] = ovf[q];
            const int nsp = ctl->nspill;
            int seen = 0;
            for (int q = 0; q < TILE / 32; ++q) {
                while (wm[q] && live) {
                    const int rr = 32 * q + (__ffs(wm[q]) - 1);
                    wm[q] &= wm[q] - 1u;
                    if ((seen++ & 7) != warp) continue;
                    const int ii = i0 + rr;
                    if (nsp <= NSP) {
                        const float tau = solve_spilled_row(cv, cnt, spv, spr, nsp, rr, rowv[rr], scale, lane);
                        if (lane == 0) {
                            rowv[TILE + rr] = -0.5f * tau;
                            out.tau[(size_t)bh * L + ii] = tau;
                        }
                        continue;
                    }
                    int lo_k, hi_k;
                    row_key_range(ii, L, a.causal, a.window, lo_k, hi_k);
                    // Q row from the swizzled tile: 16-byte chunk c of row rr at rr*128 + ((c ^ (rr & 7)) << 4)
                    uint4 qv[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        qv[c] = *reinterpret_cast<const uint4*>(sQ + rr * 128 + ((c ^ (rr & 7)) << 4));
                    float x[FB_NPL];
                    float mx = -INFINITY;
                    int na = 0;
#pragma unroll
                    for (int e = 0; e < FB_NPL; ++e) {
                        const int j = lo_k + 32 * e + lane;
                        x[e] = -INFINITY;
                        if (j <= hi_k && ((bits[j >> 5] >> (j & 31)) & 1u)) {
                            const uint4* kr = reinterpret_cast<const uint4*>(
                                static_cast<const __nv_bfloat16*>(a.K) + hkv.row(j) * HEAD_DIM);
                            float acc = 0.f;
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                const uint4 kw = __ldg(kr + c);
                                acc = fmaf(bfl(qv[c].x), bfl(kw.x), acc);
                                acc = fmaf(bfh(qv[c].x), bfh(kw.x), acc);
                                acc = fmaf(bfl(qv[c].y), bfl(kw.y), acc);
                                acc = fmaf(bfh(qv[c].y), bfh(kw.y), acc);
                                acc = fmaf(bfl(qv[c].z), bfl(kw.z), acc);
                                acc = fmaf(bfh(qv[c].z), bfh(kw.z), acc);
                                acc = fmaf(bfl(qv[c].w), bfl(kw.w), acc);
                                acc = fmaf(bfh(qv[c].w), bfh(kw.w), acc);
                            }
                            x[e] = acc * scale;
                            mx = fmaxf(mx, x[e]);
                            ++na;
                        }
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                        na += __shfl_xor_sync(0xffffffffu, na, o);
                    }
#pragma unroll
                    for (int e = 0; e < FB_NPL; ++e) x[e] -= mx;  // -inf stays -inf
                    const float tau_x = solve_tau_warp<FB_NPL>(x, -2.f, -2.f / sqrtf((float)max(na, 1)));
                    const float tau = na > 0 ? mx + tau_x : INFINITY;
                    if (lane == 0) {
                        rowv[TILE + rr] = -0.5f * tau;
                        if (ii < L) out.tau[(size_t)bh * L + ii] = tau;
                    }
                }
            }
        }
        epi_bar();  // every row's -tau/2 in place

        // ---- pass 3: P = h^2, h = [(S - tau)/2]_+ = [hs s + c]_+, as bf16 parts over the score columns
        const float hs = 0.5f * scale, c = rowv[TILE + r];
        const uint64_t hs2 = f2pack(hs, hs), c2 = f2pack(c, c);
        for (int n = 0; n < nb && live; ++n) {
            const int m = 2 * nb + n;
            live = warp_wait_d(smem_u32(&ctl->s_full[m & 1]), (uint32_t)(m >> 1) & 1u, &ctl->abort_flag, wc);
            if (!live) break;
            tc_fence_after();
            const uint32_t vm = allowed(n);
            const uint32_t tr = trow(m);
            auto p_sub = [&](int cc, bool masked) {
                float sv[SUB];
                tmem_ld16(tr + SUB * cc, sv);
                tmem_wait_ld16(sv);
                uint32_t phi[SUB / 2], plo[SUB / 2];
#pragma unroll
                for (int k = 0; k < SUB; k += 2) {
                    uint64_t h2 = weight2<false>(f2pack(sv[k], sv[k + 1]), hs2, c2);
                    if (masked) h2 = f2mask(h2, vm, SUB * cc + k);
                    f2split(f2mul(h2, h2), phi[k >> 1], plo[k >> 1]);
                }
                tmem_st8(tr + SUB * cc, phi);
                tmem_st8(tr + SUB * cc + 8, plo);
            };
            if (__all_sync(0xffffffffu, vm == 0xffffffffu)) {  // no masked pair in the warp's rows
#pragma unroll
                for (int cc = 0; cc < HB / SUB; ++cc) p_sub(cc, false);
            } else {
#pragma unroll
                for (int cc = 0; cc < HB / SUB; ++cc) p_sub(cc, true);
            }
            tmem_wait_st();
            release(m);
        }
        // O_i: half g writes dimensions [32 g, 32 g + 32); a row with no listed key block has O = 0
        const size_t orow = hq.row(i) * HEAD_DIM + 32 * g;
        float v[32];
        const bool have = nb > 0 && live && warp_wait_d(smem_u32(&ctl->acc_done), 0u, &ctl->abort_flag, wc);
        if (have) {
            tc_fence_after();
            tmem_ld32(tmem + lane_base + 128 + 32 * g, v);
            tmem_wait_ld(v);
        } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = 0.f;
        }
        if (i < L && (have || (nb == 0 && live))) {
            if (out.out_f32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out.O) + orow);
#pragma unroll
                for (int k = 0; k < 8; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            } else {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out.O) + orow);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat162 hh = __floats2bfloat162_rn(v[8 * k + 2 * e], v[8 * k + 2 * e + 1]);
                        w[e] = *reinterpret_cast<uint32_t*>(&hh);
                    }
                    dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // Past this barrier no thread waits, so the abort flag is final (uniform).  After an abort every
    // TMA load and MMA issued must complete before the CTA frees TMEM and its shared memory.
    if (flag_set(&ctl->abort_flag)) {
        drain_dense(&ctl->full_q, ctl->full, NSD, ctl->nload, ctl->last_bar, ctl->last_par, warp, lane);
        tc_fence_before();
        __syncthreads();
    }
    if (warp == W_PROD) {
        tc_fence_after();
        tmem_dealloc(ctl->tmem_base, TMEM_COLS_D);
    }
}

}  // namespace

cudaError_t launch_fwd_dense(const AttnArgs& a, const FwdOut& o, cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    cudaError_t e = make_tile_map(&mq, a.Q, a.layout, a.B, a.H, a.L, TILE);
    if (e == cudaSuccess) e = make_tile_map(&mk, a.K, a.layout, a.B, a.Hkv, a.L, BK);
    if (e == cudaSuccess) e = make_tile_map(&mv, a.V, a.layout, a.B, a.Hkv, a.L, BK);
    if (e != cudaSuccess) return e;
    const void* f = reinterpret_cast<const void*>(entmax_dense_fwd_kernel);
    e = ensure_smem_attr(f, D_SMEM_BYTES, 13);
    if (e != cudaSuccess) return e;
    dim3 grid((a.L + TILE - 1) / TILE, a.B * a.H);
    entmax_dense_fwd_kernel<<<grid, THREADS, D_SMEM_BYTES, stream>>>(mq, mk, mv, a, o);
    return cudaGetLastError();
}

size_t dense_fwd_smem_bytes() { return D_SMEM_BYTES; }

}  // namespace entmax
