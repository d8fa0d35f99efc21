// fwd_softmax.cu -- forward pass of softmax attention (alpha = 1) with its products on tcgen05.
//
// The alpha-entmax routine of page "svd-sst2-roberta-adasplash", section 4 (entmax_bisect) returns
// softmax when |alpha - 1| < 1e-4:  p_ij = exp(S_ij - tau_i) over the allowed keys, with
// tau_i = log sum_j exp(S_ij) (the threshold's place: p = exp(S - tau) sums to one), and
// O_i = sum_j p_ij V_j.  Its supports are dense, so there is nothing to gather: one CTA per 128
// queries walks the 64-key blocks that hold an allowed key for any of its rows, twice.
//   pass 1:  S = Q K^T into TMEM; the epilogue takes each row's max m.
//   pass 2:  S = Q K^T again; p~ = exp(S - m) = 2^(x - m log2 e), x = S log2 e, in (0, 1], as bf16
//            hi + lo parts written back over the S columns (tcgen05.st), and the row sum l of p~;
//            O~ += p~_hi V + p~_lo V with A read from TMEM and V (M/N-major) from shared memory.
//   end:     O = O~ / l,  tau = m + ln l.
// Two passes instead of an online rescale of O: with m known before any p~ is formed, the
// accumulator is never corrected, the extra S product costs 4 of the block's 16 MMAs, and each
// pair costs one exponential.  p~ enters the product as two bf16 parts (p~ = hi + lo to about 16
// significant bits), so O carries fp32-level accuracy.  Two TMEM sets (block n and n + 1's
// scores) let the MMA warp issue the next S while the epilogue works on the current one.  Roles and
// the TMEM part layout: dense.cuh.  A row with no allowed key gets O = 0 and tau = +inf.  The
// training forward also writes O in fp32: the backward's row scalar u_i = sum_j p_ij dA_ij is then
// dO_i . O_i, a row dot instead of a pass over the key blocks.  Every wait
// is bounded; an abort drains the CTA's own loads and MMAs at teardown.
#include <cuda_bf16.h>
#include <math.h>
#include "dense.cuh"
#include "internal.h"

namespace entmax {
namespace {

using namespace dense;

constexpr int NSF = 4;                               // input ring stages
constexpr int FO_Q = 0;                              // Q tile [128][64] bf16, SW128
constexpr int FO_RING = FO_Q + TILE_BYTES;           // NSF x (K block, V block)
constexpr int FO_BITS = FO_RING + NSF * 2 * BLK_ROW_BYTES;  // u32 [MASK_WORDS] valid keys
constexpr int FO_BLK = FO_BITS + MASK_WORDS * 4;     // u16 [MAX_L / BK] key blocks
constexpr int FO_RED = FO_BLK + (MAX_L / BK) * 2;    // float [4][TILE]: each half's row max, then its sum
constexpr int FO_CTL = FO_RED + 4 * TILE * 4;

struct FsCtl {
    uint64_t full_q;          // Q tile landed
    uint64_t full[NSF];       // K (pass 1) or K, V (pass 2) block landed
    uint64_t empty[NSF];      // stage free (its last MMA completed)
    uint64_t s_full[2];       // S of a block in TMEM set 0 / 1
    uint64_t s_free[2];       // the set free again (MMA commit after its last product)
    uint64_t p_ready[2];      // epilogue done with the set: S read, p parts stored (8 warp arrivals)
    uint64_t acc_done;        // last O MMA completed
    uint32_t tmem_base;
    int abort_flag;
    int nblk;
    int nload;
    uint32_t last_bar;
    uint32_t last_par;
};
constexpr int F_SMEM_BYTES = FO_CTL + (int)sizeof(FsCtl) + 1024;
static_assert(FO_RING % 1024 == 0 && BLK_ROW_BYTES % 1024 == 0, "operand alignment");
static_assert(F_SMEM_BYTES <= 113 * 1024, "two CTAs per SM");

__global__ void __launch_bounds__(THREADS, 2)
softmax_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const AttnArgs a, const FwdOut out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + FO_Q;
    uint8_t* ring = smem + FO_RING;
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + FO_BITS);
    uint16_t* blk = reinterpret_cast<uint16_t*>(smem + FO_BLK);
    float* red = reinterpret_cast<float*>(smem + FO_RED);
    FsCtl* ctl = reinterpret_cast<FsCtl*>(smem + FO_CTL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.L, tile = blockIdx.x, bh = blockIdx.y, b = bh / a.H;
    const int bhk = kv_head_of(bh, a.H, a.Hkv);
    const HeadRef hq{a.layout, b, bh - b * a.H, a.H, L};
    const HeadRef hkv{a.layout, b, bhk - b * a.Hkv, a.Hkv, L};
    const int i0 = tile * TILE;
    const WaitCfg wc{a.status, a.timeout_ns};

    if (tid == 0) {
        mbar_init(smem_u32(&ctl->full_q), 1);
        for (int s = 0; s < NSF; ++s) {
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
        ctl->last_bar = 0;
        ctl->last_par = 0;
        fence_barrier_init();
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
    }
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
    const int njobs = 2 * nb;  // job m < nb: pass 1 over block m; job nb + n: pass 2 over block n
    const uint32_t tmem = ctl->tmem_base;  // sets: S [0, 64) and [64, 128); O accumulator [128, 192)

    if (warp == W_PROD) {
        if (lane == 0) {
            mbar_arrive_expect_tx(smem_u32(&ctl->full_q), TILE_BYTES);
            tma_load_3d(smem_u32(sQ), &map_q, 0, hq.c1(i0), hq.c2(i0), smem_u32(&ctl->full_q));
            int issued = 0;
            for (int m = 0; m < njobs; ++m) {
                const int s = m % NSF;
                if (!wait_bounded(smem_u32(&ctl->empty[s]), ((uint32_t)(m / NSF) & 1u) ^ 1u, &ctl->abort_flag, wc))
                    break;
                const bool p2 = m >= nb;
                const int row = (int)(blk[p2 ? m - nb : m] & ~FULL_BLOCK) * BK;
                uint8_t* st = ring + s * 2 * BLK_ROW_BYTES;
                mbar_arrive_expect_tx(smem_u32(&ctl->full[s]), (p2 ? 2 : 1) * BLK_ROW_BYTES);
                tma_load_3d(smem_u32(st), &map_k, 0, hkv.c1(row), hkv.c2(row), smem_u32(&ctl->full[s]));
                if (p2)
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
            // job j's set is read (and, in pass 2, holds its p parts): O += p_hi V + p_lo V for a
            // pass-2 job, then release the stage and the set
            auto finish = [&](int j) -> bool {
                const int s = j % NSF, t = j & 1;
                if (!wait_bounded(smem_u32(&ctl->p_ready[t]), (uint32_t)(j >> 1) & 1u, &ctl->abort_flag, wc))
                    return false;
                tc_fence_after();
                if (j >= nb) {
                    const int n = j - nb;
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
                commit_to(&ctl->empty[s], (uint32_t)(j / NSF) & 1u, &last_bar, &last_par);
                commit_to(&ctl->s_free[t], (uint32_t)(j >> 1) & 1u, &last_bar, &last_par);
                return true;
            };
            for (int m = 0; m < njobs && ok; ++m) {
                const int s = m % NSF, t = m & 1;
                ok = wait_bounded(smem_u32(&ctl->full[s]), (uint32_t)(m / NSF) & 1u, &ctl->abort_flag, wc) &&
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
        const float xs = a.scale * LOG2E;  // x = S log2 e = raw score * xs
        const uint64_t xs2 = f2pack(xs, xs);
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
        bool live = true;
        // pass 1: this half's max of the raw scores over the allowed keys
        float mx = -INFINITY;
        for (int n = 0; n < nb && live; ++n) {
            live = warp_wait_d(smem_u32(&ctl->s_full[n & 1]), (uint32_t)(n >> 1) & 1u, &ctl->abort_flag, wc);
            if (!live) break;
            tc_fence_after();
            float v[32];
            tmem_ld32(trow(n), v);
            tmem_wait_ld(v);
            release(n);  // the scores are in registers: the set can take the next block
            const uint32_t vm = allowed(n);
#pragma unroll
            for (int k = 0; k < 32; ++k)
                if ((vm >> k) & 1u) mx = fmaxf(mx, v[k]);
        }
        // the row max m over both halves (-inf for a row with no allowed key); x = S log2 e, so the
        // row's exponent offset is -m xs (-inf for an empty row, so that every p there is 0)
        red[g * TILE + r] = mx;
        epi_bar();
        const float m = fmaxf(red[r], red[TILE + r]);
        const float cm = m == -INFINITY ? -INFINITY : -m * xs;
        const uint64_t c2 = f2pack(cm, cm);
        // pass 2: p~ = 2^(x - m xs) in (0, 1] for 16 columns at a time, split into bf16 parts written
        // back over the score columns just read; this half's sum of p~ accumulates beside them
        uint64_t ls2 = 0;
        for (int n = 0; n < nb && live; ++n) {
            const int mj = nb + n;
            live = warp_wait_d(smem_u32(&ctl->s_full[mj & 1]), (uint32_t)(mj >> 1) & 1u, &ctl->abort_flag, wc);
            if (!live) break;
            tc_fence_after();
            const uint32_t vm = allowed(n);
            const uint32_t tr = trow(mj);
            auto p_sub = [&](int c, bool masked) {
                float sv[SUB];
                tmem_ld16(tr + SUB * c, sv);
                tmem_wait_ld16(sv);
                uint32_t hi[SUB / 2], lo[SUB / 2];
#pragma unroll
                for (int k = 0; k < SUB; k += 2) {
                    uint64_t p2 = f2exp2(f2fma(f2pack(sv[k], sv[k + 1]), xs2, c2));
                    if (masked) p2 = f2mask(p2, vm, SUB * c + k);
                    ls2 = f2add(ls2, p2);
                    f2split(p2, hi[k >> 1], lo[k >> 1]);
                }
                tmem_st8(tr + SUB * c, hi);
                tmem_st8(tr + SUB * c + 8, lo);
            };
            if (__all_sync(0xffffffffu, vm == 0xffffffffu)) {  // no masked pair in the warp's rows
#pragma unroll
                for (int c = 0; c < HB / SUB; ++c) p_sub(c, false);
            } else {
#pragma unroll
                for (int c = 0; c < HB / SUB; ++c) p_sub(c, true);
            }
            tmem_wait_st();
            release(mj);
        }
        // l = sum_j p~_ij over both halves; tau = ln(sum_j exp S_ij) = (m xs + log2 l) ln 2 (+inf for a
        // row with no allowed key); O_i = (sum_j p~_ij V_j) / l
        {
            float x, y;
            f2unpack(ls2, x, y);
            red[(2 + g) * TILE + r] = x + y;
        }
        epi_bar();
        const float lsum = red[2 * TILE + r] + red[3 * TILE + r];
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        if (g == 0 && live && i < L) out.tau[(size_t)bh * L + i] = lsum > 0.f ? (m * xs + log2f(lsum)) * LN2 : INFINITY;
        // O_i: half g writes dimensions [32 g, 32 g + 32); a row with no listed key block has O = 0
        const size_t orow = hq.row(i) * HEAD_DIM + 32 * g;
        float v[32];
        const bool have = nb > 0 && live && warp_wait_d(smem_u32(&ctl->acc_done), 0u, &ctl->abort_flag, wc);
        if (have) {
            tc_fence_after();
            tmem_ld32(tmem + lane_base + 128 + 32 * g, v);
            tmem_wait_ld(v);
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] *= inv;
        } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = 0.f;
        }
        if (i < L && (have || (nb == 0 && live))) {
            if (out.otil) {  // the backward's auxiliary row: sum_j p_ij V_j = O_i, in fp32
                float4* dst = reinterpret_cast<float4*>(out.otil + ((size_t)bh * L + i) * HEAD_DIM + 32 * g);
#pragma unroll
                for (int k = 0; k < 8; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            }
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
                        __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * k + 2 * e], v[8 * k + 2 * e + 1]);
                        w[e] = *reinterpret_cast<uint32_t*>(&h);
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
        drain_dense(&ctl->full_q, ctl->full, NSF, ctl->nload, ctl->last_bar, ctl->last_par, warp, lane);
        tc_fence_before();
        __syncthreads();
    }
    if (warp == W_PROD) {
        tc_fence_after();
        tmem_dealloc(ctl->tmem_base, TMEM_COLS_D);
    }
}

}  // namespace

cudaError_t launch_fwd_softmax(const AttnArgs& a, const FwdOut& o, cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    cudaError_t e = make_tile_map(&mq, a.Q, a.layout, a.B, a.H, a.L, TILE);
    if (e == cudaSuccess) e = make_tile_map(&mk, a.K, a.layout, a.B, a.Hkv, a.L, BK);
    if (e == cudaSuccess) e = make_tile_map(&mv, a.V, a.layout, a.B, a.Hkv, a.L, BK);
    if (e != cudaSuccess) return e;
    const void* f = reinterpret_cast<const void*>(softmax_fwd_kernel);
    e = ensure_smem_attr(f, F_SMEM_BYTES, 11);
    if (e != cudaSuccess) return e;
    dim3 grid((a.L + TILE - 1) / TILE, a.B * a.H);
    softmax_fwd_kernel<<<grid, THREADS, F_SMEM_BYTES, stream>>>(mq, mk, mv, a, o);
    return cudaGetLastError();
}

size_t softmax_fwd_smem_bytes() { return F_SMEM_BYTES; }

}  // namespace entmax
