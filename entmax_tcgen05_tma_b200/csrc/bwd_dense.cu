// bwd_dense.cu -- backward pass with every contraction on tcgen05: 1.5-entmax attention on rows
// whose allowed keys span few key blocks (short sequences, causal windows), and softmax attention
// (alpha = 1, dense supports) at every length.
//
// Closed-form Jacobian of page "svd-sst2-roberta-adasplash", section 2.4 (model card
// "roberta-base-adasplash", section 2): with h_ij = sqrt(p_ij) = max(0, (S_ij - tau_i)/2),
// dA_ij = dO_i . V_j and u_i = sum_j h_ij dA_ij / sum_j h_ij,
//   dS_ij = h_ij (dA_ij - u_i),  dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO  (P = h^2).
// On short rows a tile of (query, key) pairs is better served by the tensor core than by gathers
// over its support: every product below is a tcgen05.mma with fp32 accumulators in TMEM.  The
// inputs come into shared memory by TMA; P and dS, formed by the epilogue from the S and dA tiles
// it reads out of TMEM, go back into the same TMEM columns (tcgen05.st) and enter their products as
// the A operand read from tensor memory, so they never touch shared memory.
//
//  * dq kernel (query-major, one CTA per 128 queries, 64-key blocks):
//      u_i: from the forward's auxiliary rows when given (u_i = dO_i . Otil_i / r_i with
//           Otil_i = sum_j h_ij V_j, r_i = sum_j h_ij), else a first pass over the blocks:
//           S = Q K^T, dA = dO V^T, u_i from the row sums of h dA and h            -> u (workspace)
//      then S, dA;  dS = h (dA - u) as bf16 hi + lo parts;  dQ += dS_hi K + dS_lo K
//  * dkdv kernel (key-major, one CTA per 128 keys, 64-query blocks over every query head that
//    reads the key/value head):
//      S^T = K Q^T, dA^T = V dO^T;  P^T = h^2, dS^T as above;  dV += P^T dO,  dK += dS^T Q  (hi + lo)
// Softmax (the pages' alpha = 1 branch, page "svd-sst2-roberta-adasplash", section 4) has the same
// Jacobian with h replaced by p = exp(S - tau) (tau = log sum_j exp(S_ij)) and P = p: both kernels
// take it as a template flag that changes only the weight of a score (dense.cuh, weight2).
// The dq kernel runs first: the dkdv kernel reads its u.  dS and P enter the tensor core as two
// bf16 parts each (x = hi + lo to about 16 significant bits), so dQ, dK and dV carry fp32-level
// accuracy (one bf16 part would leave errors of order 1e-2 in sums over a few hundred terms).  No
// atomics: every sum runs in a fixed order, so the results are the same bit for bit from run to run.
//
// Roles (320 threads, two CTAs per SM): warps 0-7 epilogue -- thread (g, r) serves TMEM lane and
// tile row r and columns [32 g, 32 g + 32) of each 64-column block, so each row's work is split
// over two warps; warp 8 TMA producer (and TMEM allocation); warp 9 MMA issuer.  Each CTA has one
// TMEM set (a block's S and dA tiles, then its P and dS parts), which goes back to the MMA issuer's
// commit after the last product that reads it; the two CTAs on an SM keep the tensor core busy in
// turn.  Blocks are 64 columns wide because a tcgen05.mma of N <= 64 costs about as much as one of
// N = 128: fewer, wider products.  Every wait is bounded; an abort drains the CTA's own loads and
// MMAs at teardown (common.cuh).
#include <cuda_bf16.h>
#include <math.h>
#include "dense.cuh"
#include "internal.h"

namespace entmax {
namespace {

using namespace dense;

// TMEM set: columns [0, 64) score tile, [64, 128) dA tile.  Epilogue half g reads columns
// [32 g, 32 g + 32) of each, 16 at a time, and writes the bf16 parts of those 16 back over them:
// the hi part (8 packed columns) first, then the lo part.  A product's K step k (block columns
// 16 k .. 16 k + 15) thus reads its hi part at column 16 k and its lo part at 16 k + 8.

// ------------------------------------------------------------------ dq kernel geometry
constexpr int NSQ = 4;                               // input ring stages (a stage lives until its block's dQ MMAs)
constexpr int QO_Q = 0;                              // Q tile [128][64] bf16, SW128
constexpr int QO_DO = QO_Q + TILE_BYTES;             // dO tile
constexpr int QO_RING = QO_DO + TILE_BYTES;          // NSQ x (K block, V block)
constexpr int QO_BITS = QO_RING + NSQ * 2 * BLK_ROW_BYTES;  // u32 [MASK_WORDS] valid keys
constexpr int QO_BLK = QO_BITS + MASK_WORDS * 4;     // u16 [MAX_L / BK] key blocks
constexpr int QO_RED = QO_BLK + (MAX_L / BK) * 2;    // float [2][TILE]: partial row sums of half 1
constexpr int QO_CTL = QO_RED + 2 * TILE * 4;

struct DqCtl {
    uint64_t full_a;          // Q and dO tiles landed
    uint64_t full[NSQ];       // K, V block landed
    uint64_t empty[NSQ];      // stage free (its last MMA completed)
    uint64_t s_full;          // S, dA of a block in the TMEM set
    uint64_t s_free;          // the set free again (MMA commit after its last product)
    uint64_t ds_ready;        // epilogue done with the set: dS parts stored (or sums taken) (8 warp arrivals)
    uint64_t acc_done;        // last dQ MMA completed
    uint32_t tmem_base;
    int abort_flag;
    int nblk;
    int nload;                // K/V stages loaded (teardown drain)
    uint32_t last_bar;        // barrier and parity of the MMA thread's last commit (teardown drain)
    uint32_t last_par;
};
constexpr int Q_SMEM_BYTES = QO_CTL + (int)sizeof(DqCtl) + 1024;
static_assert(QO_RING % 1024 == 0 && BLK_ROW_BYTES % 1024 == 0, "operand alignment");
static_assert(Q_SMEM_BYTES <= 113 * 1024, "two CTAs per SM");

// ------------------------------------------------------------------ dkdv kernel geometry
constexpr int NSK = 4;                               // input ring stages
constexpr int KO_K = 0;                              // K tile [128][64], SW128
constexpr int KO_V = KO_K + TILE_BYTES;              // V tile
constexpr int KO_RING = KO_V + TILE_BYTES;           // NSK x (Q block, dO block)
constexpr int KO_CU = KO_RING + NSK * 2 * BLK_ROW_BYTES;  // per epilogue warp: float [2][32]: woffset(tau), u of its 32 queries
constexpr int KO_CTL = KO_CU + (NUM_EPI / 32) * 2 * HB * 4;

struct DkCtl {
    uint64_t full_a;          // K and V tiles landed
    uint64_t full[NSK];       // Q, dO block landed
    uint64_t empty[NSK];
    uint64_t s_full;          // S^T, dA^T of a block in the TMEM set
    uint64_t s_free;          // the set free again (MMA commit after its dV, dK products)
    uint64_t pds_ready;       // P^T, dS^T parts stored (8 warp arrivals)
    uint64_t acc_done;
    uint32_t tmem_base;
    int abort_flag;
    int nload;
    uint32_t last_bar;
    uint32_t last_par;
};
constexpr int K_SMEM_BYTES = KO_CTL + (int)sizeof(DkCtl) + 1024;
static_assert(KO_RING % 1024 == 0, "operand alignment");
static_assert(K_SMEM_BYTES <= 113 * 1024, "two CTAs per SM");

// ================================================================== dq kernel
template <bool kPass1, bool kSoftmax>
__global__ void __launch_bounds__(THREADS, 2)
dense_dq_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                const AttnArgs a, const BwdIO io) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + QO_Q;
    uint8_t* sDO = smem + QO_DO;
    uint8_t* ring = smem + QO_RING;
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + QO_BITS);
    uint16_t* blk = reinterpret_cast<uint16_t*>(smem + QO_BLK);
    float* red = reinterpret_cast<float*>(smem + QO_RED);
    DqCtl* ctl = reinterpret_cast<DqCtl*>(smem + QO_CTL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.L, tile = blockIdx.x, bh = blockIdx.y, b = bh / a.H;
    const int bhk = kv_head_of(bh, a.H, a.Hkv);
    const HeadRef hq{a.layout, b, bh - b * a.H, a.H, L};
    const HeadRef hkv{a.layout, b, bhk - b * a.Hkv, a.Hkv, L};
    const int i0 = tile * TILE;
    const WaitCfg wc{a.status, a.timeout_ns};

    if (tid == 0) {
        mbar_init(smem_u32(&ctl->full_a), 1);
        for (int s = 0; s < NSQ; ++s) {
            mbar_init(smem_u32(&ctl->full[s]), 1);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
        }
        mbar_init(smem_u32(&ctl->s_full), 1);
        mbar_init(smem_u32(&ctl->s_free), 1);
        mbar_init(smem_u32(&ctl->ds_ready), NUM_EPI / 32);
        mbar_init(smem_u32(&ctl->acc_done), 1);
        ctl->abort_flag = 0;
        ctl->nload = 0;
        ctl->last_bar = 0;
        ctl->last_par = 0;
        fence_barrier_init();
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_do);
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
    const int np1 = kPass1 ? nb : 0;  // u-pass jobs; then nb dS jobs
    const int njobs = np1 + nb;
    const uint32_t tmem = ctl->tmem_base;  // set: S [0, 64), dA [64, 128); dQ accumulator [128, 192)

    if (warp == W_PROD) {
        if (lane == 0) {
            mbar_arrive_expect_tx(smem_u32(&ctl->full_a), 2 * TILE_BYTES);
            tma_load_3d(smem_u32(sQ), &map_q, 0, hq.c1(i0), hq.c2(i0), smem_u32(&ctl->full_a));
            tma_load_3d(smem_u32(sDO), &map_do, 0, hq.c1(i0), hq.c2(i0), smem_u32(&ctl->full_a));
            int issued = 0;
            for (int m = 0; m < njobs; ++m) {
                const int s = m % NSQ;
                if (!wait_bounded(smem_u32(&ctl->empty[s]), ((uint32_t)(m / NSQ) & 1u) ^ 1u, &ctl->abort_flag, wc))
                    break;
                const int row = (int)(blk[m < np1 ? m : m - np1] & ~FULL_BLOCK) * BK;
                uint8_t* st = ring + s * 2 * BLK_ROW_BYTES;
                mbar_arrive_expect_tx(smem_u32(&ctl->full[s]), 2 * BLK_ROW_BYTES);
                tma_load_3d(smem_u32(st), &map_k, 0, hkv.c1(row), hkv.c2(row), smem_u32(&ctl->full[s]));
                tma_load_3d(smem_u32(st + BLK_ROW_BYTES), &map_v, 0, hkv.c1(row), hkv.c2(row), smem_u32(&ctl->full[s]));
                ++issued;
            }
            ctl->nload = issued;
        }
        __syncwarp();
    } else if (warp == W_MMA) {
        if (lane == 0) {
            constexpr uint32_t IDESC_S = umma_idesc_bf16_f32(TILE, BK);
            constexpr uint32_t IDESC_DQ = umma_idesc_bf16_f32_bmn(TILE, HEAD_DIM);
            uint32_t last_bar = 0, last_par = 0;
            bool ok = wait_bounded(smem_u32(&ctl->full_a), 0, &ctl->abort_flag, wc);
            const uint64_t dq = umma_desc_kmajor_sw128(smem_u32(sQ));
            const uint64_t ddo = umma_desc_kmajor_sw128(smem_u32(sDO));
            if (ok) tc_fence_after();
            for (int m = 0; m < njobs && ok; ++m) {
                const int s = m % NSQ;
                ok = wait_bounded(smem_u32(&ctl->full[s]), (uint32_t)(m / NSQ) & 1u, &ctl->abort_flag, wc) &&
                     wait_bounded(smem_u32(&ctl->s_free), ((uint32_t)m & 1u) ^ 1u, &ctl->abort_flag, wc);
                if (!ok) break;
                tc_fence_after();
                uint8_t* st = ring + s * 2 * BLK_ROW_BYTES;
                const uint64_t dk = umma_desc_kmajor_sw128(smem_u32(st));
                const uint64_t dv = umma_desc_kmajor_sw128(smem_u32(st + BLK_ROW_BYTES));
#pragma unroll
                for (int k = 0; k < HEAD_DIM / 16; ++k)
                    tc_mma_bf16(tmem, dq + 2u * k, dk + 2u * k, IDESC_S, k > 0 ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < HEAD_DIM / 16; ++k)
                    tc_mma_bf16(tmem + 64, ddo + 2u * k, dv + 2u * k, IDESC_S, k > 0 ? 1u : 0u);
                commit_to(&ctl->s_full, (uint32_t)m & 1u, &last_bar, &last_par);
                // the epilogue is done with the set: for a dS job, dQ += dS_hi K + dS_lo K with the
                // parts read from the set (A in TMEM) and the K block of this stage (B, M/N-major)
                ok = wait_bounded(smem_u32(&ctl->ds_ready), (uint32_t)m & 1u, &ctl->abort_flag, wc);
                if (!ok) break;
                tc_fence_after();
                if (m >= np1) {
                    const int n = m - np1;
                    const uint64_t dkm = umma_desc_mnmajor_sw128(smem_u32(st));
                    // 16 keys per step: hi part at column 16 k, lo part at 16 k + 8; two 8-row groups
                    // (2048 B) of the K block
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_bf16_ta(tmem + 128, tmem + 16 * k, dkm + 128u * k, IDESC_DQ, (n > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_bf16_ta(tmem + 128, tmem + 16 * k + 8, dkm + 128u * k, IDESC_DQ, 1u);
                }
                commit_to(&ctl->empty[s], (uint32_t)(m / NSQ) & 1u, &last_bar, &last_par);
                commit_to(&ctl->s_free, (uint32_t)m & 1u, &last_bar, &last_par);
            }
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
        const float tau_i = i < L ? io.tau[(size_t)bh * L + i] : INFINITY;
        const float hs = wslope<kSoftmax>(a.scale), hc = woffset<kSoftmax>(tau_i);  // weight of a raw score pair
        const uint64_t hs2 = f2pack(hs, hs), hc2 = f2pack(hc, hc);
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t trow = tmem + lane_base + (uint32_t)(HB * g);
        auto allowed = [&](int e) -> uint32_t {  // bit k: key 32 g + k of listed block e allowed for row i
            const uint16_t ent = blk[e];
            const int jc = (int)(ent & ~FULL_BLOCK) * BK + HB * g;
            if ((ent & FULL_BLOCK) && i < L) return 0xffffffffu;
            return (jc < L && i < L) ? (bits[jc >> 5] & range_bits(jc, rlo, rhi)) : 0u;
        };
        // sub-chunk c (16 columns) of this thread's half of S, dA
        auto read_sub = [&](int c, float (&sv)[SUB], float (&av)[SUB]) {
            tmem_ld16(trow + SUB * c, sv);
            tmem_ld16(trow + 64 + SUB * c, av);
            tmem_wait_ld16(sv);
            tmem_wait_ld16(av);
        };
        // this warp is done with the set (its dS parts, if any, written)
        auto done_set = [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->ds_ready));
        };
        bool live = true;
        float u = 0.f;
        if (kPass1) {
            float sh = 0.f, sw = 0.f;
            for (int n = 0; n < nb && live; ++n) {
                live = warp_wait_d(smem_u32(&ctl->s_full), (uint32_t)n & 1u, &ctl->abort_flag, wc);
                if (!live) break;
                tc_fence_after();
                const uint32_t vm = allowed(n);
                uint64_t sh2 = 0, sw2 = 0;
#pragma unroll
                for (int c = 0; c < HB / SUB; ++c) {
                    float sv[SUB], av[SUB];
                    read_sub(c, sv, av);
#pragma unroll
                    for (int k = 0; k < SUB; k += 2) {
                        const uint64_t h2 = f2mask(weight2<kSoftmax>(f2pack(sv[k], sv[k + 1]), hs2, hc2), vm, SUB * c + k);
                        sh2 = f2add(sh2, h2);
                        sw2 = f2fma(h2, f2pack(av[k], av[k + 1]), sw2);
                    }
                }
                done_set();
                float x, y;
                f2unpack(sh2, x, y);
                sh += x + y;
                f2unpack(sw2, x, y);
                sw += x + y;
            }
            // combine the two halves of the row
            if (g == 1) {
                red[r] = sh;
                red[TILE + r] = sw;
            }
            epi_bar();
            if (g == 0) {
                sh += red[r];
                sw += red[TILE + r];
                u = sh > 0.f ? sw / sh : 0.f;
                red[r] = u;
                if (live && i < L) io.u[(size_t)bh * L + i] = u;
            }
            epi_bar();
            if (g == 1) u = red[r];
        } else {
            // u_i = dO_i . Otil_i / r_i from the forward's auxiliary rows (logical row order): half g
            // takes dimensions [32 g, 32 g + 32), dO_i from the TMA'd tile (128-byte swizzled rows:
            // 16-byte chunk q of row r at r * 128 + ((q ^ (r & 7)) << 4)), and the halves add up
            const size_t row = (size_t)bh * L + i;
            float dot = 0.f;
            float4 o[8];
            if (i < L) {
                const float4* ot = reinterpret_cast<const float4*>(io.otil + row * HEAD_DIM + 32 * g);
#pragma unroll
                for (int c = 0; c < 8; ++c) o[c] = __ldg(ot + c);
            }
            live = warp_wait_d(smem_u32(&ctl->full_a), 0u, &ctl->abort_flag, wc);  // the dO tile
            if (i < L && live) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t q = (uint32_t)(4 * g + c);
                    const uint4 w = *reinterpret_cast<const uint4*>(sDO + (uint32_t)r * 128u + ((q ^ ((uint32_t)r & 7u)) << 4));
                    dot = fmaf(bf16lo(w.x), o[2 * c].x, dot);
                    dot = fmaf(bf16hi(w.x), o[2 * c].y, dot);
                    dot = fmaf(bf16lo(w.y), o[2 * c].z, dot);
                    dot = fmaf(bf16hi(w.y), o[2 * c].w, dot);
                    dot = fmaf(bf16lo(w.z), o[2 * c + 1].x, dot);
                    dot = fmaf(bf16hi(w.z), o[2 * c + 1].y, dot);
                    dot = fmaf(bf16lo(w.w), o[2 * c + 1].z, dot);
                    dot = fmaf(bf16hi(w.w), o[2 * c + 1].w, dot);
                }
            }
            if (g == 1) red[r] = dot;
            epi_bar();
            if (g == 0) red[TILE + r] = dot + red[r];
            epi_bar();
            if (i < L) {
                const float rs = kSoftmax ? 1.f : io.rsum[row];  // softmax: sum_j p_ij = 1
                u = rs > 0.f ? red[TILE + r] / rs : 0.f;
                if (g == 0) io.u[row] = u;
            }
        }
        for (int n = 0; n < nb && live; ++n) {
            const int m = np1 + n;
            live = warp_wait_d(smem_u32(&ctl->s_full), (uint32_t)m & 1u, &ctl->abort_flag, wc);
            if (!live) break;
            tc_fence_after();
            const uint32_t vm = allowed(n);
            const uint64_t u2 = f2pack(u, u);
            // dS = h (dA - u) for 16 columns, split into bf16 parts and written back over the score
            // columns this thread just read
            auto ds_sub = [&](int c, bool masked) {
                float sv[SUB], av[SUB];
                read_sub(c, sv, av);
                uint32_t hi[SUB / 2], lo[SUB / 2];
#pragma unroll
                for (int k = 0; k < SUB; k += 2) {
                    uint64_t h2 = weight2<kSoftmax>(f2pack(sv[k], sv[k + 1]), hs2, hc2);
                    if (masked) h2 = f2mask(h2, vm, SUB * c + k);
                    f2split(f2mul(h2, f2sub(f2pack(av[k], av[k + 1]), u2)), hi[k >> 1], lo[k >> 1]);
                }
                tmem_st8(trow + SUB * c, hi);
                tmem_st8(trow + SUB * c + 8, lo);
            };
            if (__all_sync(0xffffffffu, vm == 0xffffffffu)) {  // no masked pair in the warp's rows
#pragma unroll
                for (int c = 0; c < HB / SUB; ++c) ds_sub(c, false);
            } else {
#pragma unroll
                for (int c = 0; c < HB / SUB; ++c) ds_sub(c, true);
            }
            tmem_wait_st();
            done_set();
        }
        // dQ_i = scale * (accumulated dS K); half g writes dimensions [32 g, 32 g + 32).  A row with
        // no listed key block has dQ = 0.
        float4* dst = reinterpret_cast<float4*>(io.dQ + hq.row(i) * HEAD_DIM + 32 * g);
        if (nb == 0 && i < L) {
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (nb > 0 && live) live = warp_wait_d(smem_u32(&ctl->acc_done), 0u, &ctl->abort_flag, wc);
        if (nb > 0 && live) {
            tc_fence_after();
            float v[32];
            tmem_ld32(tmem + lane_base + 128 + 32 * g, v);
            tmem_wait_ld(v);
            if (i < L) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    dst[k] = make_float4(a.scale * v[4 * k], a.scale * v[4 * k + 1], a.scale * v[4 * k + 2],
                                         a.scale * v[4 * k + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // Past this barrier no thread waits, so the abort flag is final (uniform).  After an abort every
    // TMA load and MMA issued must complete before the CTA frees TMEM and its shared memory.
    if (flag_set(&ctl->abort_flag)) {
        drain_dense(&ctl->full_a, ctl->full, NSQ, ctl->nload, ctl->last_bar, ctl->last_par, warp, lane);
        tc_fence_before();
        __syncthreads();
    }
    if (warp == W_PROD) {
        tc_fence_after();
        tmem_dealloc(ctl->tmem_base, TMEM_COLS_D);
    }
}

// ================================================================== dkdv kernel
template <bool kSoftmax>
__global__ void __launch_bounds__(THREADS, 2)
dense_dkdv_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                  const AttnArgs a, const BwdIO io) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sK = smem + KO_K;
    uint8_t* sV = smem + KO_V;
    uint8_t* ring = smem + KO_RING;
    float* cu_all = reinterpret_cast<float*>(smem + KO_CU);
    DkCtl* ctl = reinterpret_cast<DkCtl*>(smem + KO_CTL);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = a.L, tile = blockIdx.x, bhk = blockIdx.y, b = bhk / a.Hkv;
    const int hk = bhk - b * a.Hkv, rep = a.H / a.Hkv;
    const HeadRef hkv{a.layout, b, hk, a.Hkv, L};
    const int j0 = tile * TILE, j_last = min(j0 + TILE - 1, L - 1);
    const WaitCfg wc{a.status, a.timeout_ns};

    // query blocks of each query head that reads this key/value head: [qb0, qb0 + nbq)
    const int qlo = a.causal ? j0 : 0;
    const int qhi = a.window > 0 ? min(L - 1, j_last + a.window - 1) : L - 1;
    const int qb0 = qlo / BK, nbq = qhi / BK - qb0 + 1;
    // key rows of the tile that are valid keys (padding and rows past L have zero gradients)
    const int jt = j0 + (tid & (TILE - 1));
    const bool my_key_ok = tid < NUM_EPI && jt < L && (a.key_mask == nullptr || a.key_mask[(size_t)b * L + jt] != 0);

    if (tid == 0) {
        mbar_init(smem_u32(&ctl->full_a), 1);
        for (int s = 0; s < NSK; ++s) {
            mbar_init(smem_u32(&ctl->full[s]), 1);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
        }
        mbar_init(smem_u32(&ctl->s_full), 1);
        mbar_init(smem_u32(&ctl->s_free), 1);
        mbar_init(smem_u32(&ctl->pds_ready), NUM_EPI / 32);
        mbar_init(smem_u32(&ctl->acc_done), 1);
        ctl->abort_flag = 0;
        ctl->nload = 0;
        ctl->last_bar = 0;
        ctl->last_par = 0;
        fence_barrier_init();
        prefetch_tmap(&map_k);
        prefetch_tmap(&map_v);
        prefetch_tmap(&map_q);
        prefetch_tmap(&map_do);
    }
    if (warp == W_PROD) {
        tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS_D);
        tmem_relinquish();
    }
    tc_fence_before();
    const bool any_key = __syncthreads_or(my_key_ok) != 0;
    tc_fence_after();
    const int njobs = any_key ? rep * nbq : 0;  // a tile of padding keys only: zero gradients, no work
    const uint32_t tmem = ctl->tmem_base;  // set: S^T [0, 64), dA^T [64, 128); dK [128, 192); dV [192, 256)

    if (warp == W_PROD) {
        if (lane == 0) {
            mbar_arrive_expect_tx(smem_u32(&ctl->full_a), 2 * TILE_BYTES);
            tma_load_3d(smem_u32(sK), &map_k, 0, hkv.c1(j0), hkv.c2(j0), smem_u32(&ctl->full_a));
            tma_load_3d(smem_u32(sV), &map_v, 0, hkv.c1(j0), hkv.c2(j0), smem_u32(&ctl->full_a));
            int issued = 0;
            for (int m = 0; m < njobs; ++m) {
                const int s = m % NSK;
                if (!wait_bounded(smem_u32(&ctl->empty[s]), ((uint32_t)(m / NSK) & 1u) ^ 1u, &ctl->abort_flag, wc))
                    break;
                const int gq = m / nbq, q0 = (qb0 + m - gq * nbq) * BK;
                const HeadRef hq{a.layout, b, hk * rep + gq, a.H, L};
                uint8_t* st = ring + s * 2 * BLK_ROW_BYTES;
                mbar_arrive_expect_tx(smem_u32(&ctl->full[s]), 2 * BLK_ROW_BYTES);
                tma_load_3d(smem_u32(st), &map_q, 0, hq.c1(q0), hq.c2(q0), smem_u32(&ctl->full[s]));
                tma_load_3d(smem_u32(st + BLK_ROW_BYTES), &map_do, 0, hq.c1(q0), hq.c2(q0), smem_u32(&ctl->full[s]));
                ++issued;
            }
            ctl->nload = issued;
        }
        __syncwarp();
    } else if (warp == W_MMA) {
        if (lane == 0) {
            constexpr uint32_t IDESC_ST = umma_idesc_bf16_f32(TILE, BK);
            constexpr uint32_t IDESC_ACC = umma_idesc_bf16_f32_bmn(TILE, HEAD_DIM);
            uint32_t last_bar = 0, last_par = 0;
            bool ok = wait_bounded(smem_u32(&ctl->full_a), 0, &ctl->abort_flag, wc);
            const uint64_t dkt = umma_desc_kmajor_sw128(smem_u32(sK));
            const uint64_t dvt = umma_desc_kmajor_sw128(smem_u32(sV));
            if (ok) tc_fence_after();
            for (int m = 0; m < njobs && ok; ++m) {
                const int s = m % NSK;
                ok = wait_bounded(smem_u32(&ctl->full[s]), (uint32_t)(m / NSK) & 1u, &ctl->abort_flag, wc) &&
                     wait_bounded(smem_u32(&ctl->s_free), ((uint32_t)m & 1u) ^ 1u, &ctl->abort_flag, wc);
                if (!ok) break;
                tc_fence_after();
                uint8_t* stq = ring + s * 2 * BLK_ROW_BYTES;
                const uint64_t dqb = umma_desc_kmajor_sw128(smem_u32(stq));
                const uint64_t dob = umma_desc_kmajor_sw128(smem_u32(stq + BLK_ROW_BYTES));
#pragma unroll
                for (int k = 0; k < HEAD_DIM / 16; ++k)
                    tc_mma_bf16(tmem, dkt + 2u * k, dqb + 2u * k, IDESC_ST, k > 0 ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < HEAD_DIM / 16; ++k)
                    tc_mma_bf16(tmem + 64, dvt + 2u * k, dob + 2u * k, IDESC_ST, k > 0 ? 1u : 0u);
                commit_to(&ctl->s_full, (uint32_t)m & 1u, &last_bar, &last_par);
                // dV += P^T_hi dO + P^T_lo dO, dK += dS^T_hi Q + dS^T_lo Q, the parts read from the
                // set (A in TMEM), dO and Q from this stage (B, M/N-major)
                ok = wait_bounded(smem_u32(&ctl->pds_ready), (uint32_t)m & 1u, &ctl->abort_flag, wc);
                if (!ok) break;
                tc_fence_after();
                const uint64_t qm = umma_desc_mnmajor_sw128(smem_u32(stq));
                const uint64_t om = umma_desc_mnmajor_sw128(smem_u32(stq + BLK_ROW_BYTES));
                // 16 queries per step: hi part at column 16 k (+ 64 for dS), lo part 8 further;
                // 2048 B of the SW128 Q / dO block
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    tc_mma_bf16_ta(tmem + 192, tmem + 16 * k, om + 128u * k, IDESC_ACC, (m > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k) tc_mma_bf16_ta(tmem + 192, tmem + 16 * k + 8, om + 128u * k, IDESC_ACC, 1u);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    tc_mma_bf16_ta(tmem + 128, tmem + 64 + 16 * k, qm + 128u * k, IDESC_ACC, (m > 0 || k > 0) ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    tc_mma_bf16_ta(tmem + 128, tmem + 64 + 16 * k + 8, qm + 128u * k, IDESC_ACC, 1u);
                commit_to(&ctl->empty[s], (uint32_t)(m / NSK) & 1u, &last_bar, &last_par);
                commit_to(&ctl->s_free, (uint32_t)m & 1u, &last_bar, &last_par);
            }
            if (ok && njobs > 0) commit_to(&ctl->acc_done, 0u, &last_bar, &last_par);
            ctl->last_bar = last_bar;
            ctl->last_par = last_par;
        }
        __syncwarp();
    } else {
        // epilogue: thread (g, r) <-> key j0 + r <-> TMEM lane r, queries [32 g, 32 g + 32) of each block
        const int r = tid & (TILE - 1), g = tid >> 7, j = j0 + r;
        const bool key_ok = my_key_ok;
        int cq_lo, cq_hi;
        col_query_range(j, L, a.causal, a.window, cq_lo, cq_hi);
        const float hs = wslope<kSoftmax>(a.scale);
        const uint64_t hs2 = f2pack(hs, hs);
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t trow = tmem + lane_base + (uint32_t)(HB * g);
        float* cu = cu_all + warp * 2 * HB;  // this warp's copy: [0, 32) woffset(tau), [32, 64) u of its 32 queries
        // lane l fetches, for job m, woffset(tau) and u of query 32 g + l of the block (-inf / 0 past L: no
        // such query row)
        auto fetch = [&](int m, float& c, float& uu) {
            c = -INFINITY;
            uu = 0.f;
            if (m < njobs) {
                const int gq = m / nbq, q = (qb0 + m - gq * nbq) * BK + HB * g + lane;
                if (q < L) {
                    const size_t row = (size_t)(b * a.H + hk * rep + gq) * L + q;
                    c = woffset<kSoftmax>(io.tau[row]);
                    uu = io.u[row];
                }
            }
        };
        float c_next, u_next;
        fetch(0, c_next, u_next);
        bool live = true;
        for (int m = 0; m < njobs && live; ++m) {
            // stage this job's (woffset(tau), u) for the warp; start fetching the next job's
            __syncwarp();
            cu[lane] = c_next;
            cu[HB + lane] = u_next;
            fetch(m + 1, c_next, u_next);
            live = warp_wait_d(smem_u32(&ctl->s_full), (uint32_t)m & 1u, &ctl->abort_flag, wc);
            if (!live) break;
            tc_fence_after();
            const int gq = m / nbq, q0 = (qb0 + m - gq * nbq) * BK;
            // every pair of the block allowed for every key of the tile: no per-pair mask
            const bool full = (!a.causal || q0 >= j_last) && (a.window == 0 || q0 + BK - 1 <= j0 + a.window - 1);
            const uint32_t vm = !key_ok ? 0u : full ? 0xffffffffu : range_bits(q0 + HB * g, cq_lo, cq_hi);
            // P^T (h^2, or p for softmax) and dS^T = w (dA^T - u) for 16 columns, split into bf16 parts
            // and written back over the S^T and dA^T columns this thread just read
            auto pds_sub = [&](int c, bool masked) {
                float sv[SUB], av[SUB];
                tmem_ld16(trow + SUB * c, sv);
                tmem_ld16(trow + 64 + SUB * c, av);
                tmem_wait_ld16(sv);
                tmem_wait_ld16(av);
                uint32_t ph[SUB / 2], pl[SUB / 2], hi[SUB / 2], lo[SUB / 2];
#pragma unroll
                for (int k4 = 0; k4 < SUB / 4; ++k4) {
                    const float4 c4 = reinterpret_cast<const float4*>(cu + SUB * c)[k4];
                    const float4 u4 = reinterpret_cast<const float4*>(cu + HB + SUB * c)[k4];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int k = 4 * k4 + 2 * e;
                        const uint64_t c2 = e ? f2pack(c4.z, c4.w) : f2pack(c4.x, c4.y);
                        const uint64_t uu2 = e ? f2pack(u4.z, u4.w) : f2pack(u4.x, u4.y);
                        uint64_t h2 = weight2<kSoftmax>(f2pack(sv[k], sv[k + 1]), hs2, c2);
                        if (masked) h2 = f2mask(h2, vm, SUB * c + k);
                        f2split(kSoftmax ? h2 : f2mul(h2, h2), ph[k >> 1], pl[k >> 1]);
                        f2split(f2mul(h2, f2sub(f2pack(av[k], av[k + 1]), uu2)), hi[k >> 1], lo[k >> 1]);
                    }
                }
                tmem_st8(trow + SUB * c, ph);
                tmem_st8(trow + SUB * c + 8, pl);
                tmem_st8(trow + 64 + SUB * c, hi);
                tmem_st8(trow + 64 + SUB * c + 8, lo);
            };
            if (__all_sync(0xffffffffu, vm == 0xffffffffu)) {  // no masked pair in the warp's keys
#pragma unroll
                for (int c = 0; c < HB / SUB; ++c) pds_sub(c, false);
            } else {
#pragma unroll
                for (int c = 0; c < HB / SUB; ++c) pds_sub(c, true);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->pds_ready));
        }
        // dK_j, dV_j: half g writes dimensions [32 g, 32 g + 32) of both
        float4* dkr = reinterpret_cast<float4*>(io.dK + hkv.row(j) * HEAD_DIM + 32 * g);
        float4* dvr = reinterpret_cast<float4*>(io.dV + hkv.row(j) * HEAD_DIM + 32 * g);
        if (njobs == 0 && j < L) {
#pragma unroll
            for (int c = 0; c < 8; ++c) dkr[c] = dvr[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (njobs > 0 && live) live = warp_wait_d(smem_u32(&ctl->acc_done), 0u, &ctl->abort_flag, wc);
        if (njobs > 0 && live) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 2; ++c) {  // dK (scaled), then dV
                float v[32];
                tmem_ld32(tmem + lane_base + 128 + 64 * c + 32 * g, v);
                tmem_wait_ld(v);
                if (j < L) {
                    const float f = c == 0 ? a.scale : 1.f;
                    float4* dst = c == 0 ? dkr : dvr;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        dst[k] = make_float4(f * v[4 * k], f * v[4 * k + 1], f * v[4 * k + 2], f * v[4 * k + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // Past this barrier no thread waits, so the abort flag is final (uniform).  After an abort every
    // TMA load and MMA issued must complete before the CTA frees TMEM and its shared memory.
    if (flag_set(&ctl->abort_flag)) {
        drain_dense(&ctl->full_a, ctl->full, NSK, ctl->nload, ctl->last_bar, ctl->last_par, warp, lane);
        tc_fence_before();
        __syncthreads();
    }
    if (warp == W_PROD) {
        tc_fence_after();
        tmem_dealloc(ctl->tmem_base, TMEM_COLS_D);
    }
}

}  // namespace

cudaError_t launch_bwd_dense(const AttnArgs& a, const BwdIO& io, cudaStream_t stream) {
    CUtensorMap mq, mdo, mk, mv;
    const void* dO = io.dO;
    cudaError_t e = make_tile_map(&mq, a.Q, a.layout, a.B, a.H, a.L, TILE);
    if (e == cudaSuccess) e = make_tile_map(&mdo, dO, a.layout, a.B, a.H, a.L, TILE);
    if (e == cudaSuccess) e = make_tile_map(&mk, a.K, a.layout, a.B, a.Hkv, a.L, BK);
    if (e == cudaSuccess) e = make_tile_map(&mv, a.V, a.layout, a.B, a.Hkv, a.L, BK);
    if (e != cudaSuccess) return e;
    // without the forward's auxiliary rows the dq kernel first derives u from a pass over the blocks
    // (1.5-entmax); softmax always has them: its auxiliary row is the forward's fp32 O, row sum 1
    const bool sm = softmax_alpha(a);
    const bool pass1 = io.otil == nullptr || (!sm && io.rsum == nullptr);
    dim3 gq((a.L + TILE - 1) / TILE, a.B * a.H);
    if (sm) {
        if (pass1) return cudaErrorInvalidValue;  // every softmax backward has the forward's fp32 O
        const void* fq = reinterpret_cast<const void*>(dense_dq_kernel<false, true>);
        e = ensure_smem_attr(fq, Q_SMEM_BYTES, 9);
        if (e != cudaSuccess) return e;
        dense_dq_kernel<false, true><<<gq, THREADS, Q_SMEM_BYTES, stream>>>(mq, mdo, mk, mv, a, io);
    } else {
        const void* fq = pass1 ? reinterpret_cast<const void*>(dense_dq_kernel<true, false>)
                               : reinterpret_cast<const void*>(dense_dq_kernel<false, false>);
        e = ensure_smem_attr(fq, Q_SMEM_BYTES, pass1 ? 6 : 8);
        if (e != cudaSuccess) return e;
        if (pass1) dense_dq_kernel<true, false><<<gq, THREADS, Q_SMEM_BYTES, stream>>>(mq, mdo, mk, mv, a, io);
        else dense_dq_kernel<false, false><<<gq, THREADS, Q_SMEM_BYTES, stream>>>(mq, mdo, mk, mv, a, io);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    CUtensorMap kk, kv, kq, kdo;
    e = make_tile_map(&kk, a.K, a.layout, a.B, a.Hkv, a.L, TILE);
    if (e == cudaSuccess) e = make_tile_map(&kv, a.V, a.layout, a.B, a.Hkv, a.L, TILE);
    if (e == cudaSuccess) e = make_tile_map(&kq, a.Q, a.layout, a.B, a.H, a.L, BK);
    if (e == cudaSuccess) e = make_tile_map(&kdo, dO, a.layout, a.B, a.H, a.L, BK);
    if (e != cudaSuccess) return e;
    const void* fk = sm ? reinterpret_cast<const void*>(dense_dkdv_kernel<true>)
                        : reinterpret_cast<const void*>(dense_dkdv_kernel<false>);
    e = ensure_smem_attr(fk, K_SMEM_BYTES, sm ? 10 : 7);
    if (e != cudaSuccess) return e;
    dim3 gk((a.L + TILE - 1) / TILE, a.B * a.Hkv);
    if (sm) dense_dkdv_kernel<true><<<gk, THREADS, K_SMEM_BYTES, stream>>>(kk, kv, kq, kdo, a, io);
    else dense_dkdv_kernel<false><<<gk, THREADS, K_SMEM_BYTES, stream>>>(kk, kv, kq, kdo, a, io);
    return cudaGetLastError();
}

size_t dense_dq_smem_bytes() { return Q_SMEM_BYTES; }
size_t dense_dkdv_smem_bytes() { return K_SMEM_BYTES; }

}  // namespace entmax
