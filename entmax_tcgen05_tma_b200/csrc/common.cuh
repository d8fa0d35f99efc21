// common.cuh -- tile geometry, bounded waits, mask bitmaps and the TMA/tcgen05 score
// pipeline shared by the forward and backward kernels.
//
// Score pipeline ("S pass"): one CTA owns a fixed 128-row tile (the A operand) and streams
// 128-row blocks of the other operand (B).  For every streamed block the tensor core computes
// the 128x128 fp32 tile A.B^T into one of two TMEM buffers; epilogue warps read it back with
// tcgen05.ld (TMEM lane = row of A) while the next block's MMA runs.
//
//   warp 4 (lane 0) : TMA producer  -- A tile once, B blocks through an NSTAGE ring
//   warp 5 (lane 0) : MMA issuer    -- 4 x (M128 N128 K16) per block, commit to mbarriers
//   warps 0-3       : epilogue      -- one thread per A row, consumes TMEM buffers
//   warp 4          : TMEM allocation / release
//
// Every wait is bounded: on timeout the CTA records ENTMAX_ERR_TIMEOUT in the device status
// word, raises a CTA-local abort flag that all roles poll, waits (again bounded) for its own
// TMA loads and MMAs in flight, releases TMEM and returns.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace entmax {

constexpr int HEAD_DIM = 64;            // d, the only head size the kernels take
constexpr int TILE = 128;               // rows of the fixed tile == MMA M
constexpr int BLK = 128;                // rows of a streamed block == MMA N
constexpr int NSTAGE = 3;               // streamed-block ring depth
constexpr int TILE_BYTES = TILE * HEAD_DIM * 2;  // 16 KiB, bf16 rows of 128 B
constexpr int BLK_BYTES = BLK * HEAD_DIM * 2;    // 16 KiB
constexpr int NUM_THREADS = 256;
constexpr int TMEM_COLS = 2 * BLK;      // two fp32 score buffers
constexpr int MAX_L = 16384;            // longest sequence the kernels take
constexpr int MASK_WORDS = MAX_L / 32;
constexpr int MAX_BLOCKS = MAX_L / BLK;
constexpr uint64_t TEARDOWN_TIMEOUT_NS = 2000000000ull;  // bound for draining in-flight copies

// device status codes (mirror entmax_status in include/entmax_attn.h)
constexpr int STATUS_OK = 0;
constexpr int STATUS_TIMEOUT = -4;

// Control block shared by all roles of a CTA (lives in shared memory).
struct PipeCtl {
    uint64_t full_a;               // A tile landed
    uint64_t full_b[NSTAGE];       // B block landed
    uint64_t empty_b[NSTAGE];      // B stage consumed by the MMA
    uint64_t s_full[2];            // score buffer written
    uint64_t s_empty[2];           // score buffer read by the epilogue warps
    uint32_t tmem_base;
    int abort_flag;
    int nblk;                      // streamed blocks this CTA visits
    int pad_;
};

struct WaitCfg {
    int* status;                   // device status word (global)
    uint64_t timeout_ns;
};

__device__ __forceinline__ bool cta_aborted(const PipeCtl* ctl) {
    return *reinterpret_cast<const volatile int*>(&ctl->abort_flag) != 0;
}

static __device__ __noinline__ void raise_timeout(PipeCtl* ctl, const WaitCfg& wc) {
    *reinterpret_cast<volatile int*>(&ctl->abort_flag) = 1;
    if (wc.status) atomicExch(wc.status, STATUS_TIMEOUT);
}

// Bounded wait on an mbarrier phase.  Returns false if the CTA aborted (this wait timed out,
// or another role already raised the abort flag).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, PipeCtl* ctl, const WaitCfg& wc) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 127u) == 0) {
            if (cta_aborted(ctl)) return false;
            if (globaltimer_ns() - t0 > wc.timeout_ns) {
                raise_timeout(ctl, wc);
                return false;
            }
        }
    }
}

// Wait used only while draining after an abort: ignores the abort flag, fixed bound.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > TEARDOWN_TIMEOUT_NS) return;
    }
}

// ------------------------------------------------------------------ masks
// Bitmap of valid keys of batch row b: bit j set iff j < L and key_mask[b, j] != 0 (or no mask).
// All threads of the CTA participate.
__device__ __forceinline__ void build_key_bitmap(uint32_t* bits, const uint8_t* key_mask, int b, int L) {
    const int nwords = (L + 31) / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int w = warp; w < nwords; w += NUM_THREADS / 32) {
        const int j = w * 32 + lane;
        bool valid = j < L;
        if (valid && key_mask) valid = key_mask[(size_t)b * L + j] != 0;
        const uint32_t word = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) bits[w] = word;
    }
}

// Keys allowed for query i by the causal / window rules: [lo, hi] (inclusive).
__device__ __forceinline__ void row_key_range(int i, int L, int causal, int window, int& lo, int& hi) {
    lo = window > 0 ? max(0, i - window + 1) : 0;
    hi = causal ? min(i, L - 1) : L - 1;
}

// Queries allowed for key j: [lo, hi] (inclusive) -- the transpose of row_key_range.
__device__ __forceinline__ void col_query_range(int j, int L, int causal, int window, int& lo, int& hi) {
    lo = causal ? j : 0;
    hi = window > 0 ? min(L - 1, j + window - 1) : L - 1;
}

// Bits k of the 32-key chunk starting at jc whose key lies in [lo, hi].
__device__ __forceinline__ uint32_t range_bits(int jc, int lo, int hi) {
    const int a = lo - jc, b = hi - jc;
    if (b < 0 || a > 31) return 0u;
    const int lb = max(a, 0), hb = min(b, 31);
    const uint32_t upper = hb == 31 ? 0xffffffffu : ((1u << (hb + 1)) - 1u);
    return upper & ~((1u << lb) - 1u);
}

// ------------------------------------------------------- TMA producer role
// Loads the fixed A tile (rows a_row0.. of head bh) and then the streamed B blocks listed in
// blk_list (block index -> rows blk*BLK..) through the NSTAGE ring.
__device__ __forceinline__ void role_producer(PipeCtl* ctl, const WaitCfg& wc, const CUtensorMap* map_a,
                                              const CUtensorMap* map_b, int bh, int a_row0,
                                              const uint16_t* blk_list, uint8_t* smem_a, uint8_t* smem_b) {
    const int nblk = ctl->nblk;
    mbar_arrive_expect_tx(smem_u32(&ctl->full_a), TILE_BYTES);
    tma_load_3d(smem_u32(smem_a), map_a, 0, a_row0, bh, smem_u32(&ctl->full_a));
    int issued = 0;
    for (int n = 0; n < nblk; ++n) {
        const int s = n % NSTAGE;
        const uint32_t ph = (uint32_t)(n / NSTAGE) & 1u;
        if (!wait_bounded(smem_u32(&ctl->empty_b[s]), ph ^ 1u, ctl, wc)) break;
        mbar_arrive_expect_tx(smem_u32(&ctl->full_b[s]), BLK_BYTES);
        tma_load_3d(smem_u32(smem_b + s * BLK_BYTES), map_b, 0, (int)blk_list[n] * BLK, bh,
                    smem_u32(&ctl->full_b[s]));
        ++issued;
    }
    if (cta_aborted(ctl)) {
        // drain: every load issued must land before the CTA's shared memory is released
        wait_drain(smem_u32(&ctl->full_a), 0);
        for (int n = max(0, issued - NSTAGE); n < issued; ++n)
            wait_drain(smem_u32(&ctl->full_b[n % NSTAGE]), (uint32_t)(n / NSTAGE) & 1u);
    }
}

// ------------------------------------------------------------ MMA issuer role
__device__ __forceinline__ void role_mma(PipeCtl* ctl, const WaitCfg& wc, const uint8_t* smem_a,
                                         const uint8_t* smem_b) {
    const int nblk = ctl->nblk;
    constexpr uint32_t idesc = umma_idesc_bf16_f32(TILE, BLK);
    int issued = 0;
    if (wait_bounded(smem_u32(&ctl->full_a), 0, ctl, wc)) {
        tc_fence_after();
        const uint64_t da = umma_desc_kmajor_sw128(smem_u32(smem_a));
        for (int n = 0; n < nblk; ++n) {
            const int s = n % NSTAGE, buf = n & 1;
            if (!wait_bounded(smem_u32(&ctl->full_b[s]), (uint32_t)(n / NSTAGE) & 1u, ctl, wc)) break;
            if (!wait_bounded(smem_u32(&ctl->s_empty[buf]), ((uint32_t)(n >> 1) & 1u) ^ 1u, ctl, wc)) break;
            tc_fence_after();
            const uint64_t db = umma_desc_kmajor_sw128(smem_u32(smem_b + s * BLK_BYTES));
            const uint32_t d_tmem = ctl->tmem_base + (uint32_t)(buf * BLK);
#pragma unroll
            for (int k = 0; k < HEAD_DIM / 16; ++k)  // 16 bf16 = 32 B = 2 descriptor units per step
                tc_mma_bf16(d_tmem, da + 2u * k, db + 2u * k, idesc, k > 0 ? 1u : 0u);
            tc_commit(smem_u32(&ctl->empty_b[s]));
            tc_commit(smem_u32(&ctl->s_full[buf]));
            ++issued;
        }
    }
    if (cta_aborted(ctl) && issued > 0) {
        const int n = issued - 1;  // the last commit covers every earlier MMA
        wait_drain(smem_u32(&ctl->s_full[n & 1]), (uint32_t)(n >> 1) & 1u);
    }
}

__device__ __forceinline__ void init_pipe(PipeCtl* ctl) {
    mbar_init(smem_u32(&ctl->full_a), 1);
    for (int s = 0; s < NSTAGE; ++s) {
        mbar_init(smem_u32(&ctl->full_b[s]), 1);
        mbar_init(smem_u32(&ctl->empty_b[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&ctl->s_full[b]), 1);
        mbar_init(smem_u32(&ctl->s_empty[b]), 4);  // one arrival per epilogue warp
    }
    ctl->abort_flag = 0;
    fence_barrier_init();
}

// Epilogue side: wait for score buffer of streamed block n; false on abort.
__device__ __forceinline__ bool epi_wait_scores(PipeCtl* ctl, const WaitCfg& wc, int n) {
    const bool ok = wait_bounded(smem_u32(&ctl->s_full[n & 1]), (uint32_t)(n >> 1) & 1u, ctl, wc);
    tc_fence_after();
    return ok;
}

// Epilogue side: this warp finished reading score buffer of block n.
__device__ __forceinline__ void epi_release_scores(PipeCtl* ctl, int n) {
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&ctl->s_empty[n & 1]));
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace entmax
