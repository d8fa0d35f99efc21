// common.cuh -- tile geometry, bounded waits, mask bitmaps and the TMA/tcgen05 score
// pipeline shared by the forward and backward kernels.
//
// Score pipeline ("S pass"), Pipe<BLK, NSTAGE, NBUF, NWG>: one CTA owns a fixed 128-row tile (the
// A operand) and streams BLK-row blocks of the other operand (B).  For every streamed block the
// tensor core computes the 128 x BLK fp32 tile A.B^T into one of NBUF TMEM buffers (block n ->
// buffer n % NBUF); NWG epilogue warpgroups read them back with tcgen05.ld (TMEM lane = row of A),
// warpgroup g taking the blocks n = g (mod NWG), while later blocks' MMAs run.
//
//   warps 0 .. 4 NWG - 1 : epilogue warpgroups -- thread (g, r) serves A row r
//   next warp (lane 0)   : TMA producer -- A tile once, B blocks through an NSTAGE ring
//   next warp (lane 0)   : MMA issuer   -- 4 x (M128 N=BLK K16) per block, commit to mbarriers
//   producer warp        : TMEM allocation / release
//
// Every wait is bounded: on timeout the CTA records ENTMAX_ERR_TIMEOUT in the device status
// word and raises a CTA-local abort flag that all roles poll; every role then stops and the CTA
// meets at its teardown barrier.  Past that barrier no thread waits on anything else, so the flag
// is final: if it is set, the producer thread waits (again bounded) for every TMA load it issued
// and the MMA thread for its last commit (drain_loads / drain_mma), and only then is TMEM released
// and the CTA returns.  A role that finished issuing before another role timed out still has its
// copies drained this way.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "internal.h"

namespace entmax {

constexpr int HEAD_DIM = 64;            // d, the only head size the kernels take
constexpr int TILE = 128;               // rows of the fixed tile == MMA M
constexpr int TILE_BYTES = TILE * HEAD_DIM * 2;  // 16 KiB, bf16 rows of 128 B
constexpr int MAX_L = 16384;            // longest sequence the kernels take
constexpr int MASK_WORDS = MAX_L / 32;
constexpr uint64_t TEARDOWN_TIMEOUT_NS = 2000000000ull;  // bound for draining in-flight copies
constexpr uint16_t FULL_BLOCK = 0x8000u;  // block-list flag: every key allowed for every row

// device status codes (mirror entmax_status in include/entmax_attn.h)
constexpr int STATUS_OK = 0;
constexpr int STATUS_TIMEOUT = -4;

struct WaitCfg {
    int* status;                   // device status word (global)
    uint64_t timeout_ns;
};

__device__ __forceinline__ bool flag_set(const int* abort_flag) {
    return *reinterpret_cast<const volatile int*>(abort_flag) != 0;
}

static __device__ __noinline__ void raise_timeout(int* abort_flag, const WaitCfg& wc) {
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
    if (wc.status) atomicExch(wc.status, STATUS_TIMEOUT);
}

constexpr uint32_t POLL_SUSPEND_NS = 1000;  // longest suspension inside one poll of a wait

// Bounded wait on an mbarrier phase.  Returns false if the CTA aborted (this wait timed out,
// or another role already raised the abort flag).  After a first non-suspending test the thread
// waits inside mbarrier.try_wait, suspended (taking no issue slots from the warps that work) until
// the phase completes or POLL_SUSPEND_NS pass, and checks the abort flag and the elapsed time
// after every poll that returns without the phase.
// Elapsed time: the global timer, or half the SM cycles elapsed if that is larger (the SM clock
// runs below 2 GHz, so cycles / 2 never overstates the nanoseconds), since the global timer may
// advance in steps coarser than a short bound.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, int* abort_flag, const WaitCfg& wc) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const long long c0 = clock64();
    // a bound shorter than a few polls gets short polls, so it is seen
    const uint32_t hint = wc.timeout_ns < 4ull * POLL_SUSPEND_NS ? 20u : POLL_SUSPEND_NS;
    for (;;) {
        if (mbar_try_wait_hint(bar, parity, hint)) return true;
        if (flag_set(abort_flag)) return false;
        const uint64_t dt = globaltimer_ns() - t0, dc = (uint64_t)(clock64() - c0) >> 1;
        if ((dt > dc ? dt : dc) > wc.timeout_ns) {
            raise_timeout(abort_flag, wc);
            return false;
        }
    }
}

// Wait used only while draining after an abort: ignores the abort flag, fixed bound.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_hint(bar, parity, POLL_SUSPEND_NS)) {
        if (globaltimer_ns() - t0 > TEARDOWN_TIMEOUT_NS) return;
    }
}

// ------------------------------------------------------------------ masks
// The allowed keys of query i follow page "svd-sst2-roberta-adasplash", section 3 ("Structural
// Masking Stage"): the padding mask of the key's batch row, the causal mask (j <= i) and the
// causal local window (j >= i - window + 1).  Masked keys are left out of the row, not filled
// with a large negative score.
// Bitmap of valid keys of batch row b: bit j set iff j < L and key_mask[b, j] != 0 (or no mask).
// All threads of the CTA participate.
__device__ __forceinline__ void build_key_bitmap(uint32_t* bits, const uint8_t* key_mask, int b, int L) {
    const int nwords = (L + 31) / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int w = warp; w < nwords; w += blockDim.x / 32) {
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

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// ------------------------------------------------------------------ score pipeline
template <int kBlk, int kNStage, int kNBuf, int kNumEpiWg>
struct Pipe {
    static constexpr int BLK = kBlk;             // rows of a streamed block == MMA N
    static constexpr int NSTAGE = kNStage;       // streamed-block ring depth
    static constexpr int NBUF = kNBuf;           // TMEM score buffers
    static constexpr int NUM_EPI_WG = kNumEpiWg;
    static constexpr int NUM_EPI = NUM_EPI_WG * 128;
    static constexpr int NUM_THREADS = NUM_EPI + 64;  // + producer warp + MMA warp
    static constexpr int NUM_WARPS = NUM_THREADS / 32;
    static constexpr int WARP_PRODUCER = NUM_EPI / 32;
    static constexpr int WARP_MMA = WARP_PRODUCER + 1;
    static constexpr int BLK_BYTES = BLK * HEAD_DIM * 2;
    static constexpr int TMEM_COLS = NBUF * BLK;
    static constexpr int CHUNKS = BLK / 32;       // 32-column chunks per block
    static constexpr int MAX_BLOCKS = MAX_L / BLK;
    static_assert(BLK % 32 == 0 && BLK >= 32 && BLK <= 256, "MMA N");
    static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation");
    static_assert(NBUF % NUM_EPI_WG == 0, "each warpgroup owns whole buffers");

    // Control block shared by all roles of a CTA (lives in shared memory).
    struct Ctl {
        uint64_t full_a;               // A tile landed
        uint64_t full_b[NSTAGE];       // B block landed
        uint64_t empty_b[NSTAGE];      // B stage consumed by the MMA
        uint64_t s_full[NBUF];         // score buffer written
        uint64_t s_empty[NBUF];        // score buffer read by its epilogue warpgroup
        uint32_t tmem_base;
        int abort_flag;
        int nblk;                      // streamed blocks this CTA visits
        int nload[2];                  // B-block loads issued (per producer/MMA pair)
        int nmma[2];                   // score blocks whose MMAs were issued (per pair)
        int pad_;
    };

    static __device__ __forceinline__ bool aborted(const Ctl* ctl) { return flag_set(&ctl->abort_flag); }

    // empty_arrivals: warps that release each score buffer (4: the owning warpgroup; NUM_EPI / 32
    // when every epilogue warp reads a share of every block).
    static __device__ __forceinline__ void init(Ctl* ctl, uint32_t empty_arrivals = 4) {
        mbar_init(smem_u32(&ctl->full_a), 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(smem_u32(&ctl->full_b[s]), 1);
            mbar_init(smem_u32(&ctl->empty_b[s]), 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(smem_u32(&ctl->s_full[b]), 1);
            mbar_init(smem_u32(&ctl->s_empty[b]), empty_arrivals);
        }
        ctl->abort_flag = 0;
        ctl->nload[0] = ctl->nload[1] = 0;
        ctl->nmma[0] = ctl->nmma[1] = 0;
        fence_barrier_init();
    }

    // Teardown after an abort, run by the producer thread past the CTA's teardown barrier: waits
    // (bounded) for the A tile and the last NSTAGE B loads -- every earlier load was waited on by
    // the MMA thread before it reused the stage.
    static __device__ __forceinline__ void drain_loads(Ctl* ctl) {
        wait_drain(smem_u32(&ctl->full_a), 0);
        const int n1 = ctl->nload[0];
        for (int n = max(0, n1 - NSTAGE); n < n1; ++n)
            wait_drain(smem_u32(&ctl->full_b[n % NSTAGE]), (uint32_t)(n / NSTAGE) & 1u);
    }

    // Teardown after an abort, run by the MMA thread: its last commit covers every MMA it issued.
    static __device__ __forceinline__ void drain_mma(Ctl* ctl) {
        const int n = ctl->nmma[0] - 1;
        if (n >= 0) wait_drain(smem_u32(&ctl->s_full[n % NBUF]), (uint32_t)(n / NBUF) & 1u);
    }

    // Streamed blocks a query tile (rows [i0, i_last]) visits: blocks kb in [klo/BLK, khi/BLK]
    // holding at least one valid key in [klo, khi].  Entry = block index | FULL_BLOCK when every key
    // of the block is valid and allowed for every row of the tile (no per-row mask work needed).
    // Built by one warp (one lane per candidate block, ballot + prefix count); returns the count.
    static __device__ __forceinline__ int build_block_list(uint16_t* list, const uint32_t* bits, int klo, int khi,
                                                           int i0, int i_last, int causal, int window) {
        const int lane = threadIdx.x & 31;
        const int kb0 = klo / BLK, kb1 = khi / BLK;
        int nb = 0;
        for (int base = kb0; base <= kb1; base += 32) {
            const int kb = base + lane;
            bool any = false, full = kb <= kb1;
            if (kb <= kb1) {
#pragma unroll
                for (int q = 0; q < CHUNKS; ++q) {
                    const int w = kb * CHUNKS + q;
                    const uint32_t word = w * 32 <= khi ? bits[w] : 0u;
                    if (w * 32 <= khi) any |= (word & range_bits(w * 32, klo, khi)) != 0u;
                    full &= word == 0xffffffffu;
                }
                const int j0 = kb * BLK, j1 = j0 + BLK - 1;
                if (causal) full &= j1 <= i0;
                if (window > 0) full &= j0 >= i_last - window + 1;
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, any);
            if (any) list[nb + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)(kb | (full ? FULL_BLOCK : 0));
            nb += __popc(bal);
        }
        return nb;
    }

    // TMA producer: the fixed A tile (rows a_row0.. of head ha), then njobs streamed B blocks of head
    // hb through the NSTAGE ring.  Job n < n1 loads listed block n * s1 (a first pass over every
    // s1-th block); job n >= n1 loads listed block n - n1 (a second pass over the whole list).
    // n1 < 0 means n1 = nblk, s1 = 1.
    static __device__ __forceinline__ void producer(Ctl* ctl, const WaitCfg& wc, const CUtensorMap* map_a,
                                                    const CUtensorMap* map_b, const HeadRef& ha, int a_row0,
                                                    const uint16_t* blk_list, uint8_t* smem_a, uint8_t* smem_b,
                                                    int njobs, const HeadRef& hb, int n1 = -1, int s1 = 1) {
        if (n1 < 0) {
            n1 = ctl->nblk;
            s1 = 1;
        }
        mbar_arrive_expect_tx(smem_u32(&ctl->full_a), TILE_BYTES);
        tma_load_3d(smem_u32(smem_a), map_a, 0, ha.c1(a_row0), ha.c2(a_row0), smem_u32(&ctl->full_a));
        int issued = 0;
        for (int n = 0; n < njobs; ++n) {
            const int s = n % NSTAGE;
            const uint32_t ph = (uint32_t)(n / NSTAGE) & 1u;
            if (!wait_bounded(smem_u32(&ctl->empty_b[s]), ph ^ 1u, &ctl->abort_flag, wc)) break;
            const int e = n < n1 ? n * s1 : n - n1;
            mbar_arrive_expect_tx(smem_u32(&ctl->full_b[s]), BLK_BYTES);
            const int row = (int)(blk_list[e] & ~FULL_BLOCK) * BLK;
            tma_load_3d(smem_u32(smem_b + s * BLK_BYTES), map_b, 0, hb.c1(row), hb.c2(row), smem_u32(&ctl->full_b[s]));
            ++issued;
        }
        ctl->nload[0] = issued;  // drained at teardown if the CTA aborts (drain_loads)
    }

    // MMA issuer (one thread).
    static __device__ __forceinline__ void mma(Ctl* ctl, const WaitCfg& wc, const uint8_t* smem_a,
                                               const uint8_t* smem_b, int njobs) {
        constexpr uint32_t idesc = umma_idesc_bf16_f32(TILE, BLK);
        int issued = 0;
        if (wait_bounded(smem_u32(&ctl->full_a), 0, &ctl->abort_flag, wc)) {
            tc_fence_after();
            const uint64_t da = umma_desc_kmajor_sw128(smem_u32(smem_a));
            for (int n = 0; n < njobs; ++n) {
                const int s = n % NSTAGE, buf = n % NBUF;
                if (!wait_bounded(smem_u32(&ctl->full_b[s]), (uint32_t)(n / NSTAGE) & 1u, &ctl->abort_flag, wc)) break;
                if (!wait_bounded(smem_u32(&ctl->s_empty[buf]), ((uint32_t)(n / NBUF) & 1u) ^ 1u, &ctl->abort_flag, wc))
                    break;
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
        ctl->nmma[0] = issued;  // drained at teardown if the CTA aborts (drain_mma)
    }

    // Epilogue side: wait for the score buffer of streamed block n; false on abort.
    static __device__ __forceinline__ bool wait_scores(Ctl* ctl, const WaitCfg& wc, int n) {
        const bool ok = wait_bounded(smem_u32(&ctl->s_full[n % NBUF]), (uint32_t)(n / NBUF) & 1u, &ctl->abort_flag, wc);
        tc_fence_after();
        return ok;
    }

    // Epilogue side: this warp finished reading the score buffer of block n.
    static __device__ __forceinline__ void release_scores(Ctl* ctl, int n) {
        tc_fence_before();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&ctl->s_empty[n % NBUF]));
    }

    // TMEM address of lane quarter (warp % 4), buffer of block n, 32-column chunk c.
    static __device__ __forceinline__ uint32_t taddr(const Ctl* ctl, int n, int c) {
        const int warp = threadIdx.x >> 5;
        return ctl->tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)((n % NBUF) * BLK + c * 32);
    }

    // Reads the 32-column chunks of score block n (the next chunk's load in flight while f runs)
    // and calls f(v, c) for chunk c.  With kRelease the buffer goes back to the MMA warp once its
    // last chunk is in registers; without, it stays readable for a later pass.
    template <bool kRelease = true, class F>
    static __device__ __forceinline__ void for_each_chunk(Ctl* ctl, int n, F&& f) {
        float va[32], vb[32];
        tmem_ld32(taddr(ctl, n, 0), va);
        tmem_wait_ld(va);
#pragma unroll
        for (int c = 0; c < CHUNKS; c += 2) {
            if (c + 1 < CHUNKS) tmem_ld32(taddr(ctl, n, c + 1), vb);
            else if (kRelease) release_scores(ctl, n);
            f(va, c);
            if (c + 1 < CHUNKS) {
                tmem_wait_ld(vb);
                if (c + 2 < CHUNKS) tmem_ld32(taddr(ctl, n, c + 2), va);
                else if (kRelease) release_scores(ctl, n);
                f(vb, c + 1);
                if (c + 2 < CHUNKS) tmem_wait_ld(va);
            }
        }
    }
};

// ------------------------------------------------------------ hit filtering
// Three-input maximum (one sm_100 instruction).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Maximum of a 32-value chunk: a tree of three-input maxima (16 instructions, depth 4).
__device__ __forceinline__ float max32(const float (&v)[32]) {
    float m[11];
#pragma unroll
    for (int k = 0; k < 10; ++k) m[k] = fmax3(v[3 * k], v[3 * k + 1], v[3 * k + 2]);
    m[10] = fmaxf(v[30], v[31]);
    const float a = fmax3(m[0], m[1], m[2]), b = fmax3(m[3], m[4], m[5]), c = fmax3(m[6], m[7], m[8]);
    const float d = fmaxf(m[9], m[10]);
    return fmaxf(fmax3(a, b, c), d);
}

// t - (a, b) for two values at once (one packed sm_100 subtraction).
__device__ __forceinline__ void sub2(float t, float a, float b, float& da, float& db) {
    uint64_t ab, tt, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(ab) : "f"(a), "f"(b));
    asm("mov.b64 %0, {%1, %1};" : "=l"(tt) : "f"(t));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(tt), "l"(ab));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(da), "=f"(db) : "l"(r));
}

// Bit (31 - k) of the result is set iff v[k] > t: the sign bit of t - v[k] (packed subtractions,
// two values each) funnel-shifted into four independent 8-bit chains (no branches).
__device__ __forceinline__ uint32_t hit_bits(const float (&v)[32], float t) {
    uint32_t h0 = 0, h1 = 0, h2 = 0, h3 = 0;
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
        float d[8];
        sub2(t, v[k], v[k + 1], d[0], d[1]);
        sub2(t, v[8 + k], v[9 + k], d[2], d[3]);
        sub2(t, v[16 + k], v[17 + k], d[4], d[5]);
        sub2(t, v[24 + k], v[25 + k], d[6], d[7]);
        h0 = __funnelshift_l(__float_as_uint(d[0]), h0, 1);
        h1 = __funnelshift_l(__float_as_uint(d[2]), h1, 1);
        h2 = __funnelshift_l(__float_as_uint(d[4]), h2, 1);
        h3 = __funnelshift_l(__float_as_uint(d[6]), h3, 1);
        h0 = __funnelshift_l(__float_as_uint(d[1]), h0, 1);
        h1 = __funnelshift_l(__float_as_uint(d[3]), h1, 1);
        h2 = __funnelshift_l(__float_as_uint(d[5]), h2, 1);
        h3 = __funnelshift_l(__float_as_uint(d[7]), h3, 1);
    }
    return (h0 << 24) | (h1 << 16) | (h2 << 8) | h3;
}

// Same with a per-value threshold t[k].
__device__ __forceinline__ uint32_t hit_bits(const float (&v)[32], const float (&t)[32]) {
    uint32_t h0 = 0, h1 = 0, h2 = 0, h3 = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        h0 = __funnelshift_l(__float_as_uint(t[k] - v[k]), h0, 1);
        h1 = __funnelshift_l(__float_as_uint(t[8 + k] - v[8 + k]), h1, 1);
        h2 = __funnelshift_l(__float_as_uint(t[16 + k] - v[16 + k]), h2, 1);
        h3 = __funnelshift_l(__float_as_uint(t[24 + k] - v[24 + k]), h3, 1);
    }
    return (h0 << 24) | (h1 << 16) | (h2 << 8) | h3;
}

// Per-thread staging of a 32-value chunk in shared memory (16-byte groups XOR-swizzled by the
// thread index, so a warp's 128-bit stores are conflict-free), read back by dynamic index.
// `slot` = the thread's epilogue index.
__device__ __forceinline__ void stage_chunk(float* stage, int slot, const float (&v)[32]) {
    float* row = stage + slot * 32;
    const int sw = slot & 7;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<float4*>(row + ((c ^ sw) << 2)) = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

__device__ __forceinline__ float staged(const float* stage, int slot, int k) {
    return stage[slot * 32 + ((((k >> 2) ^ (slot & 7))) << 2) + (k & 3)];
}

// b^e for b > 0 (0 for b <= 0), as 2^(e log2 b) with the hardware base-2 approximations
// lg2.approx and ex2.approx (close to fp32 precision; the result's relative error grows with
// |e log2 b|).
__device__ __forceinline__ float pow_pos(float b, float e) {
    float l, r;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(b));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(e * l));
    return b > 0.f ? r : 0.f;
}

// ------------------------------------------------------------ packed fp32 pairs (sm_100 f32x2)
// Two fp32 values in one 64-bit register pair: lane x in the low half, y in the high half.  The
// f32x2 arithmetic instructions round each lane as their scalar forms do.
__device__ __forceinline__ uint64_t f2pack(float x, float y) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& x, float& y) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// max(v, 0) lane by lane
__device__ __forceinline__ uint64_t f2relu(uint64_t v) {
    float x, y;
    f2unpack(v, x, y);
    return f2pack(fmaxf(x, 0.f), fmaxf(y, 0.f));
}

// A pair of fp32 values as two bf16 pairs hi + lo (x = hi + lo to about 16 significant bits): hi
// keeps each value's top 16 bits (truncation, exact in fp32), lo = bf16(x - hi) rounded to nearest
// even.  Lane x goes to the low bf16 of each word, lane y to the high one.
__device__ __forceinline__ void f2split(uint64_t v, uint32_t& hi, uint32_t& lo) {
    float x, y;
    f2unpack(v, x, y);
    const uint32_t xt = __float_as_uint(x) & 0xffff0000u, yt = __float_as_uint(y) & 0xffff0000u;
    hi = __byte_perm(xt, yt, 0x7632);  // {x_hi16, y_hi16}
    const uint64_t r = f2sub(v, f2pack(__uint_as_float(xt), __uint_as_float(yt)));
    float rx, ry;
    f2unpack(r, rx, ry);
    __nv_bfloat162 b = __floats2bfloat162_rn(rx, ry);
    lo = *reinterpret_cast<uint32_t*>(&b);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// a += sum over list slots e in [ea0, ea1) of w[e] * X[j[e]][2 lane .. 2 lane + 1] for the list in
// column ca of the [slot][TILE] arrays cj (key index) and cw (weight), and b likewise for column cb;
// the two lists go together, eight slots each per step, so a warp keeps sixteen gathered rows in
// flight.
__device__ __forceinline__ void gather_accumulate2(const __nv_bfloat16* __restrict__ X, const uint16_t* cj,
                                                   const float* cw, int ca, int ea0, int ea1, int cb, int eb0,
                                                   int eb1, int lane, float& a0, float& a1, float& b0, float& b1) {
    for (int ea = ea0, eb = eb0; ea < ea1 || eb < eb1; ea += 8, eb += 8) {
        uint32_t xa[8], xb[8];
        float wa[8], wb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const bool oka = ea + u < ea1, okb = eb + u < eb1;
            const int ja = oka ? (int)cj[(ea + u) * TILE + ca] : 0;
            const int jb = okb ? (int)cj[(eb + u) * TILE + cb] : 0;
            wa[u] = oka ? cw[(ea + u) * TILE + ca] : 0.f;
            wb[u] = okb ? cw[(eb + u) * TILE + cb] : 0.f;
            xa[u] = oka ? __ldg(reinterpret_cast<const uint32_t*>(X + (size_t)ja * HEAD_DIM) + lane) : 0u;
            xb[u] = okb ? __ldg(reinterpret_cast<const uint32_t*>(X + (size_t)jb * HEAD_DIM) + lane) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            a0 = fmaf(wa[u], bf16lo(xa[u]), a0);
            a1 = fmaf(wa[u], bf16hi(xa[u]), a1);
            b0 = fmaf(wb[u], bf16lo(xb[u]), b0);
            b1 = fmaf(wb[u], bf16hi(xb[u]), b1);
        }
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace entmax
