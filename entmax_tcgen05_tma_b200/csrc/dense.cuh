// dense.cuh -- geometry and helpers of the tensor-core kernels that walk every (query, key) tile
// of a row's allowed range (bwd_dense.cu, fwd_softmax.cu).
//
// Roles (320 threads, two CTAs per SM): warps 0-7 epilogue -- thread (g, r) serves TMEM lane and
// tile row r and columns [32 g, 32 g + 32) of each 64-column block, so each row's work is split
// over two warps; warp 8 TMA producer (and TMEM allocation); warp 9 MMA issuer.  Streamed blocks
// are 64 rows of 64 bf16 (8 KiB, 128-byte swizzle); a product's A operand of bf16 parts is written
// by the epilogue into TMEM (tcgen05.st): for block columns 16 k .. 16 k + 15 the hi parts sit in
// packed column 16 k and the lo parts in 16 k + 8 of the set that held the block's fp32 tile.
#pragma once
#include <cuda_bf16.h>
#include "common.cuh"

namespace entmax {
namespace dense {

constexpr int THREADS = 320;
constexpr int NUM_EPI = 256;          // epilogue threads: two per tile row
constexpr int W_PROD = 8, W_MMA = 9;
constexpr int TMEM_COLS_D = 256;
constexpr int BK = 64;                // rows of a streamed block
constexpr int HB = BK / 2;            // columns of a block per epilogue thread
constexpr int SUB = 16;               // columns an epilogue thread holds at a time
constexpr int BLK_ROW_BYTES = BK * HEAD_DIM * 2;   // 8 KiB: one streamed [64][64] bf16 block
constexpr float LOG2E = 1.4426950408889634f;     // log2(e): exp(x) = 2^(x log2 e)
constexpr float LN2 = 0.6931471805599453f;       // ln(2)

using BlockList = Pipe<BK, 2, 2, 1>;  // only its block-list builder (64-key blocks)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Bounded wait whose outcome the whole warp shares.
__device__ __forceinline__ bool warp_wait_d(uint32_t bar, uint32_t parity, int* abort_flag, const WaitCfg& wc) {
    return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, wc));
}

// Named barrier over the 8 epilogue warps (id 1; 0 is __syncthreads).
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(NUM_EPI) : "memory"); }

// Zeroes lane x (y) of a pair unless bit k (k + 1) of vm is set.
__device__ __forceinline__ uint64_t f2mask(uint64_t v, uint32_t vm, int k) {
    float x, y;
    f2unpack(v, x, y);
    return f2pack(((vm >> k) & 1u) ? x : 0.f, ((vm >> (k + 1)) & 1u) ? y : 0.f);
}

// 2^x lane by lane (exp2f: at most 2 ulp from the exact power).
__device__ __forceinline__ uint64_t f2exp2(uint64_t v) {
    float x, y;
    f2unpack(v, x, y);
    return f2pack(exp2f(x), exp2f(y));
}

// Weight w of a pair of raw scores s (S = scale s) given the row constants k = wslope(scale) and
// c = woffset(tau):
//   1.5-entmax  w = sqrt(p) = max(0, (S - tau) / 2)           k = scale / 2,       c = -tau / 2
//   softmax     w = p = exp(S - tau) = 2^(S log2 e - tau log2 e)  k = scale log2 e,  c = -tau log2 e
// The backward's Jacobian is w (dA - u) in both cases, u = sum w dA / sum w, and P = w^2 or w.
// A row with no allowed key has tau = +inf, so c = -inf and w = 0.
template <bool kSoftmax>
__device__ __forceinline__ float wslope(float scale) { return kSoftmax ? scale * LOG2E : 0.5f * scale; }
template <bool kSoftmax>
__device__ __forceinline__ float woffset(float tau) { return kSoftmax ? -tau * LOG2E : -0.5f * tau; }
template <bool kSoftmax>
__device__ __forceinline__ uint64_t weight2(uint64_t s2, uint64_t k2, uint64_t c2) {
    const uint64_t x = f2fma(s2, k2, c2);
    if constexpr (kSoftmax) return f2exp2(x);
    else return f2relu(x);
}

// MMA thread: commit to `bar` (phase parity `par`) and remember it as the last commit.
__device__ __forceinline__ void commit_to(uint64_t* bar, uint32_t par, uint32_t* last_bar, uint32_t* last_par) {
    tc_commit(smem_u32(bar));
    *last_bar = smem_u32(bar);
    *last_par = par;
}

// Teardown after an abort, past the CTA's teardown barrier: the producer thread waits for the
// fixed tiles and its last ns streamed loads, the MMA thread for its last commit.
__device__ __forceinline__ void drain_dense(uint64_t* full_a, uint64_t* full, int ns, int nload, uint32_t last_bar,
                                            uint32_t last_par, int warp, int lane) {
    if (lane != 0) return;
    if (warp == W_PROD) {
        wait_drain(smem_u32(full_a), 0);
        for (int m = max(0, nload - ns); m < nload; ++m) wait_drain(smem_u32(&full[m % ns]), (uint32_t)(m / ns) & 1u);
    }
    if (warp == W_MMA && last_bar) wait_drain(last_bar, last_par);
}

}  // namespace dense
}  // namespace entmax
