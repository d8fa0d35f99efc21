// bwd_saved.cu -- backward pass of 1.5-entmax attention from the forward's saved supports.
//
// Same closed-form Jacobian as bwd.cu (page "svd-sst2-roberta-adasplash", section 2.4):
//   dA_ij = dO_i . V_j,  sp_ij = sqrt(p_ij),  u_i = sum_j sp_ij dA_ij / sum_j sp_ij,
//   dS_ij = sp_ij (dA_ij - u_i),  dQ_i = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i,
//   dV_j = sum_i p_ij dO_i,
// but the supports {(j, sp_ij)} come from entmax_attn_fwd_train instead of a recomputed score pass,
// so no QK^T is formed again: the work is proportional to the number of support entries.
//
//  1. key_scan:   per head, exclusive scan of the per-key support counts -> bucket offsets.
//  2. rows:       one warp per query row.  dA_ij with one support entry per lane (each lane reads a
//                 whole V row, 8 x 16-byte loads), u_i, dS_ij, dQ_i (lanes over dimensions), and the
//                 entries (i, sp_ij, dS_ij) scattered into per-key buckets.
//  3. keys:       one warp per key: dK_j and dV_j from its bucket (gathered Q_i, dO_i rows).
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

__device__ __forceinline__ float dot64_smem(const float* g, const __nv_bfloat16* row) {
    const uint4* p = reinterpret_cast<const uint4*>(row);
    uint4 w[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) w[c] = __ldg(p + c);
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 ga = reinterpret_cast<const float4*>(g)[2 * c];
        const float4 gb = reinterpret_cast<const float4*>(g)[2 * c + 1];
        acc0 = fmaf(ga.x, bf16lo(w[c].x), acc0);
        acc1 = fmaf(ga.y, bf16hi(w[c].x), acc1);
        acc0 = fmaf(ga.z, bf16lo(w[c].y), acc0);
        acc1 = fmaf(ga.w, bf16hi(w[c].y), acc1);
        acc0 = fmaf(gb.x, bf16lo(w[c].z), acc0);
        acc1 = fmaf(gb.y, bf16hi(w[c].z), acc1);
        acc0 = fmaf(gb.z, bf16lo(w[c].w), acc0);
        acc1 = fmaf(gb.w, bf16hi(w[c].w), acc1);
    }
    return acc0 + acc1;
}

__global__ void __launch_bounds__(1024) key_scan_kernel(const int* __restrict__ key_cnt, int* __restrict__ key_off,
                                                        int* __restrict__ key_cur, int L) {
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

__global__ void __launch_bounds__(ROW_WARPS * 32) saved_rows_kernel(const AttnArgs a, const BwdIO io,
                                                                    const SavedSupport sv, const SavedBwdWs ws) {
    __shared__ __align__(16) float gsm[ROW_WARPS][HEAD_DIM];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.L;
    const long long R = (long long)a.B * a.H * L;
    const size_t cap = (size_t)L * SAVE_CAP;
    const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
    const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(a.V);
    const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
    float* gs = gsm[warp];
    for (long long row = (long long)blockIdx.x * ROW_WARPS + warp; row < R; row += (long long)gridDim.x * ROW_WARPS) {
        const int cnt = sv.row_cnt[row];
        if (cnt < 0) continue;  // not saved: the exact pass handles this row
        const long long bh = row / L;
        const int i = (int)(row - bh * L);
        const size_t head = (size_t)bh * L * HEAD_DIM;
        const uint32_t gw = reinterpret_cast<const uint32_t*>(dO + (size_t)row * HEAD_DIM)[lane];
        gs[2 * lane] = bf16lo(gw);
        gs[2 * lane + 1] = bf16hi(gw);
        __syncwarp();
        // dA_ij: one support entry per lane
        int jj[2] = {0, 0};
        float sp[2] = {0.f, 0.f}, dA[2] = {0.f, 0.f};
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            if (b * 32 < cnt) {  // uniform
                const int e = b * 32 + lane;
                if (e < cnt) {
                    jj[b] = sv.row_j[(size_t)row * SAVE_CAP + e];
                    sp[b] = sv.row_sp[(size_t)row * SAVE_CAP + e];
                    dA[b] = dot64_smem(gs, V + head + (size_t)jj[b] * HEAD_DIM);
                }
            }
        }
        const float rs = warp_sum(sp[0] + sp[1]);
        const float wsum = warp_sum(fmaf(sp[0], dA[0], sp[1] * dA[1]));
        const float u = rs > 0.f ? wsum / rs : 0.f;
        const float ds[2] = {sp[0] * (dA[0] - u), sp[1] * (dA[1] - u)};
        // dQ_i = scale sum_e dS_e K_je, lanes over dimensions, eight gathered rows in flight
        float q0 = 0.f, q1 = 0.f;
        for (int e0 = 0; e0 < cnt; e0 += 8) {
            uint32_t kw[8];
            float dsv[8];
#pragma unroll
            for (int u8 = 0; u8 < 8; ++u8) {
                const int e = e0 + u8;
                const int b = e >> 5;  // uniform
                const int j = __shfl_sync(0xffffffffu, b == 0 ? jj[0] : jj[1], e & 31);
                const float d = __shfl_sync(0xffffffffu, b == 0 ? ds[0] : ds[1], e & 31);
                const bool ok = e < cnt;
                dsv[u8] = ok ? d : 0.f;
                kw[u8] = ok ? __ldg(reinterpret_cast<const uint32_t*>(K + head + (size_t)j * HEAD_DIM) + lane) : 0u;
            }
#pragma unroll
            for (int u8 = 0; u8 < 8; ++u8) {
                q0 = fmaf(dsv[u8], bf16lo(kw[u8]), q0);
                q1 = fmaf(dsv[u8], bf16hi(kw[u8]), q1);
            }
        }
        *reinterpret_cast<float2*>(io.dQ + (size_t)row * HEAD_DIM + 2 * lane) = make_float2(a.scale * q0, a.scale * q1);
        // (i, sp, dS) into key j's bucket
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const int e = b * 32 + lane;
            if (e < cnt) {
                const size_t key = (size_t)bh * L + jj[b];
                const size_t at = (size_t)bh * cap + (size_t)ws.key_off[key] + (size_t)atomicAdd(ws.key_cur + key, 1);
                ws.bucket_i[at] = (uint32_t)i;
                ws.bucket_sp[at] = sp[b];
                ws.bucket_ds[at] = ds[b];
            }
        }
        __syncwarp();  // gs is rewritten for the next row
    }
}

__global__ void __launch_bounds__(ROW_WARPS * 32) saved_keys_kernel(const AttnArgs a, const BwdIO io,
                                                                    const SavedSupport sv, const SavedBwdWs ws) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.L;
    const long long R = (long long)a.B * a.H * L;
    const size_t cap = (size_t)L * SAVE_CAP;
    const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
    const __nv_bfloat16* dO = reinterpret_cast<const __nv_bfloat16*>(io.dO);
    for (long long key = (long long)blockIdx.x * ROW_WARPS + warp; key < R; key += (long long)gridDim.x * ROW_WARPS) {
        const int n = sv.key_cnt[key];
        const long long bh = key / L;
        const size_t head = (size_t)bh * L * HEAD_DIM;
        const size_t b0 = (size_t)bh * cap + (size_t)ws.key_off[key];
        float k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
        for (int e0 = 0; e0 < n; e0 += 32) {
            const int e = e0 + lane;
            const bool valid = e < n;
            const uint32_t ii = valid ? ws.bucket_i[b0 + e] : 0u;
            const float sp = valid ? ws.bucket_sp[b0 + e] : 0.f;
            const float ds = valid ? ws.bucket_ds[b0 + e] : 0.f;
            const int m = min(32, n - e0);
            for (int t0 = 0; t0 < m; t0 += 8) {
                uint32_t gw[8], qw[8];
                float pv[8], dv[8];
#pragma unroll
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int t = t0 + u8;
                    const uint32_t it = __shfl_sync(0xffffffffu, ii, t & 31);
                    const float st = __shfl_sync(0xffffffffu, sp, t & 31);
                    const float dt = __shfl_sync(0xffffffffu, ds, t & 31);
                    const bool ok = t < m;
                    pv[u8] = ok ? st * st : 0.f;
                    dv[u8] = ok ? dt : 0.f;
                    gw[u8] = ok ? __ldg(reinterpret_cast<const uint32_t*>(dO + head + (size_t)it * HEAD_DIM) + lane) : 0u;
                    qw[u8] = ok ? __ldg(reinterpret_cast<const uint32_t*>(Q + head + (size_t)it * HEAD_DIM) + lane) : 0u;
                }
#pragma unroll
                for (int u8 = 0; u8 < 8; ++u8) {
                    v0 = fmaf(pv[u8], bf16lo(gw[u8]), v0);
                    v1 = fmaf(pv[u8], bf16hi(gw[u8]), v1);
                    k0 = fmaf(dv[u8], bf16lo(qw[u8]), k0);
                    k1 = fmaf(dv[u8], bf16hi(qw[u8]), k1);
                }
            }
        }
        *reinterpret_cast<float2*>(io.dK + (size_t)key * HEAD_DIM + 2 * lane) = make_float2(a.scale * k0, a.scale * k1);
        *reinterpret_cast<float2*>(io.dV + (size_t)key * HEAD_DIM + 2 * lane) = make_float2(v0, v1);
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
__global__ void __launch_bounds__(UNSAVED_THREADS) unsaved_rows_kernel(const AttnArgs a, const BwdIO io,
                                                                      const SavedSupport sv) {
    extern __shared__ float sbuf[];  // [L]: sqrt(p_ij); [L, 2L): dA_ij
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
        const size_t head = (size_t)bh * L * HEAD_DIM;
        __syncthreads();
        if (tid < HEAD_DIM) {
            qf[tid] = __bfloat162float(Q[(size_t)row * HEAD_DIM + tid]);
            gf[tid] = __bfloat162float(dO[(size_t)row * HEAD_DIM + tid]);
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
                const float s = a.scale * dot64_f32(qf, K + head + (size_t)j * HEAD_DIM);
                sp = fmaxf(0.5f * (s - tau), 0.f);
            }
            float dA = 0.f;
            if (sp > 0.f) {
                dA = dot64_f32(gf, V + head + (size_t)j * HEAD_DIM);
                r += sp;
                w = fmaf(sp, dA, w);
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
                const size_t key = (size_t)bh * L + lo + e;
                const float ds = sp * (sbuf[L + e] - u);
                acc = fmaf(ds, __bfloat162float(K[key * HEAD_DIM + d]), acc);
                atomicAdd(io.dK + key * HEAD_DIM + d, a.scale * ds * qf[d]);
                atomicAdd(io.dV + key * HEAD_DIM + d, sp * sp * gf[d]);
            }
        }
        __syncthreads();
        red[tid] = acc;
        __syncthreads();
        if (tid < HEAD_DIM) {
            float q = 0.f;
#pragma unroll
            for (int p = 0; p < PH; ++p) q += red[tid + p * HEAD_DIM];
            io.dQ[(size_t)row * HEAD_DIM + tid] = a.scale * q;
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
    key_scan_kernel<<<a.B * a.H, 1024, 0, stream>>>(sv.key_cnt, ws.key_off, ws.key_cur, a.L);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>((R + ROW_WARPS - 1) / ROW_WARPS, (long long)sms * 8));
    saved_rows_kernel<<<grid, ROW_WARPS * 32, 0, stream>>>(a, io, sv, ws);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    saved_keys_kernel<<<grid, ROW_WARPS * 32, 0, stream>>>(a, io, sv, ws);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int smem = 2 * a.L * (int)sizeof(float);
    e = ensure_smem_attr(reinterpret_cast<const void*>(unsaved_rows_kernel), 2 * MAX_L * (int)sizeof(float), 3);
    if (e != cudaSuccess) return e;
    unsaved_rows_kernel<<<(unsigned)sms, UNSAVED_THREADS, smem, stream>>>(a, io, sv);
    return cudaGetLastError();
}

}  // namespace entmax
