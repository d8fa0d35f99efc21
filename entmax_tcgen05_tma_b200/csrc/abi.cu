// abi.cu -- the extern "C" entry points of libentmax_attn.so: argument checks, tensor maps,
// the device status word, fp32-input conversion, and kernel launches.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <atomic>
#include <mutex>
#include "../../include/entmax_attn.h"
#include "common.cuh"
#include "internal.h"

namespace entmax {

namespace {

__device__ int g_device_status;  // ENTMAX_OK or the first device-side error since the last read

constexpr unsigned long long DEFAULT_TIMEOUT_NS = 2000000000ull;
// process-wide settings and the last error: calls may come from several host threads
std::atomic<unsigned long long> g_timeout_ns{DEFAULT_TIMEOUT_NS};
std::atomic<int> g_last_cuda_error{0};

unsigned long long timeout_ns() { return g_timeout_ns.load(std::memory_order_relaxed); }

constexpr int MAX_DEVICES = 64;
int* g_status_ptr[MAX_DEVICES] = {};
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;

// Driver entry point `name` (version `ver`) through the runtime, once; under g_mu.
template <class F>
cudaError_t driver_fn(F* out, const char* name, int ver) {
    if (*out) return cudaSuccess;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion(name, &fn, ver, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    *out = reinterpret_cast<F>(fn);
    return cudaSuccess;
}

int record(cudaError_t e) {
    if (e == cudaSuccess) return ENTMAX_OK;
    g_last_cuda_error.store((int)e, std::memory_order_relaxed);
    return ENTMAX_ERR_CUDA;
}

// The calling thread's device, with a context current on it.  The tensor-map encoder (a driver call
// outside the runtime) needs a current context, and a host thread that has not used CUDA yet -- a new
// thread, or a framework's autograd worker whose first CUDA work is a call here -- has none until
// the runtime makes one current on its first stream operation.  So when no context is current, the
// device's primary context is made current (cudaSetDevice); a context the caller made current is
// left as it is.
cudaError_t current_device(int* dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    if (*dev < 0 || *dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        e = driver_fn(&g_ctx_current, "cuCtxGetCurrent", 4000);
    }
    if (e != cudaSuccess) return e;
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) == CUDA_SUCCESS && ctx) return cudaSuccess;
    return cudaSetDevice(*dev);
}

cudaError_t status_ptr(int** out) {
    int dev = 0;
    cudaError_t e = current_device(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_status);
        if (e != cudaSuccess) return e;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    *out = g_status_ptr[dev];
    return cudaSuccess;
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (; i < n; i += stride) dst[i] = __float2bfloat16_rn(src[i]);
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align256b(size_t n) { return (n + 255) & ~size_t(255); }

// entmax_attn_bwd's workspace: the minimum holds one float per row (the row scalar u_i); with
// room for the saved supports and the saved backward's buckets, rows that are not on the
// tensor-core path rebuild their supports from tau (support extraction) and take the support-list
// backward.
size_t bwd_min_ws_bytes(long long R) { return align256b((size_t)R * sizeof(float)); }
size_t bwd_rebuild_ws_bytes(long long R) { return saved_support_bytes(R) + saved_bwd_ws_bytes(R); }

int check_common(const void* Q, const void* K, const void* V, int in_dtype, int causal, int window, float scale,
                 int B, int H, int L, int D) {
    if (B < 0 || H < 0 || L < 0) return ENTMAX_ERR_ARG;
    if (in_dtype != ENTMAX_BF16 && in_dtype != ENTMAX_F32) return ENTMAX_ERR_ARG;
    if (!(scale > 0.f) || !isfinite(scale)) return ENTMAX_ERR_ARG;
    if (window < 0 || (causal != 0 && causal != 1)) return ENTMAX_ERR_ARG;
    if (D != HEAD_DIM) return ENTMAX_ERR_UNSUPPORTED;
    if (window > 0 && !causal) return ENTMAX_ERR_UNSUPPORTED;
    if (L > MAX_L) return ENTMAX_ERR_UNSUPPORTED;
    if ((long long)B * H > 65535) return ENTMAX_ERR_UNSUPPORTED;
    if (B == 0 || H == 0 || L == 0) return ENTMAX_OK;
    if (!Q || !K || !V) return ENTMAX_ERR_ARG;
    if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16)) return ENTMAX_ERR_ARG;
    return ENTMAX_OK;
}

// bf16 copies of fp32 inputs, in stream-ordered temporaries.
struct Bf16Copies {
    void* buf = nullptr;
    cudaStream_t stream = nullptr;
    ~Bf16Copies() {
        if (buf) cudaFreeAsync(buf, stream);
    }
};

cudaError_t convert_inputs(const void* const* src, const void** dst, int count, size_t n_each, Bf16Copies& tmp,
                           cudaStream_t stream) {
    tmp.stream = stream;
    const size_t bytes_each = n_each * 2;
    const size_t pitch = (bytes_each + 255) & ~size_t(255);
    cudaError_t e = cudaMallocAsync(&tmp.buf, pitch * count, stream);
    if (e != cudaSuccess) {
        tmp.buf = nullptr;
        return e;
    }
    for (int k = 0; k < count; ++k) {
        void* d = static_cast<uint8_t*>(tmp.buf) + pitch * k;
        e = launch_f32_to_bf16(static_cast<const float*>(src[k]), d, n_each, stream);
        if (e != cudaSuccess) return e;
        dst[k] = d;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_f32_to_bf16(const float* src, void* dst, size_t n, cudaStream_t stream) {
    const int threads = 256;
    const size_t blocks = std::min<size_t>((n + threads - 1) / threads, 148 * 16);
    f32_to_bf16_kernel<<<(unsigned)std::max<size_t>(blocks, 1), threads, 0, stream>>>(
        src, static_cast<__nv_bfloat16*>(dst), n);
    return cudaGetLastError();
}

cudaError_t ensure_smem_attr(const void* func, int bytes, int slot) {
    constexpr int SLOTS = 16;
    static std::atomic<bool> done[SLOTS][MAX_DEVICES] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= MAX_DEVICES || slot < 0 || slot >= SLOTS) return cudaErrorInvalidValue;
    if (done[slot][dev].load(std::memory_order_acquire)) return cudaSuccess;
    // setting the attributes twice (two threads racing here) is harmless
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    // the whole unified L1/shared array as shared memory, so kernels sized for two CTAs per SM get two
    if (e == cudaSuccess) e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess) done[slot][dev].store(true, std::memory_order_release);
    return e;
}

cudaError_t make_tile_map(CUtensorMap* map, const void* base, int layout, int B, int nh, int L, int box_rows) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        cudaError_t e = driver_fn(&g_encode, "cuTensorMapEncodeTiled", 12000);
        if (e != cudaSuccess) return e;
    }
    // layout 0 [B, nh, L, 64]: (d, L, B*nh); layout 1 [B, L, nh, 64]: (d, nh, B*L) -- see HeadRef
    const cuuint64_t row_bytes = (cuuint64_t)HEAD_DIM * 2;
    const cuuint64_t dims[3] = {(cuuint64_t)HEAD_DIM, (cuuint64_t)(layout ? nh : L),
                                (cuuint64_t)(layout ? (long long)B * L : (long long)B * nh)};
    const cuuint64_t strides[2] = {row_bytes, (layout ? (cuuint64_t)nh : (cuuint64_t)L) * row_bytes};
    const cuuint32_t box[3] = {(cuuint32_t)HEAD_DIM, layout ? 1u : (cuuint32_t)box_rows, layout ? (cuuint32_t)box_rows : 1u};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r == CUDA_SUCCESS) return cudaSuccess;
    return r == CUDA_ERROR_INVALID_CONTEXT ? cudaErrorDeviceUninitialized : cudaErrorInvalidValue;
}

}  // namespace entmax

using namespace entmax;

extern "C" {

int entmax_attn_version(void) { return 100; }

const char* entmax_attn_strerror(int status) {
    switch (status) {
        case ENTMAX_OK: return "ok";
        case ENTMAX_ERR_ARG: return "invalid argument";
        case ENTMAX_ERR_UNSUPPORTED: return "unsupported configuration";
        case ENTMAX_ERR_CUDA: return "CUDA error";
        case ENTMAX_ERR_TIMEOUT: return "device wait timed out";
        case ENTMAX_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

int entmax_attn_last_cuda_error(void) { return g_last_cuda_error.load(std::memory_order_relaxed); }

void entmax_attn_set_wait_timeout_ns(unsigned long long ns) {
    g_timeout_ns.store(ns ? ns : DEFAULT_TIMEOUT_NS, std::memory_order_relaxed);
}

int entmax_attn_device_status(cudaStream_t stream) {
    int* p = nullptr;
    int rc = record(status_ptr(&p));
    if (rc) return rc;
    rc = record(cudaStreamSynchronize(stream));
    if (rc) return rc;
    int v = 0;
    rc = record(cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost));
    if (rc) return rc;
    const int zero = 0;
    rc = record(cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice));
    if (rc) return rc;
    return v;
}

}  // extern "C"

namespace {
// Key/value head count check of the grouped-query entry points.  Grouped inputs must be bf16 (fp32
// inputs would need per-tensor conversion sizes).
int check_kv_heads(int H, int Hkv, int in_dtype) {
    if (Hkv < 0) return ENTMAX_ERR_ARG;
    if (H == 0 || Hkv == 0) return H == Hkv ? ENTMAX_OK : ENTMAX_ERR_ARG;
    if (H % Hkv != 0) return ENTMAX_ERR_ARG;
    if (Hkv != H && in_dtype != ENTMAX_BF16) return ENTMAX_ERR_UNSUPPORTED;
    return ENTMAX_OK;
}

// alpha of alpha-entmax: [1, 2].  Like the pages' entmax_bisect routine (page
// "svd-sst2-roberta-adasplash", section 4), |alpha - 1| < 1e-4 means softmax; am1 (alpha - 1) is then
// exactly 0, the kernels' softmax flag.
int check_alpha(float alpha, float* am1) {
    if (fabsf(alpha - 1.f) < 1e-4f) {
        *am1 = 0.f;
        return ENTMAX_OK;
    }
    if (!(alpha > 1.f && alpha <= 2.f)) return ENTMAX_ERR_ARG;
    *am1 = alpha - 1.f;
    return ENTMAX_OK;
}

int fwd_impl(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask, int causal,
             int window, float scale, float alpha, int B, int H, int Hkv, int L, int D, int layout, void* O,
             int out_dtype, float* tau, cudaStream_t stream, float* otil = nullptr, float* rsum = nullptr) {
    int rc = check_common(Q, K, V, in_dtype, causal, window, scale, B, H, L, D);
    if (rc) return rc;
    float am1 = 0.5f;
    rc = check_alpha(alpha, &am1);
    if (rc) return rc;
    if (layout != ENTMAX_LAYOUT_BHLD && layout != ENTMAX_LAYOUT_BLHD) return ENTMAX_ERR_ARG;
    rc = check_kv_heads(H, Hkv, in_dtype);
    if (rc) return rc;
    if (out_dtype != ENTMAX_BF16 && out_dtype != ENTMAX_F32) return ENTMAX_ERR_ARG;
    if (B == 0 || H == 0 || L == 0) return ENTMAX_OK;
    if (!O || !tau) return ENTMAX_ERR_ARG;
    if (!aligned(O, 16) || !aligned(tau, 4)) return ENTMAX_ERR_ARG;
    int* status = nullptr;
    rc = record(status_ptr(&status));
    if (rc) return rc;

    const size_t n = (size_t)B * H * L * HEAD_DIM;
    AttnArgs a{Q, K, V, key_mask, B, H, L, causal, window, scale, status, timeout_ns(), Hkv, am1, layout};
    Bf16Copies tmp;
    if (in_dtype == ENTMAX_F32) {
        const void* src[3] = {Q, K, V};
        const void* dst[3];
        rc = record(convert_inputs(src, dst, 3, n, tmp, stream));
        if (rc) return rc;
        a.Q = dst[0];
        a.K = dst[1];
        a.V = dst[2];
    }
    FwdOut o{O, out_dtype == ENTMAX_F32, tau, SavedSupport{}, otil, rsum};
    if (softmax_alpha(a)) return record(launch_fwd_softmax(a, o, stream));
    // the auxiliary rows come from the gather forward alone
    if (dense_fwd(a) && !otil) return record(launch_fwd_dense(a, o, stream));
    return record(launch_fwd(a, o, stream));
}
}  // namespace

extern "C" {

int entmax_attn_fwd(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask, int causal,
                    int window, float scale, int B, int H, int L, int D, void* O, int out_dtype, float* tau,
                    cudaStream_t stream) {
    return fwd_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, 1.5f, B, H, H, L, D, 0, O, out_dtype,
                    tau, stream);
}

int entmax_attn_fwd_gqa(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask,
                        int causal, int window, float scale, int B, int H, int Hkv, int L, int D, void* O,
                        int out_dtype, float* tau, cudaStream_t stream) {
    return fwd_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, 1.5f, B, H, Hkv, L, D, 0, O, out_dtype,
                    tau, stream);
}

size_t entmax_attn_bwd_workspace_size(int B, int H, int L, int D) {
    (void)D;
    if (B <= 0 || H <= 0 || L <= 0) return 0;
    const long long R = (long long)B * H * L;
    // rows of at most 512 keys always take the tensor-core backward, which needs the minimum only
    return L <= 512 ? bwd_min_ws_bytes(R) : std::max(bwd_min_ws_bytes(R), bwd_rebuild_ws_bytes(R));
}

}  // extern "C"

namespace {
int bwd_impl(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask, int causal,
             int window, float scale, int B, int H, int L, int D, const float* tau, const void* dO, float* dQ,
             float* dK, float* dV, void* workspace, size_t ws_bytes, cudaStream_t stream,
             const float* otil = nullptr, const float* rsum = nullptr) {
    int rc = check_common(Q, K, V, in_dtype, causal, window, scale, B, H, L, D);
    if (rc) return rc;
    if (B == 0 || H == 0 || L == 0) return ENTMAX_OK;
    if (!tau || !dO || !dQ || !dK || !dV) return ENTMAX_ERR_ARG;
    if (!aligned(dO, 16) || !aligned(dQ, 8) || !aligned(dK, 8) || !aligned(dV, 8) || !aligned(tau, 4))
        return ENTMAX_ERR_ARG;
    const long long R = (long long)B * H * L;
    if (!workspace || ws_bytes < bwd_min_ws_bytes(R)) return ENTMAX_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return ENTMAX_ERR_ARG;
    int* status = nullptr;
    rc = record(status_ptr(&status));
    if (rc) return rc;

    const size_t n = (size_t)B * H * L * HEAD_DIM;
    AttnArgs a{Q, K, V, key_mask, B, H, L, causal, window, scale, status, timeout_ns(), H, 0.5f, 0};
    BwdIO io{tau, dO, dQ, dK, dV, static_cast<float*>(workspace), otil, rsum};
    Bf16Copies tmp;
    if (in_dtype == ENTMAX_F32) {
        const void* src[4] = {Q, K, V, dO};
        const void* dst[4];
        rc = record(convert_inputs(src, dst, 4, n, tmp, stream));
        if (rc) return rc;
        a.Q = dst[0];
        a.K = dst[1];
        a.V = dst[2];
        io.dO = dst[3];
    }
    // the tensor-core kernels and the support-list backward store gradient rows 16 bytes at a time
    const bool g16 = aligned(dQ, 16) && aligned(dK, 16) && aligned(dV, 16);
    if (dense_bwd(a) && g16) return record(launch_bwd_dense(a, io, stream));
    if (!otil && g16 && ws_bytes >= bwd_rebuild_ws_bytes(R) && aligned(workspace, 256)) {
        // Rebuild the forward's supports from the caller's tau: one score pass on the tensor cores,
        // cut at tau_i, lists each row's support into the workspace; then the support-list backward.
        uint8_t* p = static_cast<uint8_t*>(workspace);
        const SavedSupport sv = carve_saved(p, R);
        p += saved_support_bytes(R);
        rc = record(cudaMemsetAsync(sv.key_cnt, 0, sizeof(int) * (size_t)R, stream));
        if (rc) return rc;
        rc = record(cudaMemsetAsync(sv.unsaved_cnt, 0, sizeof(int), stream));
        if (rc) return rc;
        FwdOut o{nullptr, 0, const_cast<float*>(tau), sv};  // tau is only read in extraction
        rc = record(launch_fwd(a, o, stream, true));
        if (rc) return rc;
        io.u = nullptr;
        io.guard = status;  // if the extraction gave up, its lists hold anything: the backward does nothing
        return record(launch_bwd_saved(a, io, sv, carve_saved_bwd_ws(p, R), stream));
    }
    return record(launch_bwd(a, io, stream));
}
}  // namespace

extern "C" {

int entmax_attn_bwd(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask, int causal,
                    int window, float scale, int B, int H, int L, int D, const float* tau, const void* dO, float* dQ,
                    float* dK, float* dV, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    return bwd_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, B, H, L, D, tau, dO, dQ, dK, dV, workspace,
                    ws_bytes, stream);
}

int entmax_attn_fwd_aux(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask,
                        int causal, int window, float scale, int B, int H, int L, int D, void* O, int out_dtype,
                        float* tau, float* Otil, float* rsum, cudaStream_t stream) {
    if (B > 0 && H > 0 && L > 0 && (!Otil || !rsum || !aligned(Otil, 16) || !aligned(rsum, 4))) return ENTMAX_ERR_ARG;
    return fwd_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, 1.5f, B, H, H, L, D, 0, O, out_dtype, tau,
                    stream, Otil, rsum);
}

int entmax_attn_bwd_aux(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask,
                        int causal, int window, float scale, int B, int H, int L, int D, const float* tau,
                        const float* Otil, const float* rsum, const void* dO, float* dQ, float* dK, float* dV,
                        void* workspace, size_t ws_bytes, cudaStream_t stream) {
    if (B > 0 && H > 0 && L > 0 && (!Otil || !rsum || !aligned(Otil, 16) || !aligned(rsum, 4))) return ENTMAX_ERR_ARG;
    return bwd_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, B, H, L, D, tau, dO, dQ, dK, dV, workspace,
                    ws_bytes, stream, Otil, rsum);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Training path: the forward saves each row's support, the backward works from those lists.
extern "C" {

size_t entmax_attn_saved_bytes(int B, int H, int L, int D) {
    (void)D;
    if (B <= 0 || H <= 0 || L <= 0) return 0;
    return saved_support_bytes((long long)B * H * L);
}

size_t entmax_attn_bwd_saved_workspace_size(int B, int H, int L, int D) {
    (void)D;
    if (B <= 0 || H <= 0 || L <= 0) return 0;
    return saved_bwd_ws_bytes((long long)B * H * L);
}

}  // extern "C"

namespace {
int fwd_train_impl(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask, int causal,
                   int window, float scale, float alpha, int B, int H, int Hkv, int L, int D, int layout, void* O,
                   int out_dtype, float* tau, void* saved, size_t saved_bytes, cudaStream_t stream) {
    int rc = check_common(Q, K, V, in_dtype, causal, window, scale, B, H, L, D);
    if (rc) return rc;
    float am1 = 0.5f;
    rc = check_alpha(alpha, &am1);
    if (rc) return rc;
    if (layout != ENTMAX_LAYOUT_BHLD && layout != ENTMAX_LAYOUT_BLHD) return ENTMAX_ERR_ARG;
    rc = check_kv_heads(H, Hkv, in_dtype);
    if (rc) return rc;
    if (out_dtype != ENTMAX_BF16 && out_dtype != ENTMAX_F32) return ENTMAX_ERR_ARG;
    if (B == 0 || H == 0 || L == 0) return ENTMAX_OK;
    if (!O || !tau) return ENTMAX_ERR_ARG;
    if (!aligned(O, 16) || !aligned(tau, 4)) return ENTMAX_ERR_ARG;
    const long long R = (long long)B * H * L;
    if (!saved || saved_bytes < saved_support_bytes(R)) return ENTMAX_ERR_WORKSPACE;
    if (!aligned(saved, 256)) return ENTMAX_ERR_ARG;
    int* status = nullptr;
    rc = record(status_ptr(&status));
    if (rc) return rc;
    const size_t n = (size_t)R * HEAD_DIM;
    AttnArgs a{Q, K, V, key_mask, B, H, L, causal, window, scale, status, timeout_ns(), Hkv, am1, layout};
    // the tensor-core backward recomputes the scores and reads no support lists: none are saved
    // (it derives u_i in a pass of its own, which costs less than writing the auxiliary rows here)
    const bool save = !dense_bwd(a);
    const SavedSupport sv = save ? carve_saved(saved, R) : SavedSupport{};
    if (save) {
        rc = record(cudaMemsetAsync(sv.key_cnt, 0, sizeof(int) * (size_t)R, stream));
        if (rc) return rc;
        rc = record(cudaMemsetAsync(sv.unsaved_cnt, 0, sizeof(int), stream));
        if (rc) return rc;
    }
    Bf16Copies tmp;
    if (in_dtype == ENTMAX_F32) {
        const void* src[3] = {Q, K, V};
        const void* dst[3];
        rc = record(convert_inputs(src, dst, 3, n, tmp, stream));
        if (rc) return rc;
        a.Q = dst[0];
        a.K = dst[1];
        a.V = dst[2];
    }
    FwdOut o{O, out_dtype == ENTMAX_F32, tau, sv};
    if (softmax_alpha(a)) {
        // the saved buffer holds O in fp32, the softmax backward's auxiliary row (u_i = dO_i . O_i)
        static_assert(SAVE_CAP * 6 >= HEAD_DIM * 4, "the saved buffer holds an fp32 row of O");
        o.otil = static_cast<float*>(saved);
        return record(launch_fwd_softmax(a, o, stream));
    }
    return record(dense_fwd(a) ? launch_fwd_dense(a, o, stream) : launch_fwd(a, o, stream));
}

int bwd_saved_impl(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask, int causal,
                   int window, float scale, float alpha, int B, int H, int Hkv, int L, int D, int layout,
                   const float* tau, const void* saved, size_t saved_bytes, const void* dO, float* dQ, float* dK,
                   float* dV, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    int rc = check_common(Q, K, V, in_dtype, causal, window, scale, B, H, L, D);
    if (rc) return rc;
    float am1 = 0.5f;
    rc = check_alpha(alpha, &am1);
    if (rc) return rc;
    if (layout != ENTMAX_LAYOUT_BHLD && layout != ENTMAX_LAYOUT_BLHD) return ENTMAX_ERR_ARG;
    rc = check_kv_heads(H, Hkv, in_dtype);
    if (rc) return rc;
    if (B == 0 || H == 0 || L == 0) return ENTMAX_OK;
    if (!tau || !dO || !dQ || !dK || !dV) return ENTMAX_ERR_ARG;
    if (!aligned(dO, 16) || !aligned(dQ, 16) || !aligned(dK, 16) || !aligned(dV, 16) || !aligned(tau, 4))
        return ENTMAX_ERR_ARG;
    const long long R = (long long)B * H * L;
    if (!saved || saved_bytes < saved_support_bytes(R)) return ENTMAX_ERR_WORKSPACE;
    if (!workspace || ws_bytes < saved_bwd_ws_bytes(R)) return ENTMAX_ERR_WORKSPACE;
    if (!aligned(saved, 256) || !aligned(workspace, 256)) return ENTMAX_ERR_ARG;
    int* status = nullptr;
    rc = record(status_ptr(&status));
    if (rc) return rc;
    const size_t n = (size_t)R * HEAD_DIM;
    AttnArgs a{Q, K, V, key_mask, B, H, L, causal, window, scale, status, timeout_ns(), Hkv, am1, layout};
    BwdIO io{tau, dO, dQ, dK, dV, nullptr};
    io.guard = status;  // a recorded device error (a forward that gave up): its lists are not read
    Bf16Copies tmp;
    if (in_dtype == ENTMAX_F32) {
        const void* src[4] = {Q, K, V, dO};
        const void* dst[4];
        rc = record(convert_inputs(src, dst, 4, n, tmp, stream));
        if (rc) return rc;
        a.Q = dst[0];
        a.K = dst[1];
        a.V = dst[2];
        io.dO = dst[3];
    }
    const SavedBwdWs ws = carve_saved_bwd_ws(workspace, R);
    if (dense_bwd(a)) {
        io.u = reinterpret_cast<float*>(ws.key_off);  // R floats of the workspace hold u
        if (softmax_alpha(a)) io.otil = static_cast<const float*>(saved);  // the forward's fp32 O
        return record(launch_bwd_dense(a, io, stream));
    }
    return record(launch_bwd_saved(a, io, carve_saved(const_cast<void*>(saved), R), ws, stream));
}
}  // namespace

extern "C" {

int entmax_attn_fwd_train(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask,
                          int causal, int window, float scale, int B, int H, int L, int D, void* O, int out_dtype,
                          float* tau, void* saved, size_t saved_bytes, cudaStream_t stream) {
    return fwd_train_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, 1.5f, B, H, H, L, D, 0, O, out_dtype,
                          tau, saved, saved_bytes, stream);
}

int entmax_attn_fwd_train_gqa(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask,
                              int causal, int window, float scale, int B, int H, int Hkv, int L, int D, void* O,
                              int out_dtype, float* tau, void* saved, size_t saved_bytes, cudaStream_t stream) {
    return fwd_train_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, 1.5f, B, H, Hkv, L, D, 0, O,
                          out_dtype, tau, saved, saved_bytes, stream);
}

int entmax_attn_bwd_saved(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask,
                          int causal, int window, float scale, int B, int H, int L, int D, const float* tau,
                          const void* saved, size_t saved_bytes, const void* dO, float* dQ, float* dK, float* dV,
                          void* workspace, size_t ws_bytes, cudaStream_t stream) {
    return bwd_saved_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, 1.5f, B, H, H, L, D, 0, tau, saved,
                          saved_bytes, dO, dQ, dK, dV, workspace, ws_bytes, stream);
}

int entmax_attn_bwd_saved_gqa(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask,
                              int causal, int window, float scale, int B, int H, int Hkv, int L, int D,
                              const float* tau, const void* saved, size_t saved_bytes, const void* dO, float* dQ,
                              float* dK, float* dV, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    return bwd_saved_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, 1.5f, B, H, Hkv, L, D, 0, tau, saved,
                          saved_bytes, dO, dQ, dK, dV, workspace, ws_bytes, stream);
}

int entmax_attn_fwd_ex(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask, int causal,
                       int window, float scale, float alpha, int B, int H, int Hkv, int L, int D, int layout, void* O,
                       int out_dtype, float* tau, void* saved, size_t saved_bytes, cudaStream_t stream) {
    if (!saved && saved_bytes == 0)
        return fwd_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, alpha, B, H, Hkv, L, D, layout, O,
                        out_dtype, tau, stream);
    return fwd_train_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, alpha, B, H, Hkv, L, D, layout, O,
                          out_dtype, tau, saved, saved_bytes, stream);
}

int entmax_attn_bwd_saved_ex(const void* Q, const void* K, const void* V, int in_dtype, const uint8_t* key_mask,
                             int causal, int window, float scale, float alpha, int B, int H, int Hkv, int L, int D,
                             int layout, const float* tau, const void* saved, size_t saved_bytes, const void* dO,
                             float* dQ, float* dK, float* dV, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    return bwd_saved_impl(Q, K, V, in_dtype, key_mask, causal, window, scale, alpha, B, H, Hkv, L, D, layout, tau,
                          saved, saved_bytes, dO, dQ, dK, dV, workspace, ws_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Allocation-free backward.  Same computation and kernels as entmax_attn_bwd; the per-row scratch
// (one float per query row) lives in a fixed device array owned by this library instead of a
// caller-provided workspace.
namespace entmax {

constexpr long long NOALLOC_MAX_ROWS = 1ll << 20;  // B*H*L limit: 4 MiB of scratch per device

// File-scope device scratch, present on every GPU that loads the library until the process exits.
static __device__ __align__(256) float g_noalloc_scratch[NOALLOC_MAX_ROWS];

namespace {
float* g_noalloc_ptr[MAX_DEVICES] = {};

// Device address of the scratch array on the current device.  Looked up once per device (host code
// may not use the array's symbol as an address); the lookup allocates nothing.
cudaError_t noalloc_scratch(float** out) {
    int dev = 0;
    cudaError_t e = current_device(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}
}  // namespace
}  // namespace entmax

extern "C" int entmax_attn_bwd_noalloc(const void* Q, const void* K, const void* V, int in_dtype,
                                       const uint8_t* key_mask, int causal, int window, float scale, int B, int H,
                                       int L, int D, const float* tau, const void* dO, float* dQ, float* dK,
                                       float* dV, cudaStream_t stream) {
    int rc = check_common(Q, K, V, in_dtype, causal, window, scale, B, H, L, D);
    if (rc) return rc;
    if (in_dtype != ENTMAX_BF16) return ENTMAX_ERR_UNSUPPORTED;  // fp32 inputs would need bf16 copies
    if ((long long)B * H * L > NOALLOC_MAX_ROWS) return ENTMAX_ERR_UNSUPPORTED;
    if (B == 0 || H == 0 || L == 0) return ENTMAX_OK;
    if (!tau || !dO || !dQ || !dK || !dV) return ENTMAX_ERR_ARG;
    if (!aligned(dO, 16) || !aligned(dQ, 8) || !aligned(dK, 8) || !aligned(dV, 8) || !aligned(tau, 4))
        return ENTMAX_ERR_ARG;
    int* status = nullptr;
    rc = record(status_ptr(&status));
    if (rc) return rc;
    float* scratch = nullptr;
    rc = record(noalloc_scratch(&scratch));
    if (rc) return rc;
    AttnArgs a{Q, K, V, key_mask, B, H, L, causal, window, scale, status, timeout_ns(), H, 0.5f, 0};
    BwdIO io{tau, dO, dQ, dK, dV, scratch};
    // the tensor-core kernels store gradient rows 16 bytes at a time
    const bool dense = dense_bwd(a) && aligned(dQ, 16) && aligned(dK, 16) && aligned(dV, 16);
    return record(dense ? launch_bwd_dense(a, io, stream) : launch_bwd(a, io, stream));
}
