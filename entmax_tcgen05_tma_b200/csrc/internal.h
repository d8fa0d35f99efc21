// internal.h -- argument blocks and launchers shared by the C ABI (abi.cu) and the kernel
// translation units.  Not part of the public interface.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace entmax {

struct AttnArgs {
    const void* Q;           // [B,H,L,64] bf16
    const void* K;
    const void* V;
    const uint8_t* key_mask; // [B,L] or null
    int B, H, L;
    int causal, window;
    float scale;
    int* status;             // device status word
    unsigned long long timeout_ns;
};

struct FwdOut {
    void* O;                 // [B,H,L,64] bf16 or fp32
    int out_f32;
    float* tau;              // [B,H,L]
};

struct BwdIO {
    const float* tau;        // [B,H,L] from the forward
    const void* dO;          // [B,H,L,64] bf16
    float* dQ;               // [B,H,L,64] fp32
    float* dK;
    float* dV;
    float* u;                // workspace [B,H,L]: u_i = sum_j sqrt(p_ij) dA_ij / sum_j sqrt(p_ij)
};

// Tensor map over a [B*H, L, 64] bf16 tensor, 128-row boxes, 128-byte swizzle.
cudaError_t make_tile_map(CUtensorMap* map, const void* base, int BH, int L);

cudaError_t launch_fwd(const AttnArgs& a, const FwdOut& o, cudaStream_t stream);
cudaError_t launch_bwd(const AttnArgs& a, const BwdIO& io, cudaStream_t stream);
cudaError_t launch_f32_to_bf16(const float* src, void* dst, size_t n, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit once per (kernel slot, device).
cudaError_t ensure_smem_attr(const void* func, int bytes, int slot);

size_t fwd_smem_bytes();
size_t bwd_rows_smem_bytes();
size_t bwd_keys_smem_bytes();

}  // namespace entmax
