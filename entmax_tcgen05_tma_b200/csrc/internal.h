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
    const void* K;           // [B,Hkv,L,64] bf16
    const void* V;
    const uint8_t* key_mask; // [B,L] or null
    int B, H, L;
    int causal, window;
    float scale;
    int* status;             // device status word
    unsigned long long timeout_ns;
    int Hkv;                 // key/value heads (H % Hkv == 0); query head h of batch b reads KV head
                             // b * Hkv + h / (H / Hkv) -- grouped-query attention when Hkv < H
    float am1;               // alpha - 1 in (0, 1]: p = max(0, am1 (S - tau))^(1 / am1); 0.5 is 1.5-entmax.
                             // 0: softmax, p = exp(S - tau) with tau = log sum_j exp(S_ij)
    int layout;              // 0: Q, K, V, O, dO, dQ, dK, dV are [B, heads, L, 64]; 1: [B, L, heads, 64]
};

// One head of a [B, nh, L, 64] (layout 0) or [B, L, nh, 64] (layout 1) tensor: its memory rows
// (units of 64 elements) and the TMA coordinates of a box of its rows.  Layout 0 maps are
// (d, L, B*nh) with boxes (64, rows, 1) at (0, row, b*nh + hh); layout 1 maps are (d, nh, B*L)
// with boxes (64, 1, rows) at (0, hh, b*L + row).  Either box lands in shared memory as `rows`
// consecutive 128-byte rows.  A layout-1 box that runs past row L of its batch reads the next
// batch's rows (or the zero fill after the last batch): the kernels mask rows and keys >= L.
struct HeadRef {
    int layout, b, hh, nh, L;
    __host__ __device__ __forceinline__ int c1(int row) const { return layout ? hh : row; }
    __host__ __device__ __forceinline__ int c2(int row) const { return layout ? b * L + row : b * nh + hh; }
    __host__ __device__ __forceinline__ size_t row(int i) const {
        return layout ? ((size_t)b * L + i) * nh + hh : ((size_t)b * nh + hh) * L + i;
    }
    __host__ __device__ __forceinline__ size_t step() const { return layout ? (size_t)nh : 1; }
};

// alpha = 1.5 runs the specialised kernels (closed-form tau finish, p = h^2); any other alpha in
// (1, 2] the generic ones; alpha = 1 (softmax) the tensor-core kernels of fwd_softmax.cu and
// bwd_dense.cu.
__host__ __device__ __forceinline__ bool softmax_alpha(const AttnArgs& a) { return a.am1 == 0.f; }
__host__ __device__ __forceinline__ bool generic_alpha(const AttnArgs& a) { return a.am1 != 0.5f; }

// Key/value head of query head bh = b * H + h.
__host__ __device__ __forceinline__ int kv_head_of(int bh, int H, int Hkv) { return (bh / H) * Hkv + (bh % H) / (H / Hkv); }

// Saved support of the forward pass, consumed by the support-list backward.  R = B*H*L rows.
constexpr int SAVE_CAP = 64;  // support entries kept per row
struct SavedSupport {
    int* row_cnt;            // [R] entries of row, or -1 when the row's support was not saved
    uint16_t* row_j;         // [R][SAVE_CAP] key index of each entry
    float* row_sp;           // [R][SAVE_CAP] b_ij = am1 (S_ij - tau_i) of each entry (sqrt(p_ij) at alpha 1.5)
    int* key_cnt;            // [B*Hkv*L] rows whose support holds key j of a KV head (zeroed before the forward)
    int* unsaved_cnt;        // [1] rows whose support was not saved (zeroed before the forward)
    int* unsaved_rows;       // [R] their row ids
};

struct FwdOut {
    void* O;                 // [B,H,L,64] bf16 or fp32
    int out_f32;
    float* tau;              // [B,H,L]
    SavedSupport save;       // row_cnt == nullptr: nothing saved
    float* otil;             // optional: [B*H*L][64] sum_j w_ij V_j, logical row order, w the Jacobian's
                             // weight (sqrt(p) at alpha 1.5; p for softmax, where otil is the fp32 O)
    float* rsum;             // optional with otil at alpha 1.5: [B*H*L] sum_j sqrt(p_ij) (softmax: 1, not written)
};

// Carves a caller buffer of entmax_attn_saved_bytes() into its arrays.
size_t saved_support_bytes(long long R);
SavedSupport carve_saved(void* base, long long R);



struct BwdIO {
    const float* tau;        // [B,H,L] from the forward
    const void* dO;          // [B,H,L,64] bf16
    float* dQ;               // [B,H,L,64] fp32
    float* dK;
    float* dV;
    float* u;                // workspace [B,H,L]: u_i = sum_j sqrt(p_ij) dA_ij / sum_j sqrt(p_ij)
    const float* otil;       // optional [B*H*L][64]: the forward's sum_j w_ij V_j (logical row order)
    const float* rsum;       // optional [B*H*L]: the forward's sum_j w_ij; with otil, u_i = dO_i . otil_i / rsum_i
                             // (softmax: rsum = 1, passed as null)
    const int* guard;        // optional (support-list backward): the device status word; when it is set
                             // (the forward that wrote the lists gave up), the kernels do nothing
};

// Workspace of the support-list backward.
struct SavedBwdWs {
    int* key_off;            // [R] head-local start of key j's bucket
    int* key_cur;            // [R] fill cursor
    uint32_t* bucket_i;      // [R * SAVE_CAP] query row of each (key, row) entry (head-local)
    float* bucket_sp;        // [R * SAVE_CAP] sqrt(p_ij)
    float* bucket_ds;        // [R * SAVE_CAP] dS_ij
};
size_t saved_bwd_ws_bytes(long long R);
SavedBwdWs carve_saved_bwd_ws(void* base, long long R);
cudaError_t launch_bwd_saved(const AttnArgs& a, const BwdIO& io, const SavedSupport& sv, const SavedBwdWs& ws,
                             cudaStream_t stream);

// Tensor map over a [B*H, L, 64] bf16 tensor, boxes of box_rows rows, 128-byte swizzle.
cudaError_t make_tile_map(CUtensorMap* map, const void* base, int layout, int B, int nh, int L, int box_rows);

// Gather forward (fwd.cu).  extract: support extraction for a backward given tau alone -- o.tau is
// read (the caller's tau), o.save receives the support lists, o.O, o.otil and o.rsum are unused.
cudaError_t launch_fwd(const AttnArgs& a, const FwdOut& o, cudaStream_t stream, bool extract = false);
// Softmax forward (fwd_softmax.cu): writes O and tau = log sum_j exp(S_ij), and O in fp32 into o.otil
// when given; o.save and o.rsum unused.
cudaError_t launch_fwd_softmax(const AttnArgs& a, const FwdOut& o, cudaStream_t stream);
cudaError_t launch_bwd(const AttnArgs& a, const BwdIO& io, cudaStream_t stream);

// The tensor-core backward (bwd_dense.cu) serves 1.5-entmax rows whose allowed keys span few key
// blocks -- sequences of at most 512 keys, or causal windows of at most 128 keys: there a 128 x 64
// tile of (query, key) pairs costs less as tcgen05 products than as gathers over its support -- and
// softmax (dense supports) at every length.  Every backward entry point dispatches on this, and the
// training forward saves no support lists when it holds (the tensor-core backward does not read them).
__host__ __device__ __forceinline__ bool dense_bwd(const AttnArgs& a) {
    return softmax_alpha(a) || (a.am1 == 0.5f && (a.L <= 512 || (a.causal && a.window > 0 && a.window <= 128)));
}
// The tensor-core forward of 1.5-entmax (fwd_dense.cu) serves the same configurations; the gather
// forward (fwd.cu) keeps the auxiliary rows and the support lists, which it alone writes.
__host__ __device__ __forceinline__ bool dense_fwd(const AttnArgs& a) { return a.am1 == 0.5f && dense_bwd(a); }
cudaError_t launch_fwd_dense(const AttnArgs& a, const FwdOut& o, cudaStream_t stream);
// dq kernel (writes io.u, one float per query row, and dQ), then dkdv kernel (dK, dV).
cudaError_t launch_bwd_dense(const AttnArgs& a, const BwdIO& io, cudaStream_t stream);
cudaError_t launch_f32_to_bf16(const float* src, void* dst, size_t n, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit once per (kernel slot, device).
cudaError_t ensure_smem_attr(const void* func, int bytes, int slot);

size_t fwd_smem_bytes();
size_t bwd_rows_smem_bytes();
size_t bwd_keys_smem_bytes();
size_t dense_dq_smem_bytes();
size_t dense_dkdv_smem_bytes();
size_t softmax_fwd_smem_bytes();
size_t dense_fwd_smem_bytes();

}  // namespace entmax
