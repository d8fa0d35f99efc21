/*
 * entmax_attn.h -- C ABI of the B200 (sm_100a) 1.5-entmax attention library.
 *
 * Operation (page "svd-sst2-roberta-adasplash", sections 2.2-2.4 and 3; model cards
 * "roberta-base-adasplash" and "distilbert-sst2-adasplash", "Mathematical Formulation"):
 * multi-head attention whose softmax is replaced by Tsallis 1.5-entmax.  For each batch b,
 * head h and query row i:
 *
 *   S_ij   = scale * <Q_i, K_j>                      for the allowed keys j,
 *   tau_i  : the unique root of sum_j max(0, (S_ij - tau_i)/2)^2 = 1   (Theorem 1),
 *            found by bisection on [max_j S_ij - 2, max_j S_ij - 2/sqrt(n_i)] (Theorem 2 and the
 *            model cards' bracket; n_i = number of allowed keys), at most 25 halvings,
 *   A_ij   = max(0, (S_ij - tau_i)/2)^2  (exact zeros off the support),
 *   O_i    = sum_j A_ij V_j.
 *
 * Allowed keys (section 3, "Structural Masking Stage"): key j is allowed for query i iff
 *   key_mask[b, j] != 0 (key padding; NULL means every key is valid),
 *   and, if causal, j <= i,
 *   and, if window > 0, j >= i - window + 1 (a causal sliding window of `window` keys
 *   including the query itself; window requires causal).
 * Masked keys are excluded, not filled with a large negative value.  A row with no allowed
 * key gets O_i = 0, tau_i = +inf and zero gradients.
 *
 * Layout: Q, K, V, dO, O, dQ, dK, dV are contiguous row-major [B, H, L, D] tensors (the _ex entry
 * points also take [B, L, H, D]: entmax_layout); tau is [B, H, L]; key_mask is [B, L] bytes.
 * D must be 64.  All pointers are DEVICE pointers owned by the caller; the library keeps no
 * reference after a call returns.  Every call is asynchronous on `stream` (0 = the legacy
 * default stream) and works on the calling thread's current device.
 *
 * Host threads: any entry point may be called from several threads at once.  The wait bound
 * (entmax_attn_set_wait_timeout_ns), the last CUDA error and each device's status word are
 * shared by the whole process.
 *
 * Contexts: the first call on a device looks up, once, the device addresses of the library's own
 * device variables (the status word; the scratch array of entmax_attn_bwd_noalloc) in that
 * device's primary context and keeps them for the life of the process.  Destroying or resetting
 * the primary context (cudaDeviceReset, cuDevicePrimaryCtxReset) invalidates them: do not call
 * the library on that device again in the same process after such a reset.
 *
 * Errors: arguments are checked on the host before any launch; a bad argument returns a
 * negative status and launches nothing.  Problems found on the device (a bounded wait that
 * timed out) are recorded in a device status word; entmax_attn_device_status() reads it.
 */
#ifndef ENTMAX_ATTN_H
#define ENTMAX_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define ENTMAX_API __attribute__((visibility("default")))
#else
#define ENTMAX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ENTMAX_OK = 0,
    ENTMAX_ERR_ARG = -1,          /* null pointer, bad size, bad dtype, misaligned pointer, scale <= 0 */
    ENTMAX_ERR_UNSUPPORTED = -2,  /* D != 64, L > 16384, B*H > 65535, window without causal */
    ENTMAX_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed (see entmax_attn_last_cuda_error) */
    ENTMAX_ERR_TIMEOUT = -4,      /* a device-side bounded wait expired */
    ENTMAX_ERR_WORKSPACE = -5     /* workspace missing or smaller than the entry point's minimum */
} entmax_status;

typedef enum {
    ENTMAX_BF16 = 0,
    ENTMAX_F32 = 1
} entmax_dtype;

/* Memory layout of Q, K, V, O, dO, dQ, dK, dV for the _ex entry points (every other entry point
 * takes ENTMAX_LAYOUT_BHLD).  BLHD is the [B, L, heads, 64] tensor that the attention layer of page
 * "svd-sst2-roberta-adasplash" (section 3, the reshape-and-transpose step) views as [B, heads, L, 64]:
 * passing it directly avoids a transposing copy.  tau is [B, H, L] in both. */
typedef enum {
    ENTMAX_LAYOUT_BHLD = 0, /* [B, heads, L, 64], rows of one head contiguous */
    ENTMAX_LAYOUT_BLHD = 1  /* [B, L, heads, 64], heads of one position contiguous */
} entmax_layout;

/*
 * Forward pass.
 *   Q, K, V   [B,H,L,D] in `in_dtype`.  ENTMAX_F32 inputs are rounded to bf16 (round to
 *             nearest even) on the device before use; the arithmetic is bf16 x bf16 products
 *             with fp32 accumulation either way.  16-byte aligned.
 *   key_mask  [B,L] uint8, 1 = valid key; NULL = all valid.
 *   causal    0/1.   window: keys per row including the query (0 = off; > 0 needs causal).
 *   scale     > 0, multiplies Q.K (1/sqrt(D) on the pages' encoders).
 *   O         [B,H,L,D] in `out_dtype` (bf16 or fp32), 16-byte aligned (16-byte stores).
 *   tau       [B,H,L] fp32, the threshold in score units: A_ij = max(0,(S_ij - tau_i)/2)^2.
 *             Needed by the backward pass.
 * Returns ENTMAX_OK once the work is queued on `stream`.  B, H or L equal to 0 is a no-op.
 */
ENTMAX_API int entmax_attn_fwd(const void* Q, const void* K, const void* V, int in_dtype,
                    const uint8_t* key_mask, int causal, int window, float scale,
                    int B, int H, int L, int D,
                    void* O, int out_dtype, float* tau, cudaStream_t stream);

/* Bytes of device workspace for entmax_attn_bwd's fastest path; 0 when B, H or L is 0.
 * The minimum entmax_attn_bwd accepts is one float per query row (the row scalar u_i passed from
 * the dQ kernel to the dK/dV kernel), rounded up to 256 bytes, and that is what this returns for
 * L <= 512 (every such row takes the tensor-core backward).  For L > 512 it returns room for
 * support lists and the support-list backward's buckets (about 1.1 KB per query row): given that
 * much, 256-byte aligned, rows off the tensor-core path rebuild their supports from tau in one
 * score pass on the tensor cores (support extraction) and take the support-list backward, instead
 * of recomputing each row's support on CUDA cores in every kernel of the backward. */
ENTMAX_API size_t entmax_attn_bwd_workspace_size(int B, int H, int L, int D);

/*
 * Backward pass for the loss gradient dO = dL/dO, by the closed-form Jacobian of section 2.4
 * (page "svd-sst2-roberta-adasplash"; model card "roberta-base-adasplash", section 2):
 *   dA_ij = <dO_i, V_j>,  sp_ij = sqrt(A_ij),  u_i = sum_j sp_ij dA_ij / sum_j sp_ij,
 *   dS_ij = sp_ij (dA_ij - u_i),
 *   dQ_i = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i,  dV_j = sum_i A_ij dO_i.
 *   Q, K, V, dO  [B,H,L,D] in `in_dtype` (fp32 inputs are rounded to bf16 first).
 *   tau          [B,H,L] from entmax_attn_fwd with the same Q, K, masks and scale.
 *   dQ, dK, dV   [B,H,L,D] fp32, fully overwritten.  8-byte aligned.
 *   workspace    device buffer of at least one float per query row (rounded up to 256 bytes),
 *                16-byte aligned, owned by the caller; its contents need no initialisation.  With
 *                entmax_attn_bwd_workspace_size(B,H,L,D) bytes, 256-byte aligned, long rows take the
 *                faster path described there: each row's support {j : S_ij > tau_i} is listed
 *                into the workspace from the caller's tau.  On that path a device error recorded
 *                before or during the call (see entmax_attn_device_status) leaves dQ, dK, dV
 *                unwritten: the support lists of an extraction that gave up are not read.
 * fp32 inputs additionally use stream-ordered temporaries (cudaMallocAsync) for their bf16
 * copies; bf16 inputs allocate nothing.
 */
ENTMAX_API int entmax_attn_bwd(const void* Q, const void* K, const void* V, int in_dtype,
                    const uint8_t* key_mask, int causal, int window, float scale,
                    int B, int H, int L, int D,
                    const float* tau, const void* dO,
                    float* dQ, float* dK, float* dV,
                    void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Auxiliary rows of the forward pass, for the backward's row scalar (page "svd-sst2-roberta-adasplash",
 * section 2.4: u_i = sum_j sqrt(A_ij) dA_ij / sum_j sqrt(A_ij) with dA_ij = dO_i . V_j; since dA is
 * linear in V, u_i = dO_i . Otil_i / r_i).  entmax_attn_fwd_aux computes exactly what entmax_attn_fwd
 * computes and also, for every query row,
 *   Otil   [B,H,L,D] fp32, Otil_i = sum_j sqrt(A_ij) V_j, rows in [B,H,L] order, 16-byte aligned,
 *   rsum   [B,H,L] fp32,   r_i = sum_j sqrt(A_ij)  (0 for a row with no allowed key),
 * both caller-owned device buffers, fully written.  entmax_attn_bwd_aux computes exactly what
 * entmax_attn_bwd computes, taking u_i from these rows instead of deriving it: on the tensor-core
 * configurations (L <= 512, or a causal window of at most 128 keys) that removes a pass over the
 * scores.  Elsewhere the rows are checked but not needed (the support gathers form u_i on the way).
 *   Otil, rsum   from entmax_attn_fwd_aux with the same Q, K, V, masks and scale.
 *   workspace    as for entmax_attn_bwd (entmax_attn_bwd_workspace_size bytes).
 * Other arguments and errors: as entmax_attn_fwd / entmax_attn_bwd; a null or misaligned Otil or rsum
 * returns ENTMAX_ERR_ARG.
 */
ENTMAX_API int entmax_attn_fwd_aux(const void* Q, const void* K, const void* V, int in_dtype,
                                   const uint8_t* key_mask, int causal, int window, float scale,
                                   int B, int H, int L, int D,
                                   void* O, int out_dtype, float* tau, float* Otil, float* rsum,
                                   cudaStream_t stream);
ENTMAX_API int entmax_attn_bwd_aux(const void* Q, const void* K, const void* V, int in_dtype,
                                   const uint8_t* key_mask, int causal, int window, float scale,
                                   int B, int H, int L, int D,
                                   const float* tau, const float* Otil, const float* rsum, const void* dO,
                                   float* dQ, float* dK, float* dV,
                                   void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Training path.  entmax_attn_fwd_train computes exactly what entmax_attn_fwd computes and also saves
 * each row's support {(j, sqrt(A_ij)) : A_ij > 0} (up to 64 entries per row; rows with more, and rows
 * the forward had to redo exactly on CUDA cores, are marked and recomputed by the backward) plus, per
 * key, how many rows hold it.  entmax_attn_bwd_saved then evaluates the same closed-form gradients as
 * entmax_attn_bwd from those lists without forming Q K^T again: its cost scales with the number of
 * support entries.  (Page "svd-sst2-roberta-adasplash", section 2.4: the gradient is zero off the
 * support, and the support is what the forward's tau already fixed.)
 *   saved      device buffer of entmax_attn_saved_bytes(B,H,L,D) bytes, 256-byte aligned, written by
 *              entmax_attn_fwd_train and read by entmax_attn_bwd_saved for the same Q, K, masks and
 *              scale; owned by the caller.
 *   workspace  device buffer of entmax_attn_bwd_saved_workspace_size(B,H,L,D) bytes, 256-byte aligned.
 *   O (training forward) and dQ, dK, dV (this backward): 16-byte aligned (16-byte stores); the
 *   other arguments as in entmax_attn_fwd / entmax_attn_bwd.
 * On the tensor-core configurations (L <= 512, or a causal window of at most 128 keys, at alpha 1.5)
 * the backward recomputes the scores on tcgen05 and reads nothing from `saved` but its size; every
 * output is then the same bit for bit from run to run.  Elsewhere dK and dV are summed in an order
 * that depends on scheduling (last-bit differences between runs); dQ, O and tau are deterministic.
 * A training forward that reported a device error (ENTMAX_ERR_TIMEOUT) left `saved` invalid: do not
 * pass it to the backward.  While such an error is recorded and not yet read, the support-list
 * backward does nothing (it does not read lists that may be half-written) and dQ, dK, dV are left
 * unwritten.
 */
ENTMAX_API size_t entmax_attn_saved_bytes(int B, int H, int L, int D);
ENTMAX_API size_t entmax_attn_bwd_saved_workspace_size(int B, int H, int L, int D);
ENTMAX_API int entmax_attn_fwd_train(const void* Q, const void* K, const void* V, int in_dtype,
                                     const uint8_t* key_mask, int causal, int window, float scale,
                                     int B, int H, int L, int D,
                                     void* O, int out_dtype, float* tau,
                                     void* saved, size_t saved_bytes, cudaStream_t stream);
ENTMAX_API int entmax_attn_bwd_saved(const void* Q, const void* K, const void* V, int in_dtype,
                                     const uint8_t* key_mask, int causal, int window, float scale,
                                     int B, int H, int L, int D,
                                     const float* tau, const void* saved, size_t saved_bytes,
                                     const void* dO, float* dQ, float* dK, float* dV,
                                     void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Grouped-query attention.  The page "svd-sst2-roberta-adasplash" (section 3, the step-by-step
 * tensor trace, and the attention layer's forward in section 4) projects keys and values to H_kv
 * heads and repeats each of them H/H_kv times before the scores, so query head h of batch b attends
 * with key/value head b*H_kv + h/(H/H_kv).  These three entry points compute exactly what
 * entmax_attn_fwd, entmax_attn_fwd_train and entmax_attn_bwd_saved compute on the repeated K and V,
 * without materialising the repeat:
 *   K, V       [B, H_kv, L, 64] bf16 (in_dtype must be ENTMAX_BF16 when H_kv < H;
 *              ENTMAX_F32 returns ENTMAX_ERR_UNSUPPORTED there).
 *   Q, O, tau, dO, dQ, saved: as in the non-grouped calls, over B*H query rows.
 *   dK, dV     [B, H_kv, L, 64] fp32: the gradient of each key/value head, i.e. the sum over the
 *              H/H_kv query heads that share it.
 *   H_kv       1 <= H_kv <= H and H % H_kv == 0, else ENTMAX_ERR_ARG (H_kv = H is the plain
 *              multi-head case; H = 0 requires H_kv = 0).
 *   saved / workspace sizes: entmax_attn_saved_bytes(B,H,L,D) and
 *              entmax_attn_bwd_saved_workspace_size(B,H,L,D) with the QUERY head count H.
 */
ENTMAX_API int entmax_attn_fwd_gqa(const void* Q, const void* K, const void* V, int in_dtype,
                                   const uint8_t* key_mask, int causal, int window, float scale,
                                   int B, int H, int H_kv, int L, int D,
                                   void* O, int out_dtype, float* tau, cudaStream_t stream);
ENTMAX_API int entmax_attn_fwd_train_gqa(const void* Q, const void* K, const void* V, int in_dtype,
                                         const uint8_t* key_mask, int causal, int window, float scale,
                                         int B, int H, int H_kv, int L, int D,
                                         void* O, int out_dtype, float* tau,
                                         void* saved, size_t saved_bytes, cudaStream_t stream);
ENTMAX_API int entmax_attn_bwd_saved_gqa(const void* Q, const void* K, const void* V, int in_dtype,
                                         const uint8_t* key_mask, int causal, int window, float scale,
                                         int B, int H, int H_kv, int L, int D,
                                         const float* tau, const void* saved, size_t saved_bytes,
                                         const void* dO, float* dQ, float* dK, float* dV,
                                         void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * alpha-entmax attention for any alpha in [1, 2] (page "svd-sst2-roberta-adasplash", section 4: the
 * attention layer's entmax_bisect routine solves sum_j max(0, (alpha-1) s_j - tau')^(1/(alpha-1)) = 1
 * by bisection for alpha in (1, 2] and returns softmax for |alpha - 1| < 1e-4; alpha = 1.5 is the
 * 1.5-entmax of every other entry point, alpha = 2 is sparsemax).  For alpha in (1, 2], with
 * a = alpha - 1 and tau in score units (tau' = a tau):
 *   p_ij = max(0, a (S_ij - tau_i))^(1/a),  sum_j p_ij = 1,  O_i = sum_j p_ij V_j,
 * and the backward uses the Jacobian w_i (delta_ij - w_j / sum_k w_k), w = p^(2 - alpha).
 *   alpha      in [1, 2]; any other value (or NaN) returns ENTMAX_ERR_ARG.  alpha = 1.5 runs exactly
 *              the kernels of the entry points above; other values in (1, 2] run variants whose tau
 *              solve is Newton's method from the bracket's lower end (bisection as the backstop)
 *              instead of bisection with a closed-form finish.  Supports grow as alpha approaches 1:
 *              rows with more candidates than the kernels list are recomputed on CUDA cores, so
 *              small alpha - 1 is correct but slow.
 *              Softmax: like the pages' routine, |alpha - 1| < 1e-4 computes softmax attention,
 *              p_ij = exp(S_ij - tau_i) with tau_i = log sum_j exp(S_ij) over the allowed keys (the
 *              alpha -> 1 limit; every allowed key is in the support).  Its forward and backward run
 *              every product on the tensor cores (two passes over the key blocks in the forward:
 *              the row max, then O and tau); the training forward saves no supports but writes O in
 *              fp32 into saved ([B*H*L][64], logical row order), from which the backward forms
 *              u_i = sum_j p_ij dA_ij as the row dot dO_i . O_i; the backward recomputes the scores.
 *              Its gradients are the same bit for bit from run to run.
 *   H_kv       key/value heads as in the _gqa calls (H_kv = H: plain multi-head attention).
 *   saved      entmax_attn_fwd_ex: NULL with saved_bytes = 0 computes the forward only
 *              (entmax_attn_fwd / _gqa); otherwise the training forward (entmax_attn_fwd_train /
 *              _gqa).  entmax_attn_bwd_saved_ex reads supports written by entmax_attn_fwd_ex with
 *              the same alpha, Q, K, masks and scale.  Each saved entry holds b_ij = a (S_ij - tau_i)
 *              (sqrt(p_ij) at alpha = 1.5).
 *   tau        fp32 [B, H, L], score units for every alpha (+inf for a row with no allowed key).
 *   layout     ENTMAX_LAYOUT_BHLD or ENTMAX_LAYOUT_BLHD (else ENTMAX_ERR_ARG), for all of Q, K, V,
 *              O, dO, dQ, dK, dV alike (K, V, dK, dV with H_kv heads).  The saved supports do not
 *              depend on it.
 * Other arguments, layouts and errors: as entmax_attn_fwd / _fwd_train / _bwd_saved and their _gqa
 * forms.
 */
ENTMAX_API int entmax_attn_fwd_ex(const void* Q, const void* K, const void* V, int in_dtype,
                                  const uint8_t* key_mask, int causal, int window, float scale, float alpha,
                                  int B, int H, int H_kv, int L, int D, int layout,
                                  void* O, int out_dtype, float* tau,
                                  void* saved, size_t saved_bytes, cudaStream_t stream);
ENTMAX_API int entmax_attn_bwd_saved_ex(const void* Q, const void* K, const void* V, int in_dtype,
                                        const uint8_t* key_mask, int causal, int window, float scale,
                                        float alpha, int B, int H, int H_kv, int L, int D, int layout,
                                        const float* tau, const void* saved, size_t saved_bytes,
                                        const void* dO, float* dQ, float* dK, float* dV,
                                        void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Allocation-free variant of entmax_attn_bwd (no counterpart in the AdaSplash pages; it exists for
 * this library's users).  Some callers cannot allocate device memory at the point where they run
 * the backward pass: engines that plan all memory ahead of time and forbid allocation inside their
 * execution callbacks, code running while a stream is being captured, or latency-critical loops
 * where an allocator call would synchronise the device.  This entry point takes the same arguments
 * as entmax_attn_bwd minus the workspace: its per-row scratch (one float per query row) is a fixed
 * array inside the library, 4 MiB on every GPU that loads the library, held until the process exits.
 *   - B*H*L must not exceed 1,048,576 (1 << 20) rows: larger problems return ENTMAX_ERR_UNSUPPORTED
 *     (use entmax_attn_bwd with a caller workspace instead).
 *   - Inputs must be bf16 (ENTMAX_F32 returns ENTMAX_ERR_UNSUPPORTED: converting them would need
 *     temporary memory).
 *   - It calls no allocation routine.  The first call on a device looks up the array's device
 *     address (cudaGetSymbolAddress) for that device; make that first call before any stream
 *     capture.
 *   - All calls share the one array, which keeps the previous call's contents (every value a call
 *     reads it writes first).  Calls whose execution overlaps on the GPU, e.g. on two streams,
 *     race on it: serialise them.
 */
ENTMAX_API int entmax_attn_bwd_noalloc(const void* Q, const void* K, const void* V, int in_dtype,
                                       const uint8_t* key_mask, int causal, int window, float scale,
                                       int B, int H, int L, int D,
                                       const float* tau, const void* dO,
                                       float* dQ, float* dK, float* dV, cudaStream_t stream);

/* Static description of a status code. */
ENTMAX_API const char* entmax_attn_strerror(int status);

/* Synchronises `stream`, then returns and clears the device status word of the current device:
 * ENTMAX_OK, or ENTMAX_ERR_TIMEOUT if a kernel's bounded wait expired since the last read. */
ENTMAX_API int entmax_attn_device_status(cudaStream_t stream);

/* cudaError_t value of the most recent failed CUDA call inside the library (0 if none). */
ENTMAX_API int entmax_attn_last_cuda_error(void);

/* Bound on each device-side wait, in nanoseconds; 0 restores the default (2 s).  Affects
 * launches made after the call.  Intended for tests of the timeout path. */
ENTMAX_API void entmax_attn_set_wait_timeout_ns(unsigned long long ns);

/* Library version, major*10000 + minor*100 + patch. */
ENTMAX_API int entmax_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ENTMAX_ATTN_H */
