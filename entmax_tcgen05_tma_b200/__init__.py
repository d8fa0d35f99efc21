"""B200-native 1.5-entmax ("AdaSplash") attention.

Multi-head attention whose softmax is replaced by Tsallis 1.5-entmax: per query row,
tau solves sum_j max(0, (S_ij - tau)/2)^2 = 1 by bisection, A = max(0, (S - tau)/2)^2 has exact
zeros, O = A V; the backward pass uses the closed-form Jacobian.  The _ex entry points take any
alpha in [1, 2] (alpha within 1e-4 of 1: softmax).  The work runs in hand-written
sm_100a kernels (tcgen05 tensor cores, TMEM, TMA) behind the C ABI in include/entmax_attn.h;
this package is its thin Python binding.
"""
from ._binding import (  # noqa: F401
    ENTMAX_BF16,
    ENTMAX_ERR_ARG,
    ENTMAX_ERR_CUDA,
    ENTMAX_ERR_TIMEOUT,
    ENTMAX_ERR_UNSUPPORTED,
    ENTMAX_ERR_WORKSPACE,
    ENTMAX_F32,
    ENTMAX_LAYOUT_BHLD,
    ENTMAX_LAYOUT_BLHD,
    ENTMAX_OK,
    EXPORTED,
    LIB_PATH,
    EntmaxAttention,
    EntmaxError,
    bwd_min_workspace_size,
    entmax_attn_bwd,
    entmax_attn_bwd_aux,
    entmax_attn_bwd_noalloc,
    entmax_attn_bwd_saved,
    entmax_attn_bwd_saved_ex,
    entmax_attn_bwd_saved_gqa,
    entmax_attn_bwd_saved_workspace_size,
    entmax_attn_bwd_workspace_size,
    entmax_attn_device_status,
    entmax_attn_fwd,
    entmax_attn_fwd_aux,
    entmax_attn_fwd_ex,
    entmax_attn_fwd_gqa,
    entmax_attn_fwd_train,
    entmax_attn_fwd_train_gqa,
    entmax_attn_last_cuda_error,
    entmax_attn_saved_bytes,
    entmax_attn_set_wait_timeout_ns,
    lib,
    strerror,
    version,
)
