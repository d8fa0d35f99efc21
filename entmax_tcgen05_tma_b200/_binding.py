"""ctypes binding of libentmax_attn.so (include/entmax_attn.h).

Argument marshalling only: checks tensor placement/dtype/contiguity, allocates outputs with
torch when the caller gives none, passes raw device pointers and the current CUDA stream, and
turns status codes into exceptions.  All arithmetic runs in the library's CUDA kernels; there is
no CPU path.  A missing or unloadable library raises ImportError at the first call.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libentmax_attn.so"

ENTMAX_OK = 0
ENTMAX_ERR_ARG = -1
ENTMAX_ERR_UNSUPPORTED = -2
ENTMAX_ERR_CUDA = -3
ENTMAX_ERR_TIMEOUT = -4
ENTMAX_ERR_WORKSPACE = -5
ENTMAX_BF16 = 0
ENTMAX_F32 = 1
ENTMAX_LAYOUT_BHLD = 0
ENTMAX_LAYOUT_BLHD = 1

EXPORTED = (
    "entmax_attn_fwd",
    "entmax_attn_bwd_workspace_size",
    "entmax_attn_bwd",
    "entmax_attn_bwd_noalloc",
    "entmax_attn_fwd_aux",
    "entmax_attn_bwd_aux",
    "entmax_attn_saved_bytes",
    "entmax_attn_bwd_saved_workspace_size",
    "entmax_attn_fwd_train",
    "entmax_attn_bwd_saved",
    "entmax_attn_fwd_gqa",
    "entmax_attn_fwd_train_gqa",
    "entmax_attn_bwd_saved_gqa",
    "entmax_attn_fwd_ex",
    "entmax_attn_bwd_saved_ex",
    "entmax_attn_strerror",
    "entmax_attn_device_status",
    "entmax_attn_last_cuda_error",
    "entmax_attn_set_wait_timeout_ns",
    "entmax_attn_version",
)


class EntmaxError(RuntimeError):
    """A library call returned a negative status (``status``); the message names the call, the
    status and, for ENTMAX_ERR_CUDA, the CUDA error code."""

    def __init__(self, status: int, what: str):
        self.status = status
        msg = "%s failed: %s (%d)" % (what, strerror(status), status)
        if status == ENTMAX_ERR_CUDA:
            msg += ", cudaError %d" % lib.entmax_attn_last_cuda_error()
        super().__init__(msg)


def _load_library() -> ctypes.CDLL:
    if not LIB_PATH.exists():
        raise ImportError(
            "libentmax_attn.so is not built (%s); run `python -m entmax_tcgen05_tma_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(str(LIB_PATH))
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.entmax_attn_fwd.restype = i
    lib.entmax_attn_fwd.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, vp, i, vp, vp]
    lib.entmax_attn_bwd_workspace_size.restype = sz
    lib.entmax_attn_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.entmax_attn_bwd.restype = i
    lib.entmax_attn_bwd.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.entmax_attn_bwd_noalloc.restype = i
    lib.entmax_attn_bwd_noalloc.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, vp, vp, vp, vp, vp, vp]
    lib.entmax_attn_fwd_aux.restype = i
    lib.entmax_attn_fwd_aux.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, vp, i, vp, vp, vp, vp]
    lib.entmax_attn_bwd_aux.restype = i
    lib.entmax_attn_bwd_aux.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                        vp]
    lib.entmax_attn_saved_bytes.restype = sz
    lib.entmax_attn_saved_bytes.argtypes = [i, i, i, i]
    lib.entmax_attn_bwd_saved_workspace_size.restype = sz
    lib.entmax_attn_bwd_saved_workspace_size.argtypes = [i, i, i, i]
    lib.entmax_attn_fwd_train.restype = i
    lib.entmax_attn_fwd_train.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, vp, i, vp, vp, sz, vp]
    lib.entmax_attn_bwd_saved.restype = i
    lib.entmax_attn_bwd_saved.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, vp, vp, sz, vp, vp, vp, vp, vp, sz,
                                          vp]
    lib.entmax_attn_fwd_gqa.restype = i
    lib.entmax_attn_fwd_gqa.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, i, vp, i, vp, vp]
    lib.entmax_attn_fwd_train_gqa.restype = i
    lib.entmax_attn_fwd_train_gqa.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, i, vp, i, vp, vp, sz, vp]
    lib.entmax_attn_bwd_saved_gqa.restype = i
    lib.entmax_attn_bwd_saved_gqa.argtypes = [vp, vp, vp, i, vp, i, i, f, i, i, i, i, i, vp, vp, sz, vp, vp, vp, vp,
                                              vp, sz, vp]
    lib.entmax_attn_fwd_ex.restype = i
    lib.entmax_attn_fwd_ex.argtypes = [vp, vp, vp, i, vp, i, i, f, f, i, i, i, i, i, i, vp, i, vp, vp, sz, vp]
    lib.entmax_attn_bwd_saved_ex.restype = i
    lib.entmax_attn_bwd_saved_ex.argtypes = [vp, vp, vp, i, vp, i, i, f, f, i, i, i, i, i, i, vp, vp, sz, vp, vp,
                                             vp, vp, vp, sz, vp]
    lib.entmax_attn_strerror.restype = ctypes.c_char_p
    lib.entmax_attn_strerror.argtypes = [i]
    lib.entmax_attn_device_status.restype = i
    lib.entmax_attn_device_status.argtypes = [vp]
    lib.entmax_attn_last_cuda_error.restype = i
    lib.entmax_attn_last_cuda_error.argtypes = []
    lib.entmax_attn_set_wait_timeout_ns.restype = None
    lib.entmax_attn_set_wait_timeout_ns.argtypes = [ctypes.c_ulonglong]
    lib.entmax_attn_version.restype = i
    lib.entmax_attn_version.argtypes = []
    return lib


class _LazyLibrary:
    """Loads libentmax_attn.so on first use, so the package (and its build module) imports without
    the library; any call into the library raises ImportError if it has not been built."""

    _cdll = None

    def __getattr__(self, name):
        if _LazyLibrary._cdll is None:
            _LazyLibrary._cdll = _load_library()
        return getattr(_LazyLibrary._cdll, name)


lib = _LazyLibrary()


def strerror(status: int) -> str:
    """Static description of a status code."""
    return lib.entmax_attn_strerror(int(status)).decode()


def version() -> int:
    """Library version, major * 10000 + minor * 100 + patch."""
    return lib.entmax_attn_version()


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ENTMAX_BF16
    if t.dtype == torch.float32:
        return ENTMAX_F32
    raise TypeError("inputs must be bfloat16 or float32, got %s" % t.dtype)


def _check_input(name: str, t: torch.Tensor, shape, dtype=None, layout: int = ENTMAX_LAYOUT_BHLD) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if layout == ENTMAX_LAYOUT_BHLD and not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if layout == ENTMAX_LAYOUT_BLHD and not t.transpose(1, 2).is_contiguous():
        raise ValueError("%s must be a [B,H,L,D] view of a contiguous [B,L,H,D] tensor, like Q" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))


def _mask_ptr(key_mask, B: int, L: int, device) -> int | None:
    if key_mask is None:
        return None
    _check_input("key_mask", key_mask, (B, L))
    if key_mask.dtype not in (torch.uint8, torch.bool):
        raise TypeError("key_mask must be uint8 or bool")
    if key_mask.device != device:
        raise ValueError("key_mask must be on the same device as Q")
    return key_mask.data_ptr()


def _layout_of(Q) -> int:
    """ENTMAX_LAYOUT_BHLD for a contiguous [B,H,L,D] tensor; ENTMAX_LAYOUT_BLHD for the [B,H,L,D] view
    (x.transpose(1, 2)) of a contiguous [B,L,H,D] tensor x."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be a 4-D [B,H,L,D] tensor")
    if Q.is_contiguous():
        return ENTMAX_LAYOUT_BHLD
    if Q.transpose(1, 2).is_contiguous():
        return ENTMAX_LAYOUT_BLHD
    raise ValueError("Q must be contiguous [B,H,L,D], or the transpose(1, 2) view of a contiguous [B,L,H,D]")


def _empty(shape, dtype, device, layout: int) -> torch.Tensor:
    """Output tensor of shape [B,H,L,D] in the given memory layout."""
    if layout == ENTMAX_LAYOUT_BLHD:
        B, H, L, D = shape
        return torch.empty((B, L, H, D), dtype=dtype, device=device).transpose(1, 2)
    return torch.empty(shape, dtype=dtype, device=device)


def _kv_heads(Q, K, grouped: bool) -> int:
    """Key/value head count: K.shape[1] for the grouped calls, which must divide H; H otherwise."""
    H = Q.shape[1]
    if not grouped:
        return H
    if K.dim() != 4:
        raise ValueError("K must be [B,H_kv,L,D]")
    Hkv = K.shape[1]
    if Hkv < 1 or H % Hkv != 0:
        raise ValueError("H (%d) must be a multiple of K's head count (%d)" % (H, Hkv))
    return Hkv


def _fwd(Q, K, V, key_mask, causal, window, scale, out_dtype, O, tau, stream, grouped, alpha=None):
    B, H, L, D = Q.shape
    Hkv = _kv_heads(Q, K, grouped or alpha is not None)
    lay = _layout_of(Q) if alpha is not None else ENTMAX_LAYOUT_BHLD  # strided inputs: _ex calls only
    _check_input("Q", Q, (B, H, L, D), None, lay)
    _check_input("K", K, (B, Hkv, L, D), Q.dtype, lay)
    _check_input("V", V, (B, Hkv, L, D), Q.dtype, lay)
    if scale is None:
        scale = D ** -0.5
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be bfloat16 or float32")
    if O is None:
        O = _empty((B, H, L, D), out_dtype, Q.device, lay)
    else:
        _check_input("O", O, (B, H, L, D), out_dtype, lay)
    if tau is None:
        tau = torch.empty((B, H, L), dtype=torch.float32, device=Q.device)
    else:
        _check_input("tau", tau, (B, H, L), torch.float32)
    if alpha is not None:
        args = (Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q), _mask_ptr(key_mask, B, L, Q.device),
                int(bool(causal)), int(window), float(scale), float(alpha), B, H, Hkv, L, D, lay, O.data_ptr(),
                ENTMAX_F32 if out_dtype == torch.float32 else ENTMAX_BF16, tau.data_ptr(), None, 0,
                _stream_handle(stream))
        name = "entmax_attn_fwd_ex"
    else:
        args = (Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q), _mask_ptr(key_mask, B, L, Q.device),
                int(bool(causal)), int(window), float(scale), B, H) + ((Hkv,) if grouped else ()) + (
                L, D, O.data_ptr(), ENTMAX_F32 if out_dtype == torch.float32 else ENTMAX_BF16, tau.data_ptr(),
                _stream_handle(stream))
        name = "entmax_attn_fwd_gqa" if grouped else "entmax_attn_fwd"
    st = getattr(lib, name)(*args)
    if st != ENTMAX_OK:
        raise EntmaxError(st, name)
    return O, tau


def entmax_attn_fwd(Q, K, V, key_mask=None, causal=False, window=0, scale=None, out_dtype=torch.bfloat16,
                    O=None, tau=None, stream=None):
    """1.5-entmax attention forward.  Q, K, V: [B,H,L,64] bf16 or fp32 CUDA tensors.

    Returns (O, tau): O [B,H,L,64] in ``out_dtype``; tau [B,H,L] fp32 thresholds.
    """
    return _fwd(Q, K, V, key_mask, causal, window, scale, out_dtype, O, tau, stream, False)


def entmax_attn_fwd_gqa(Q, K, V, key_mask=None, causal=False, window=0, scale=None, out_dtype=torch.bfloat16,
                        O=None, tau=None, stream=None):
    """Grouped-query forward: Q [B,H,L,64], K and V [B,H_kv,L,64] bf16 with H % H_kv == 0; query
    head h uses key/value head h // (H // H_kv).  Returns (O, tau) as entmax_attn_fwd."""
    return _fwd(Q, K, V, key_mask, causal, window, scale, out_dtype, O, tau, stream, True)


def entmax_attn_bwd_workspace_size(B: int, H: int, L: int, D: int = 64) -> int:
    """Bytes of device workspace for entmax_attn_bwd's fastest path (long rows list their supports
    from tau in it); the minimum it accepts is bwd_min_workspace_size."""
    return int(lib.entmax_attn_bwd_workspace_size(B, H, L, D))


def bwd_min_workspace_size(B: int, H: int, L: int) -> int:
    """The smallest workspace entmax_attn_bwd and entmax_attn_bwd_aux accept: one float per query
    row, rounded up to 256 bytes."""
    return (B * H * L * 4 + 255) // 256 * 256


def entmax_attn_bwd(Q, K, V, tau, dO, key_mask=None, causal=False, window=0, scale=None, dQ=None, dK=None,
                    dV=None, workspace=None, stream=None):
    """Closed-form backward.  Returns (dQ, dK, dV), fp32 [B,H,L,64]."""
    B, H, L, D = Q.shape
    _check_input("Q", Q, (B, H, L, D))
    _check_input("K", K, (B, H, L, D), Q.dtype)
    _check_input("V", V, (B, H, L, D), Q.dtype)
    _check_input("dO", dO, (B, H, L, D), Q.dtype)
    _check_input("tau", tau, (B, H, L), torch.float32)
    if scale is None:
        scale = D ** -0.5
    outs = []
    for name, t in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        if t is None:
            t = torch.empty((B, H, L, D), dtype=torch.float32, device=Q.device)
        else:
            _check_input(name, t, (B, H, L, D), torch.float32)
        outs.append(t)
    ws_bytes = entmax_attn_bwd_workspace_size(B, H, L, D)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=Q.device)
    st = lib.entmax_attn_bwd(Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q),
                             _mask_ptr(key_mask, B, L, Q.device), int(bool(causal)), int(window), float(scale),
                             B, H, L, D, tau.data_ptr(), dO.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(),
                             outs[2].data_ptr(), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream_handle(stream))
    if st != ENTMAX_OK:
        raise EntmaxError(st, "entmax_attn_bwd")
    return tuple(outs)


def entmax_attn_bwd_noalloc(Q, K, V, tau, dO, key_mask=None, causal=False, window=0, scale=None, dQ=None, dK=None,
                            dV=None, stream=None):
    """Backward pass without a workspace argument: the library's own fixed device scratch is used
    (bf16 inputs, at most 2**20 query rows; calls must not overlap on the GPU).  Returns (dQ, dK, dV)."""
    B, H, L, D = Q.shape
    _check_input("Q", Q, (B, H, L, D))
    _check_input("K", K, (B, H, L, D), Q.dtype)
    _check_input("V", V, (B, H, L, D), Q.dtype)
    _check_input("dO", dO, (B, H, L, D), Q.dtype)
    _check_input("tau", tau, (B, H, L), torch.float32)
    if scale is None:
        scale = D ** -0.5
    outs = []
    for name, t in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        if t is None:
            t = torch.empty((B, H, L, D), dtype=torch.float32, device=Q.device)
        else:
            _check_input(name, t, (B, H, L, D), torch.float32)
        outs.append(t)
    st = lib.entmax_attn_bwd_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q),
                                     _mask_ptr(key_mask, B, L, Q.device), int(bool(causal)), int(window),
                                     float(scale), B, H, L, D, tau.data_ptr(), dO.data_ptr(), outs[0].data_ptr(),
                                     outs[1].data_ptr(), outs[2].data_ptr(), _stream_handle(stream))
    if st != ENTMAX_OK:
        raise EntmaxError(st, "entmax_attn_bwd_noalloc")
    return tuple(outs)


def entmax_attn_fwd_aux(Q, K, V, key_mask=None, causal=False, window=0, scale=None, out_dtype=torch.bfloat16,
                        O=None, tau=None, Otil=None, rsum=None, stream=None):
    """Forward pass that also returns the auxiliary rows: Otil [B,H,L,64] fp32 (sum_j sqrt(p_ij) V_j)
    and rsum [B,H,L] fp32 (sum_j sqrt(p_ij)).  Returns (O, tau, Otil, rsum)."""
    B, H, L, D = Q.shape
    _check_input("Q", Q, (B, H, L, D))
    _check_input("K", K, (B, H, L, D), Q.dtype)
    _check_input("V", V, (B, H, L, D), Q.dtype)
    if scale is None:
        scale = D ** -0.5
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be bfloat16 or float32")
    outs = []
    for name, t, shape, dt in (("O", O, (B, H, L, D), out_dtype), ("tau", tau, (B, H, L), torch.float32),
                               ("Otil", Otil, (B, H, L, D), torch.float32), ("rsum", rsum, (B, H, L), torch.float32)):
        if t is None:
            t = torch.empty(shape, dtype=dt, device=Q.device)
        else:
            _check_input(name, t, shape, dt)
        outs.append(t)
    st = lib.entmax_attn_fwd_aux(Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q),
                                 _mask_ptr(key_mask, B, L, Q.device), int(bool(causal)), int(window), float(scale), B,
                                 H, L, D, outs[0].data_ptr(), ENTMAX_F32 if out_dtype == torch.float32 else ENTMAX_BF16,
                                 outs[1].data_ptr(), outs[2].data_ptr(), outs[3].data_ptr(), _stream_handle(stream))
    if st != ENTMAX_OK:
        raise EntmaxError(st, "entmax_attn_fwd_aux")
    return tuple(outs)


def entmax_attn_bwd_aux(Q, K, V, tau, Otil, rsum, dO, key_mask=None, causal=False, window=0, scale=None, dQ=None,
                        dK=None, dV=None, workspace=None, stream=None):
    """Backward pass taking the auxiliary rows of entmax_attn_fwd_aux.  Returns (dQ, dK, dV) fp32."""
    B, H, L, D = Q.shape
    _check_input("Q", Q, (B, H, L, D))
    _check_input("K", K, (B, H, L, D), Q.dtype)
    _check_input("V", V, (B, H, L, D), Q.dtype)
    _check_input("dO", dO, (B, H, L, D), Q.dtype)
    _check_input("tau", tau, (B, H, L), torch.float32)
    _check_input("Otil", Otil, (B, H, L, D), torch.float32)
    _check_input("rsum", rsum, (B, H, L), torch.float32)
    if scale is None:
        scale = D ** -0.5
    outs = []
    for name, t in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        if t is None:
            t = torch.empty((B, H, L, D), dtype=torch.float32, device=Q.device)
        else:
            _check_input(name, t, (B, H, L, D), torch.float32)
        outs.append(t)
    ws_bytes = bwd_min_workspace_size(B, H, L)  # the auxiliary rows' path needs the minimum only
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=Q.device)
    st = lib.entmax_attn_bwd_aux(Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q),
                                 _mask_ptr(key_mask, B, L, Q.device), int(bool(causal)), int(window), float(scale), B,
                                 H, L, D, tau.data_ptr(), Otil.data_ptr(), rsum.data_ptr(), dO.data_ptr(),
                                 outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if st != ENTMAX_OK:
        raise EntmaxError(st, "entmax_attn_bwd_aux")
    return tuple(outs)


def entmax_attn_saved_bytes(B: int, H: int, L: int, D: int = 64) -> int:
    """Bytes of the buffer the training forward saves the supports into (H: query heads)."""
    return int(lib.entmax_attn_saved_bytes(B, H, L, D))


def entmax_attn_bwd_saved_workspace_size(B: int, H: int, L: int, D: int = 64) -> int:
    """Bytes of device workspace the saved-support backward needs (H: query heads)."""
    return int(lib.entmax_attn_bwd_saved_workspace_size(B, H, L, D))


def _byte_buffer(t, nbytes: int, device, name: str):
    if t is None:
        return torch.empty((max(nbytes, 1),), dtype=torch.uint8, device=device)
    if not t.is_cuda or t.numel() * t.element_size() < nbytes:
        raise ValueError("%s must be a CUDA buffer of at least %d bytes" % (name, nbytes))
    return t


def _fwd_train(Q, K, V, key_mask, causal, window, scale, out_dtype, O, tau, saved, stream, grouped, alpha=None):
    B, H, L, D = Q.shape
    Hkv = _kv_heads(Q, K, grouped or alpha is not None)
    lay = _layout_of(Q) if alpha is not None else ENTMAX_LAYOUT_BHLD
    _check_input("Q", Q, (B, H, L, D), None, lay)
    _check_input("K", K, (B, Hkv, L, D), Q.dtype, lay)
    _check_input("V", V, (B, Hkv, L, D), Q.dtype, lay)
    if scale is None:
        scale = D ** -0.5
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be bfloat16 or float32")
    if O is None:
        O = _empty((B, H, L, D), out_dtype, Q.device, lay)
    else:
        _check_input("O", O, (B, H, L, D), out_dtype, lay)
    if tau is None:
        tau = torch.empty((B, H, L), dtype=torch.float32, device=Q.device)
    else:
        _check_input("tau", tau, (B, H, L), torch.float32)
    nbytes = entmax_attn_saved_bytes(B, H, L, D)
    saved = _byte_buffer(saved, nbytes, Q.device, "saved")
    if alpha is not None:
        args = (Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q), _mask_ptr(key_mask, B, L, Q.device),
                int(bool(causal)), int(window), float(scale), float(alpha), B, H, Hkv, L, D, lay, O.data_ptr(),
                ENTMAX_F32 if out_dtype == torch.float32 else ENTMAX_BF16, tau.data_ptr(), saved.data_ptr(),
                saved.numel() * saved.element_size(), _stream_handle(stream))
        name = "entmax_attn_fwd_ex"
    else:
        args = (Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q), _mask_ptr(key_mask, B, L, Q.device),
                int(bool(causal)), int(window), float(scale), B, H) + ((Hkv,) if grouped else ()) + (
                L, D, O.data_ptr(), ENTMAX_F32 if out_dtype == torch.float32 else ENTMAX_BF16, tau.data_ptr(),
                saved.data_ptr(), saved.numel() * saved.element_size(), _stream_handle(stream))
        name = "entmax_attn_fwd_train_gqa" if grouped else "entmax_attn_fwd_train"
    st = getattr(lib, name)(*args)
    if st != ENTMAX_OK:
        raise EntmaxError(st, name)
    return O, tau, saved


def entmax_attn_fwd_train(Q, K, V, key_mask=None, causal=False, window=0, scale=None, out_dtype=torch.bfloat16,
                          O=None, tau=None, saved=None, stream=None):
    """Forward pass that also saves each row's support for entmax_attn_bwd_saved.

    Returns (O, tau, saved); ``saved`` is an opaque uint8 device buffer."""
    return _fwd_train(Q, K, V, key_mask, causal, window, scale, out_dtype, O, tau, saved, stream, False)


def entmax_attn_fwd_train_gqa(Q, K, V, key_mask=None, causal=False, window=0, scale=None,
                              out_dtype=torch.bfloat16, O=None, tau=None, saved=None, stream=None):
    """Grouped-query training forward (K, V [B,H_kv,L,64] bf16).  Returns (O, tau, saved)."""
    return _fwd_train(Q, K, V, key_mask, causal, window, scale, out_dtype, O, tau, saved, stream, True)


def _bwd_saved(Q, K, V, tau, saved, dO, key_mask, causal, window, scale, dQ, dK, dV, workspace, stream, grouped,
               alpha=None):
    B, H, L, D = Q.shape
    Hkv = _kv_heads(Q, K, grouped or alpha is not None)
    lay = _layout_of(Q) if alpha is not None else ENTMAX_LAYOUT_BHLD
    _check_input("Q", Q, (B, H, L, D), None, lay)
    _check_input("K", K, (B, Hkv, L, D), Q.dtype, lay)
    _check_input("V", V, (B, Hkv, L, D), Q.dtype, lay)
    _check_input("dO", dO, (B, H, L, D), Q.dtype, lay)
    _check_input("tau", tau, (B, H, L), torch.float32)
    if scale is None:
        scale = D ** -0.5
    outs = []
    for name, t, heads in (("dQ", dQ, H), ("dK", dK, Hkv), ("dV", dV, Hkv)):
        if t is None:
            t = _empty((B, heads, L, D), torch.float32, Q.device, lay)
        else:
            _check_input(name, t, (B, heads, L, D), torch.float32, lay)
        outs.append(t)
    ws = _byte_buffer(workspace, entmax_attn_bwd_saved_workspace_size(B, H, L, D), Q.device, "workspace")
    head = (float(alpha), B, H, Hkv) if alpha is not None else (B, H, Hkv) if grouped else (B, H)
    args = (Q.data_ptr(), K.data_ptr(), V.data_ptr(), _dtype_code(Q), _mask_ptr(key_mask, B, L, Q.device),
            int(bool(causal)), int(window), float(scale)) + head + (L, D) + ((lay,) if alpha is not None else ()) + (
            tau.data_ptr(), saved.data_ptr(), saved.numel() * saved.element_size(), dO.data_ptr(),
            outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(), ws.data_ptr(),
            ws.numel() * ws.element_size(), _stream_handle(stream))
    name = ("entmax_attn_bwd_saved_ex" if alpha is not None else
            "entmax_attn_bwd_saved_gqa" if grouped else "entmax_attn_bwd_saved")
    st = getattr(lib, name)(*args)
    if st != ENTMAX_OK:
        raise EntmaxError(st, name)
    return tuple(outs)


def entmax_attn_bwd_saved(Q, K, V, tau, saved, dO, key_mask=None, causal=False, window=0, scale=None, dQ=None,
                          dK=None, dV=None, workspace=None, stream=None):
    """Backward pass from the supports saved by entmax_attn_fwd_train.  Returns (dQ, dK, dV) fp32."""
    return _bwd_saved(Q, K, V, tau, saved, dO, key_mask, causal, window, scale, dQ, dK, dV, workspace, stream,
                      False)


def entmax_attn_bwd_saved_gqa(Q, K, V, tau, saved, dO, key_mask=None, causal=False, window=0, scale=None, dQ=None,
                              dK=None, dV=None, workspace=None, stream=None):
    """Grouped-query backward from entmax_attn_fwd_train_gqa's supports.  Returns dQ [B,H,L,64] and
    dK, dV [B,H_kv,L,64] (fp32), each key/value head's gradient summed over the query heads sharing it."""
    return _bwd_saved(Q, K, V, tau, saved, dO, key_mask, causal, window, scale, dQ, dK, dV, workspace, stream,
                      True)


def entmax_attn_fwd_ex(Q, K, V, key_mask=None, causal=False, window=0, scale=None, alpha=1.5, save=False,
                       out_dtype=torch.bfloat16, O=None, tau=None, saved=None, stream=None):
    """alpha-entmax forward, alpha in [1, 2] (|alpha - 1| < 1e-4: softmax, tau = log sum exp of the
    row's scores); K and V may have fewer heads than Q (H % H_kv == 0).

    Q, K, V are [B,H,L,64] tensors: contiguous, or all three the transpose(1, 2) views of contiguous
    [B,L,H,64] tensors (then O is returned in that layout too).  Returns (O, tau) or, with
    ``save=True``, (O, tau, saved) for entmax_attn_bwd_saved_ex."""
    if save:
        return _fwd_train(Q, K, V, key_mask, causal, window, scale, out_dtype, O, tau, saved, stream, True, alpha)
    return _fwd(Q, K, V, key_mask, causal, window, scale, out_dtype, O, tau, stream, True, alpha)


def entmax_attn_bwd_saved_ex(Q, K, V, tau, saved, dO, key_mask=None, causal=False, window=0, scale=None, alpha=1.5,
                             dQ=None, dK=None, dV=None, workspace=None, stream=None):
    """Backward of entmax_attn_fwd_ex(save=True) with the same alpha.  Returns dQ [B,H,L,64] and
    dK, dV [B,H_kv,L,64], fp32, in the memory layout of Q (dO must share it)."""
    return _bwd_saved(Q, K, V, tau, saved, dO, key_mask, causal, window, scale, dQ, dK, dV, workspace, stream, True,
                      alpha)


def entmax_attn_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(lib.entmax_attn_device_status(_stream_handle(stream)))


def entmax_attn_set_wait_timeout_ns(ns: int) -> None:
    """Bound on each device-side wait for later launches, in nanoseconds (0: the default, 2 s)."""
    lib.entmax_attn_set_wait_timeout_ns(int(ns))


def entmax_attn_last_cuda_error() -> int:
    """cudaError_t value of the most recent failed CUDA call inside the library (0 if none)."""
    return int(lib.entmax_attn_last_cuda_error())


class EntmaxAttention(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run in the library's kernels."""

    @staticmethod
    def forward(ctx, Q, K, V, key_mask=None, causal=False, window=0, scale=None, alpha=1.5):
        grouped = K.shape[1] != Q.shape[1]  # K, V with fewer heads than Q: grouped-query attention
        # other alpha, or [B,L,H,D] memory behind the [B,H,L,D] views: the _ex entry points
        a = None if alpha == 1.5 and Q.is_contiguous() else float(alpha)
        O, tau, saved = _fwd_train(Q, K, V, key_mask, causal, window, scale, torch.bfloat16, None, None, None, None,
                                   grouped, a)
        ctx.save_for_backward(Q, K, V, tau, saved, key_mask if key_mask is not None else torch.empty(0))
        ctx.cfg = (key_mask is not None, causal, window, scale, grouped, a)
        return O

    @staticmethod
    def backward(ctx, dO):
        Q, K, V, tau, saved, km = ctx.saved_tensors
        has_mask, causal, window, scale, grouped, a = ctx.cfg
        g = dO.to(Q.dtype)
        if a is not None and _layout_of(Q) == ENTMAX_LAYOUT_BLHD:
            g = g.transpose(1, 2).contiguous().transpose(1, 2)  # dO in Q's memory layout
        else:
            g = g.contiguous()
        dQ, dK, dV = _bwd_saved(Q, K, V, tau, saved, g, km if has_mask else None, causal, window, scale, None, None,
                                None, None, None, grouped, a)
        return dQ.to(Q.dtype), dK.to(K.dtype), dV.to(V.dtype), None, None, None, None, None
