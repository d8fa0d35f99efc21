"""fp64 CPU oracle for 1.5-entmax attention -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may
import this module.  The product path (the CUDA library and its binding)
never calls it, and it imports nothing from the product package.

Thin ctypes wrapper over ``entmax_oracle.c``; every function below names the
passage of the AdaSplash pages it restates (page "svd-sst2-roberta-adasplash",
sections 2.1-2.4; model cards "roberta-base-adasplash" and
"distilbert-sst2-adasplash", section "Mathematical Formulation").

Parity status: every function here is pinned by tests/test_oracle_pins.py to
facts fixed by the pages or by mathematics (closed forms, the argmax
definition solved by a generic optimiser, KKT brute force on tiny rows,
finite differences); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "entmax_oracle.c"
_LIB = _HERE / "liboracle.so"

_dp = ctypes.POINTER(ctypes.c_double)
_fp = ctypes.POINTER(ctypes.c_float)
_u8p = ctypes.POINTER(ctypes.c_ubyte)
_i64p = ctypes.POINTER(ctypes.c_longlong)


def build(force: bool = False) -> Path:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, OpenMP, no fast-math)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(".so.tmp%d" % os.getpid())
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(tmp), str(_SRC), "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(str(build()))
        lib.eo_round_bf16.restype = ctypes.c_double
        lib.eo_round_bf16.argtypes = [ctypes.c_float]
        lib.eo_round_bf16_array.argtypes = [_fp, _dp, ctypes.c_longlong]
        lib.eo_g.restype = ctypes.c_double
        lib.eo_g.argtypes = [_dp, ctypes.c_int, ctypes.c_double]
        lib.eo_tau_sort.restype = ctypes.c_int
        lib.eo_tau_sort.argtypes = [_dp, ctypes.c_int, _dp]
        for name in ("eo_tau_bisect", "eo_tau_bisect_wide"):
            f = getattr(lib, name)
            f.restype = ctypes.c_double
            f.argtypes = [_dp, ctypes.c_int, ctypes.c_int]
        lib.eo_tau_bisect_bracket.restype = ctypes.c_double
        lib.eo_tau_bisect_bracket.argtypes = [_dp, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int]
        lib.eo_entmax15.argtypes = [_dp, ctypes.c_int, ctypes.c_double, _dp]
        lib.eo_entmax15_jvp.argtypes = [_dp, _dp, ctypes.c_int, _dp]
        lib.eo_attn_fwd_rows.argtypes = [_dp, _dp, _dp, _u8p, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                         ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         _i64p, ctypes.c_longlong, ctypes.c_int, ctypes.c_int, _dp, _dp]
        lib.eo_attn_fwd.argtypes = [_dp, _dp, _dp, _u8p, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                    ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, _dp, _dp]
        lib.eo_attn_aux_rows.argtypes = [_dp, _dp, _dp, _u8p, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i64p,
                                         ctypes.c_longlong, _dp, _dp]
        lib.eo_attn_bwd_heads.argtypes = [_dp, _dp, _dp, _u8p, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          _dp, _i64p, ctypes.c_int, _dp, _dp, _dp]
        lib.eo_g_alpha.restype = ctypes.c_double
        lib.eo_g_alpha.argtypes = [_dp, ctypes.c_int, ctypes.c_double, ctypes.c_double]
        lib.eo_tau_alpha.restype = ctypes.c_double
        lib.eo_tau_alpha.argtypes = [_dp, ctypes.c_int, ctypes.c_double]
        lib.eo_tau_alpha_bisect.restype = ctypes.c_double
        lib.eo_tau_alpha_bisect.argtypes = [_dp, ctypes.c_int, ctypes.c_double, ctypes.c_int]
        lib.eo_entmax_alpha.argtypes = [_dp, ctypes.c_int, ctypes.c_double, ctypes.c_double, _dp]
        lib.eo_entmax_alpha_jvp.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_double, _dp]
        lib.eo_tau_softmax.restype = ctypes.c_double
        lib.eo_tau_softmax.argtypes = [_dp, ctypes.c_int]
        lib.eo_softmax.argtypes = [_dp, ctypes.c_int, ctypes.c_double, _dp]
        lib.eo_num_threads.restype = ctypes.c_int
        lib.eo_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _d(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def num_threads() -> int:
    return _load().eo_num_threads()


def set_num_threads(n: int) -> None:
    _load().eo_set_num_threads(int(n))


# --------------------------------------------------------------------------
# element-level functions
# --------------------------------------------------------------------------
def round_bf16(x) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even), returned as fp64."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.float64)
    _load().eo_round_bf16_array(x.ctypes.data_as(_fp), _d(out), x.size)
    return out


def g(s, tau: float) -> float:
    """g(tau) = sum_i [(s_i - tau)/2]_+^2 (Theorem 1)."""
    s = _f64(s)
    return _load().eo_g(_d(s), s.size, float(tau))


def tau_sort(s):
    """Exact tau by the sorted closed form; returns (tau, support size)."""
    s = _f64(s)
    t = ctypes.c_double()
    k = _load().eo_tau_sort(_d(s), s.size, ctypes.byref(t))
    return t.value, k


def tau_bisect(s, n_iter: int = 25) -> float:
    """Bisection on the model cards' bracket [max-2, max-2/sqrt(n)] (Theorem 2)."""
    s = _f64(s)
    return _load().eo_tau_bisect(_d(s), s.size, int(n_iter))


def tau_bisect_wide(s, n_iter: int = 25) -> float:
    """Bisection on Theorem 2's bracket [min-2, max]."""
    s = _f64(s)
    return _load().eo_tau_bisect_wide(_d(s), s.size, int(n_iter))


def entmax15(s, tau: float | None = None) -> np.ndarray:
    """p = [(s - tau)/2]_+^2 with tau exact (Theorem 1) unless given."""
    s = _f64(s)
    if tau is None:
        tau = tau_sort(s)[0]
    p = np.empty_like(s)
    _load().eo_entmax15(_d(s), s.size, float(tau), _d(p))
    return p


def entmax15_jvp(p, gvec) -> np.ndarray:
    """dL/ds from dL/dp by the closed-form Jacobian of section 2.4."""
    p = _f64(p)
    gvec = _f64(gvec)
    ds = np.empty_like(p)
    _load().eo_entmax15_jvp(_d(p), _d(gvec), p.size, _d(ds))
    return ds


def g_alpha(s, tau: float, alpha: float) -> float:
    """sum_i max(0, (alpha-1)(s_i - tau))^(1/(alpha-1)) (the alpha-entmax constraint function)."""
    s = _f64(s)
    return _load().eo_g_alpha(_d(s), s.size, float(tau), float(alpha))


def tau_alpha(s, alpha: float) -> float:
    """alpha-entmax threshold (score units) by bisection run to fp64 convergence on
    [max - 1/(alpha-1), max - n^(1-alpha)/(alpha-1)] -- the pages' bisection (page
    "svd-sst2-roberta-adasplash", section 4, entmax_bisect) taken to its limit."""
    s = _f64(s)
    return _load().eo_tau_alpha(_d(s), s.size, float(alpha))


def tau_alpha_bisect(s, alpha: float, n_iter: int = 25) -> float:
    """The same bracket halved n_iter times, final midpoint."""
    s = _f64(s)
    return _load().eo_tau_alpha_bisect(_d(s), s.size, float(alpha), int(n_iter))


def entmax_alpha(s, alpha: float, tau: float | None = None) -> np.ndarray:
    """p = max(0, (alpha-1)(s - tau))^(1/(alpha-1)), tau from tau_alpha unless given."""
    s = _f64(s)
    if tau is None:
        tau = tau_alpha(s, alpha)
    p = np.empty_like(s)
    _load().eo_entmax_alpha(_d(s), s.size, float(tau), float(alpha), _d(p))
    return p


def entmax_alpha_jvp(p, gvec, alpha: float) -> np.ndarray:
    """dL/ds from dL/dp for alpha-entmax: w = p^(2-alpha), ds = w (g - <w, g>/sum w)."""
    p = _f64(p)
    gvec = _f64(gvec)
    ds = np.empty_like(p)
    _load().eo_entmax_alpha_jvp(_d(p), _d(gvec), p.size, float(alpha), _d(ds))
    return ds


def tau_softmax(s) -> float:
    """alpha = 1 (softmax): tau = log sum_k exp(s_k), so that p = exp(s - tau) sums to 1 (the pages'
    branch for |alpha - 1| < 1e-4, page "svd-sst2-roberta-adasplash", section 4, entmax_bisect)."""
    s = _f64(s)
    return _load().eo_tau_softmax(_d(s), s.size)


def softmax(s, tau: float | None = None) -> np.ndarray:
    """p = exp(s - tau), tau from tau_softmax unless given."""
    s = _f64(s)
    if tau is None:
        tau = tau_softmax(s)
    p = np.empty_like(s)
    _load().eo_softmax(_d(s), s.size, float(tau), _d(p))
    return p


# --------------------------------------------------------------------------
# attention (alpha = 1.5 unless given; other alpha in (1, 2] use tau_alpha, alpha = 1 is softmax)
# --------------------------------------------------------------------------
def _mask_arg(key_mask, B, L):
    if key_mask is None:
        return None, None
    m = np.ascontiguousarray(np.asarray(key_mask, dtype=np.uint8).reshape(B, L))
    return m, m.ctypes.data_as(_u8p)


def _alpha_arg(alpha) -> float:
    a = float(alpha)
    if not (a == 1.0 or 1.0 < a <= 2.0):
        raise ValueError("alpha must be 1 (softmax) or lie in (1, 2], got %r" % alpha)
    return a


def attn_fwd(Q, K, V, key_mask=None, causal=False, window=0, scale=0.125, tau_method="sort", alpha=1.5):
    """Full forward. Q,K,V: [B,H,L,D] (values already bf16-rounded). Returns (O, tau)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, L, D = Q.shape
    m, mp = _mask_arg(key_mask, B, L)
    O = np.empty_like(Q)
    tau = np.empty((B, H, L), dtype=np.float64)
    _load().eo_attn_fwd(_d(Q), _d(K), _d(V), mp, int(bool(causal)), int(window), float(scale), _alpha_arg(alpha),
                        B, H, L, D, 0 if tau_method == "sort" else 1, _d(O), _d(tau))
    return O, tau


def attn_fwd_rows(Q, K, V, row_ids, key_mask=None, causal=False, window=0, scale=0.125,
                  tau_method="sort", n_iter=25, alpha=1.5):
    """Forward for selected rows (row id = (b*H + h)*L + i). Returns (O_rows, tau_rows)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, L, D = Q.shape
    m, mp = _mask_arg(key_mask, B, L)
    ids = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    O = np.empty((ids.size, D), dtype=np.float64)
    tau = np.empty((ids.size,), dtype=np.float64)
    _load().eo_attn_fwd_rows(_d(Q), _d(K), _d(V), mp, int(bool(causal)), int(window), float(scale),
                             _alpha_arg(alpha), B, H, L, D, ids.ctypes.data_as(_i64p), ids.size,
                             0 if tau_method == "sort" else 1, int(n_iter), _d(O), _d(tau))
    return O, tau


def attn_aux_rows(Q, K, V, row_ids, key_mask=None, causal=False, window=0, scale=0.125):
    """Auxiliary rows (1.5-entmax) of selected rows: Otil_i = sum_j sqrt(p_ij) V_j and
    r_i = sum_j sqrt(p_ij), the factors of the backward's row scalar u_i = dO_i . Otil_i / r_i (page
    "svd-sst2-roberta-adasplash", section 2.4).  Returns (Otil_rows [n, D], r_rows [n])."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, L, D = Q.shape
    m, mp = _mask_arg(key_mask, B, L)
    ids = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    Ot = np.empty((ids.size, D), dtype=np.float64)
    r = np.empty((ids.size,), dtype=np.float64)
    _load().eo_attn_aux_rows(_d(Q), _d(K), _d(V), mp, int(bool(causal)), int(window), float(scale), B, H, L, D,
                             ids.ctypes.data_as(_i64p), ids.size, _d(Ot), _d(r))
    return Ot, r


def attn_bwd_heads(Q, K, V, dO, bh_ids, key_mask=None, causal=False, window=0, scale=0.125, alpha=1.5):
    """Gradients (dQ, dK, dV) of <dO, O> for the listed heads bh = b*H + h, each [n, L, D]."""
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    B, H, L, D = Q.shape
    m, mp = _mask_arg(key_mask, B, L)
    ids = np.ascontiguousarray(np.asarray(bh_ids, dtype=np.int64))
    n = ids.size
    dQ = np.empty((n, L, D), dtype=np.float64)
    dK = np.empty((n, L, D), dtype=np.float64)
    dV = np.empty((n, L, D), dtype=np.float64)
    _load().eo_attn_bwd_heads(_d(Q), _d(K), _d(V), mp, int(bool(causal)), int(window), float(scale),
                              _alpha_arg(alpha), B, H, L, D, _d(dO), ids.ctypes.data_as(_i64p), n, _d(dQ), _d(dK),
                              _d(dV))
    return dQ, dK, dV


def attn_bwd(Q, K, V, dO, key_mask=None, causal=False, window=0, scale=0.125, alpha=1.5):
    """Full backward; returns dQ, dK, dV shaped [B,H,L,D]."""
    B, H, L, D = np.shape(Q)
    dQ, dK, dV = attn_bwd_heads(Q, K, V, dO, np.arange(B * H), key_mask, causal, window, scale, alpha)
    return dQ.reshape(B, H, L, D), dK.reshape(B, H, L, D), dV.reshape(B, H, L, D)


# --------------------------------------------------------------------------
# grouped-query attention
# --------------------------------------------------------------------------
def repeat_kv(X, n_rep: int) -> np.ndarray:
    """[B, H_kv, L, D] -> [B, H_kv*n_rep, L, D]: each key/value head copied n_rep times in a row, so
    query head h reads key/value head h // n_rep.  Page "svd-sst2-roberta-adasplash", section 3 (the
    grouped-query repeat step of the tensor trace, taken before the scores) and section 4 (the
    attention layer's forward repeats k and v by H // H_kv)."""
    X = _f64(X)
    return np.repeat(X, int(n_rep), axis=1)


def _n_rep(Q, K) -> int:
    H, Hkv = np.shape(Q)[1], np.shape(K)[1]
    if Hkv < 1 or H % Hkv:
        raise ValueError("query heads (%d) must be a multiple of key/value heads (%d)" % (H, Hkv))
    return H // Hkv


def attn_fwd_gqa(Q, K, V, key_mask=None, causal=False, window=0, scale=0.125, tau_method="sort", alpha=1.5):
    """Grouped-query forward: K, V [B,H_kv,L,D] repeated to H heads, then attn_fwd.  (O, tau)."""
    r = _n_rep(Q, K)
    return attn_fwd(Q, repeat_kv(K, r), repeat_kv(V, r), key_mask, causal, window, scale, tau_method, alpha)


def attn_fwd_rows_gqa(Q, K, V, row_ids, key_mask=None, causal=False, window=0, scale=0.125,
                      tau_method="sort", n_iter=25, alpha=1.5):
    """attn_fwd_rows on the repeated K and V (row id = (b*H + h)*L + i over the query heads)."""
    r = _n_rep(Q, K)
    return attn_fwd_rows(Q, repeat_kv(K, r), repeat_kv(V, r), row_ids, key_mask, causal, window, scale,
                         tau_method, n_iter, alpha)


def attn_bwd_gqa(Q, K, V, dO, key_mask=None, causal=False, window=0, scale=0.125, alpha=1.5):
    """Grouped-query backward.  The repeat copies each key/value head to n_rep query heads, so by the
    chain rule its gradient is the sum of the copies' gradients over those heads.  Returns dQ
    [B,H,L,D] and dK, dV [B,H_kv,L,D]."""
    r = _n_rep(Q, K)
    B, Hkv, L, D = np.shape(K)
    dQ, dKr, dVr = attn_bwd(Q, repeat_kv(K, r), repeat_kv(V, r), dO, key_mask, causal, window, scale, alpha)
    return dQ, dKr.reshape(B, Hkv, r, L, D).sum(axis=2), dVr.reshape(B, Hkv, r, L, D).sum(axis=2)
