"""Softmax attention (alpha = 1) on the GPU vs the fp64 oracle.

The alpha-entmax routine of page "svd-sst2-roberta-adasplash", section 4 (entmax_bisect) returns
softmax when |alpha - 1| < 1e-4; the _ex entry points do the same: p_ij = exp(S_ij - tau_i) with
tau_i = log sum_j exp(S_ij) over the allowed keys.  Forward (O, tau) and backward (dQ, dK, dV) run on
the tensor cores.  Shapes span several 128-row tiles and 64-key blocks with ragged tails, padding
down to one key, causal masks and windows, grouped heads and the [B, L, H, 64] layout; a long
sequence is compared on sampled rows and heads.  Tolerances: tests/gpu_helpers.py (the same bounds
as the entmax paths; softmax gets no wider ones).
"""
import numpy as np
import pytest
import torch

from entmax_tcgen05_tma_b200 import (
    EntmaxAttention,
    entmax_attn_bwd_saved_ex,
    entmax_attn_device_status,
    entmax_attn_fwd_ex,
)
from entmax_tcgen05_tma_b200.workloads import Workload, make_inputs
from oracle import oracle as orc
from tests.gpu_helpers import GRAD_TOL, O_TOL, TAU_TOL, assert_bf16_is_rounded, check_rows, inputs_f64, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _dev(inp):
    Q, K, V, dO = (inp[k].to(DEV) for k in ("Q", "K", "V", "dO"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(DEV)
    return Q, K, V, dO, km


def _mask_np(inp):
    return None if inp["key_mask"] is None else inp["key_mask"].numpy()


def _blhd(x: torch.Tensor) -> torch.Tensor:
    """The same values as x [B,H,L,D], held in [B,L,H,D] memory (a transpose(1, 2) view)."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


CASES = [
    # B, H, H_kv, L, scale, causal, window, len_range
    (1, 2, 2, 64, 1 / 8, False, 0, None),
    (2, 2, 2, 129, 2 / 8, False, 0, None),
    (3, 2, 2, 300, 1 / 8, False, 0, (1, 300)),
    (2, 2, 2, 300, 2 / 8, True, 32, None),
    (1, 2, 2, 513, 1 / 8, True, 0, (200, 513)),
    (1, 1, 1, 700, 2 / 8, True, 5, None),
    (1, 2, 2, 1000, 1 / 8, False, 0, None),
    (2, 4, 2, 257, 1 / 8, True, 0, (30, 257)),
    (1, 6, 2, 640, 2 / 8, False, 0, None),
]


@pytest.mark.parametrize("B,H,Hkv,L,scale,causal,window,lens", CASES)
def test_softmax_small_full_parity(B, H, Hkv, L, scale, causal, window, lens):
    w = Workload(0, "softmax", B, H, L, 64, scale, causal, window, lens, H_kv=Hkv)
    inp = make_inputs(w, seed=71 + L + H)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    Q, K, V, dO, kmd = _dev(inp)
    O, tau = entmax_attn_fwd_ex(Q, K, V, kmd, causal, window, scale, alpha=1.0, out_dtype=torch.float32)
    assert entmax_attn_device_status() == 0
    r = H // Hkv
    Kr, Vr = orc.repeat_kv(d["K"], r), orc.repeat_kv(d["V"], r)
    O_ref, tau_ref = orc.attn_fwd(d["Q"], Kr, Vr, km, causal, window, scale, alpha=1.0)
    Og, tg = to64(O), to64(tau)
    assert np.array_equal(np.isfinite(tg), np.isfinite(tau_ref))
    assert np.max(np.abs(Og - O_ref)) <= O_TOL
    fin = np.isfinite(tau_ref)
    assert np.max(np.abs(tg[fin] - tau_ref[fin]), initial=0.0) <= TAU_TOL
    check_rows(d["Q"], Kr, np.arange(B * H * L), tg.reshape(-1), tau_ref.reshape(-1), km, causal, window, scale, H,
               L, alpha=1.0)
    # the training forward and bf16 output: the same values
    Ob, taub, saved = entmax_attn_fwd_ex(Q, K, V, kmd, causal, window, scale, alpha=1.0, save=True)
    assert torch.equal(tau, taub)
    assert_bf16_is_rounded(Ob, O)
    dQ, dK, dV = entmax_attn_bwd_saved_ex(Q, K, V, taub, saved, dO, kmd, causal, window, scale, alpha=1.0)
    assert entmax_attn_device_status() == 0
    rQ, rK, rV = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], km, causal, window, scale, alpha=1.0)
    for name, g, ref in (("dQ", dQ, rQ), ("dK", dK, rK), ("dV", dV, rV)):
        err = np.max(np.abs(to64(g) - ref))
        assert err <= GRAD_TOL, (name, err)


def test_softmax_band_and_blhd_layout():
    """alpha within 1e-4 of 1 is softmax (bit-equal to alpha = 1); [B,L,H,64] memory gives the same
    O, tau and gradients bit for bit (the same arithmetic in both layouts, no atomics)."""
    w = Workload(0, "softmax-layout", 2, 4, 300, 64, 1 / 8, True, 0, (1, 300), H_kv=2)
    inp = make_inputs(w, seed=79)
    Q, K, V, dO, km = _dev(inp)
    O, tau, saved = entmax_attn_fwd_ex(Q, K, V, km, True, 0, w.scale, alpha=1.0, save=True, out_dtype=torch.float32)
    g = entmax_attn_bwd_saved_ex(Q, K, V, tau, saved, dO, km, True, 0, w.scale, alpha=1.0)
    for a in (1.00005, 0.99995):
        O2, tau2 = entmax_attn_fwd_ex(Q, K, V, km, True, 0, w.scale, alpha=a, out_dtype=torch.float32)
        assert torch.equal(O, O2) and torch.equal(tau, tau2)
    Ql, Kl, Vl, dOl = (_blhd(x) for x in (Q, K, V, dO))
    O3, tau3, saved3 = entmax_attn_fwd_ex(Ql, Kl, Vl, km, True, 0, w.scale, alpha=1.0, save=True,
                                          out_dtype=torch.float32)
    g3 = entmax_attn_bwd_saved_ex(Ql, Kl, Vl, tau3, saved3, dOl, km, True, 0, w.scale, alpha=1.0)
    assert entmax_attn_device_status() == 0
    assert torch.equal(O3, O) and torch.equal(tau3, tau)
    for x, y in zip(g3, g):
        assert torch.equal(x, y)


def test_softmax_fully_padded_batch_and_repeatability():
    w = Workload(0, "softmax-empty", 2, 2, 200, 64, 1 / 8, len_range=(50, 50))
    inp = make_inputs(w, seed=83)
    inp["key_mask"][1] = 0
    Q, K, V, dO, km = _dev(inp)
    outs = []
    for _ in range(2):
        O, tau, saved = entmax_attn_fwd_ex(Q, K, V, km, False, 0, w.scale, alpha=1.0, save=True)
        g = entmax_attn_bwd_saved_ex(Q, K, V, tau, saved, dO, km, False, 0, w.scale, alpha=1.0)
        assert entmax_attn_device_status() == 0
        outs.append((O, tau) + tuple(g))
    O, tau, dQ, dK, dV = outs[0]
    assert torch.all(O[1] == 0) and torch.all(torch.isinf(tau[1])) and torch.all(torch.isfinite(tau[0]))
    for t in (dQ, dK, dV):
        assert torch.all(t[1] == 0) and torch.isfinite(t).all()
    for x, y in zip(outs[0], outs[1]):
        assert torch.equal(x, y)


def test_softmax_autograd_function():
    w = Workload(0, "softmax-autograd", 1, 2, 200, 64, 1 / 8, True, 0)
    inp = make_inputs(w, seed=89)
    d = inputs_f64(inp, False)
    Q, K, V, dO, _ = _dev(inp)
    Q.requires_grad_(True)
    K.requires_grad_(True)
    V.requires_grad_(True)
    O = EntmaxAttention.apply(Q, K, V, None, True, 0, w.scale, 1.0)
    O.backward(dO)
    refs = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], None, True, 0, w.scale, alpha=1.0)
    for name, g, ref in zip(("dQ", "dK", "dV"), (Q.grad, K.grad, V.grad), refs):
        err = np.max(np.abs(to64(g) - ref))
        assert err <= GRAD_TOL + 2 ** -8 * np.max(np.abs(ref)), (name, err)  # gradients returned in bf16


@pytest.mark.parametrize("shape", [
    # B, H, L, scale, causal, window: long rows (workload 4's shape) and a causal decoder shape
    (4, 12, 4096, 2 / 8, False, 0),
    (8, 12, 1024, 1 / 8, True, 0),
])
def test_softmax_full_size(shape):
    B, H, L, scale, causal, window = shape
    w = Workload(0, "softmax-full", B, H, L, 64, scale, causal, window)
    inp = make_inputs(w, seed=97)
    d = inputs_f64(inp, False)
    Q, K, V, dO, _ = _dev(inp)
    Ob, tau, saved = entmax_attn_fwd_ex(Q, K, V, None, causal, window, scale, alpha=1.0, save=True)
    O, tau2 = entmax_attn_fwd_ex(Q, K, V, None, causal, window, scale, alpha=1.0, out_dtype=torch.float32)
    assert entmax_attn_device_status() == 0
    assert torch.equal(tau, tau2)
    assert_bf16_is_rounded(Ob, O)
    BH = B * H
    rng = np.random.default_rng(L)
    ids = np.unique(np.concatenate([rng.integers(0, BH * L, size=160), [0, L - 1, BH * L - 1]]))
    O_ref, tau_ref = orc.attn_fwd_rows(d["Q"], d["K"], d["V"], ids, None, causal, window, scale, alpha=1.0)
    assert np.max(np.abs(to64(O).reshape(-1, 64)[ids] - O_ref)) <= O_TOL
    check_rows(d["Q"], d["K"], ids, to64(tau).reshape(-1)[ids], tau_ref, None, causal, window, scale, H, L,
               alpha=1.0)
    dQ, dK, dV = entmax_attn_bwd_saved_ex(Q, K, V, tau, saved, dO, None, causal, window, scale, alpha=1.0)
    assert entmax_attn_device_status() == 0
    heads = [0, BH - 1]
    refs = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], heads, None, causal, window, scale, alpha=1.0)
    for name, g, ref in zip(("dQ", "dK", "dV"), (dQ, dK, dV), refs):
        err = np.max(np.abs(to64(g).reshape(BH, L, 64)[heads] - ref))
        assert err <= GRAD_TOL, (name, err)
