"""Grouped-query attention on the GPU (the *_gqa entry points) vs the fp64 oracle.

Query head h of batch b reads key/value head b*H_kv + h // (H/H_kv).  The oracle repeats K and V to H
heads and sums the repeated heads' dK/dV over each group.  Shapes span several 128-row tiles with
ragged tails; one case is a decoder-sized head layout compared on sampled rows and one group's
heads.  Tolerances: tests/gpu_helpers.py.
"""
import numpy as np
import pytest
import torch

from entmax_tcgen05_tma_b200 import (
    EntmaxAttention,
    EntmaxError,
    entmax_attn_bwd_saved,
    entmax_attn_bwd_saved_gqa,
    entmax_attn_device_status,
    entmax_attn_fwd,
    entmax_attn_fwd_gqa,
    entmax_attn_fwd_train,
    entmax_attn_fwd_train_gqa,
)
from entmax_tcgen05_tma_b200.workloads import Workload, make_inputs
from oracle import oracle as orc
from tests.gpu_helpers import GRAD_TOL, O_TOL, assert_bf16_is_rounded, check_rows, inputs_f64, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _dev(inp):
    Q, K, V, dO = (inp[k].to(DEV) for k in ("Q", "K", "V", "dO"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(DEV)
    return Q, K, V, dO, km


def _mask_np(inp):
    return None if inp["key_mask"] is None else inp["key_mask"].numpy()


GQA = [
    # B, H, H_kv, L, scale, causal, window, len_range
    (1, 4, 1, 64, 1 / 8, False, 0, None),
    (2, 4, 2, 300, 1 / 8, False, 0, (1, 300)),
    (2, 6, 3, 129, 2 / 8, False, 0, None),
    (1, 8, 2, 513, 1 / 8, True, 0, (200, 513)),
    (2, 8, 4, 700, 1 / 8, True, 32, None),
    (1, 3, 3, 200, 1 / 8, True, 0, None),  # H_kv = H through the grouped entry points
]


@pytest.mark.parametrize("B,H,Hkv,L,scale,causal,window,lens", GQA)
def test_gqa_small_full_parity(B, H, Hkv, L, scale, causal, window, lens):
    w = Workload(0, "gqa", B, H, L, 64, scale, causal, window, lens, H_kv=Hkv)
    inp = make_inputs(w, seed=31 + L + H + Hkv)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    Q, K, V, dO, kmd = _dev(inp)
    O, tau = entmax_attn_fwd_gqa(Q, K, V, kmd, causal, window, scale, out_dtype=torch.float32)
    assert entmax_attn_device_status() == 0
    O_ref, tau_ref = orc.attn_fwd_gqa(d["Q"], d["K"], d["V"], km, causal, window, scale)
    Og, tg = to64(O), to64(tau)
    assert np.array_equal(np.isfinite(tg), np.isfinite(tau_ref))
    assert np.max(np.abs(Og - O_ref)) <= O_TOL
    Kr = orc.repeat_kv(d["K"], H // Hkv)
    check_rows(d["Q"], Kr, np.arange(B * H * L), tg.reshape(-1), tau_ref.reshape(-1), km, causal, window, scale, H,
               L)
    # training forward: the same O and tau, plus the saved supports for the backward
    O2, tau2, saved = entmax_attn_fwd_train_gqa(Q, K, V, kmd, causal, window, scale, out_dtype=torch.float32)
    assert torch.equal(O, O2) and torch.equal(tau, tau2)
    dQ, dK, dV = entmax_attn_bwd_saved_gqa(Q, K, V, tau2, saved, dO, kmd, causal, window, scale)
    assert entmax_attn_device_status() == 0
    assert dK.shape == K.shape and dV.shape == V.shape and dQ.shape == Q.shape
    rQ, rK, rV = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], km, causal, window, scale)
    for name, g, r in (("dQ", dQ, rQ), ("dK", dK, rK), ("dV", dV, rV)):
        err = np.max(np.abs(to64(g) - r))
        assert err <= GRAD_TOL, (name, err)


def test_gqa_equals_attention_on_repeated_heads():
    """The grouped kernels read K/V through the head map; on explicitly repeated K and V the plain
    kernels do the same arithmetic, so O, tau and dQ agree bit for bit and dK/dV up to the order
    of the group sum."""
    B, H, Hkv, L = 2, 8, 2, 384
    w = Workload(0, "gqa", B, H, L, 64, 1 / 8, True, 0, (100, 384), H_kv=Hkv)
    inp = make_inputs(w, seed=5)
    Q, K, V, dO, km = _dev(inp)
    r = H // Hkv
    Kr = K.repeat_interleave(r, dim=1).contiguous()
    Vr = V.repeat_interleave(r, dim=1).contiguous()
    O, tau, saved = entmax_attn_fwd_train_gqa(Q, K, V, km, True, 0, 1 / 8)
    O1, tau1 = entmax_attn_fwd_gqa(Q, K, V, km, True, 0, 1 / 8)
    Op, taup, savedp = entmax_attn_fwd_train(Q, Kr, Vr, km, True, 0, 1 / 8)
    O2, tau2 = entmax_attn_fwd(Q, Kr, Vr, km, True, 0, 1 / 8)
    for a, b in ((O, Op), (tau, taup), (O1, O2), (tau1, tau2), (O, O1)):
        assert torch.equal(a, b)
    dQ, dK, dV = entmax_attn_bwd_saved_gqa(Q, K, V, tau, saved, dO, km, True, 0, 1 / 8)
    pQ, pK, pV = entmax_attn_bwd_saved(Q, Kr, Vr, taup, savedp, dO, km, True, 0, 1 / 8)
    assert entmax_attn_device_status() == 0
    assert torch.equal(dQ, pQ)
    for g, p in ((dK, pK), (dV, pV)):
        summed = p.view(B, Hkv, r, L, 64).sum(dim=2)
        assert torch.allclose(g, summed, atol=1e-4, rtol=1e-5), (g - summed).abs().max().item()


def test_gqa_decoder_heads_sampled():
    """32 query heads over 8 key/value heads, L = 2048, causal: the layout of a grouped-query
    decoder layer.  Sampled rows for the forward; one key/value group (4 query heads) for the
    backward."""
    B, H, Hkv, L = 2, 32, 8, 2048
    w = Workload(0, "gqa-decoder", B, H, L, 64, 1 / 8, True, 0, H_kv=Hkv)
    inp = make_inputs(w, seed=9)
    d = inputs_f64(inp, False)
    Q, K, V, dO, km = _dev(inp)
    O, tau, saved = entmax_attn_fwd_train_gqa(Q, K, V, None, True, 0, 1 / 8, out_dtype=torch.bfloat16)
    O32, tau32 = entmax_attn_fwd_gqa(Q, K, V, None, True, 0, 1 / 8, out_dtype=torch.float32)
    assert entmax_attn_device_status() == 0
    assert_bf16_is_rounded(O, O32)
    assert torch.equal(tau, tau32)
    rng = np.random.default_rng(9)
    ids = np.unique(np.concatenate([rng.integers(0, B * H * L, size=160), [0, L - 1, B * H * L - 1, 37 * L + 5]]))
    O_ref, tau_ref = orc.attn_fwd_rows_gqa(d["Q"], d["K"], d["V"], ids, None, True, 0, 1 / 8)
    assert np.max(np.abs(to64(O32).reshape(-1, 64)[ids] - O_ref)) <= O_TOL
    Kr = orc.repeat_kv(d["K"], H // Hkv)
    check_rows(d["Q"], Kr, ids, to64(tau).reshape(-1)[ids], tau_ref, None, True, 0, 1 / 8, H, L)
    dQ, dK, dV = entmax_attn_bwd_saved_gqa(Q, K, V, tau, saved, dO, None, True, 0, 1 / 8)
    assert entmax_attn_device_status() == 0
    r = H // Hkv
    b, g = 1, 5  # key/value head 5 of batch 1: query heads 20..23
    heads = [b * H + g * r + k for k in range(r)]
    Vr = orc.repeat_kv(d["V"], r)
    rQ, rK, rV = orc.attn_bwd_heads(d["Q"], Kr, Vr, d["dO"], heads, None, True, 0, 1 / 8)
    assert np.max(np.abs(to64(dQ).reshape(B * H, L, 64)[heads] - rQ)) <= GRAD_TOL
    assert np.max(np.abs(to64(dK)[b, g] - rK.sum(axis=0))) <= GRAD_TOL
    assert np.max(np.abs(to64(dV)[b, g] - rV.sum(axis=0))) <= GRAD_TOL
    for x in (dQ, dK, dV):
        assert torch.isfinite(x).all()


@pytest.mark.parametrize("L", [100, 300])
def test_gqa_unsaved_rows(L):
    """Uniform rows (Q = 0) overflow the saved lists: the exact pass adds their dK/dV terms into the
    shared key/value heads."""
    w = Workload(0, "uniform", 1, 4, L, 64, 1 / 8, H_kv=2)
    inp = make_inputs(w, seed=13)
    inp["Q"].zero_()
    d = inputs_f64(inp, False)
    Q, K, V, dO, km = _dev(inp)
    O, tau, saved = entmax_attn_fwd_train_gqa(Q, K, V, out_dtype=torch.float32)
    grads = entmax_attn_bwd_saved_gqa(Q, K, V, tau, saved, dO)
    assert entmax_attn_device_status() == 0
    O_ref, _ = orc.attn_fwd_gqa(d["Q"], d["K"], d["V"], scale=1 / 8)
    assert np.max(np.abs(to64(O) - O_ref)) <= O_TOL
    refs = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], None, False, 0, 1 / 8)
    for g, r in zip(grads, refs):
        assert np.max(np.abs(to64(g) - r)) <= GRAD_TOL


def test_gqa_autograd_and_errors():
    w = Workload(0, "gqa", 1, 6, 200, 64, 1 / 8, True, 0, H_kv=2)
    inp = make_inputs(w, seed=17)
    d = inputs_f64(inp, False)
    Q, K, V, dO, _ = _dev(inp)
    for x in (Q, K, V):
        x.requires_grad_(True)
    O = EntmaxAttention.apply(Q, K, V, None, True, 0, 1 / 8)
    O.backward(dO)
    assert K.grad.shape == K.shape and V.grad.shape == V.shape
    refs = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], None, True, 0, 1 / 8)
    for g, r in zip((Q.grad, K.grad, V.grad), refs):
        # gradients are returned in the input dtype (bf16): allow its rounding on top
        assert np.all(np.abs(to64(g) - r) <= GRAD_TOL + np.abs(r) * 2.0 ** -8)
    # fp32 inputs with grouped heads are refused by the library, not computed on another path
    q32 = torch.zeros(1, 4, 64, 64, device=DEV)
    k32 = torch.zeros(1, 2, 64, 64, device=DEV)
    with pytest.raises(EntmaxError):
        entmax_attn_fwd_gqa(q32, k32, k32)
