"""alpha-entmax attention on the GPU (entmax_attn_fwd_ex / entmax_attn_bwd_saved_ex) vs the fp64
oracle, for alpha other than 1.5: p = max(0, (alpha-1)(S - tau))^(1/(alpha-1)).

Small shapes compared in full (several 128-row tiles, ragged tails, padding, causal window,
grouped heads); the generic kernels next to alpha = 1.5 against the specialised ones; rows whose
supports overflow the candidate lists (exact CUDA-core path) and the saved lists (exact backward
pass); a long-context shape on sampled rows.  Tolerances: tests/gpu_helpers.py.
"""
import numpy as np
import pytest
import torch

from entmax_tcgen05_tma_b200 import (
    EntmaxAttention,
    entmax_attn_bwd_saved,
    entmax_attn_bwd_saved_ex,
    entmax_attn_device_status,
    entmax_attn_fwd_ex,
    entmax_attn_fwd_train,
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


CASES = [
    # alpha, B, H, H_kv, L, scale, causal, window, len_range
    (2.0, 1, 2, 2, 64, 1 / 8, False, 0, None),
    (2.0, 2, 2, 2, 300, 1 / 8, False, 0, (1, 300)),
    (1.75, 2, 3, 3, 129, 1 / 8, False, 0, None),
    (1.75, 1, 4, 2, 513, 1 / 8, True, 0, (200, 513)),
    (1.25, 2, 2, 2, 300, 2 / 8, True, 32, None),
    (1.25, 1, 2, 1, 700, 2 / 8, False, 0, None),
    (1.6, 2, 2, 2, 17, 1 / 8, False, 0, None),
]


def _run(inp, alpha, causal, window, scale, out_dtype=torch.float32):
    Q, K, V, dO, km = _dev(inp)
    O, tau, saved = entmax_attn_fwd_ex(Q, K, V, km, causal, window, scale, alpha=alpha, save=True,
                                       out_dtype=out_dtype)
    O2, tau2 = entmax_attn_fwd_ex(Q, K, V, km, causal, window, scale, alpha=alpha, out_dtype=out_dtype)
    assert torch.equal(O, O2) and torch.equal(tau, tau2)
    grads = entmax_attn_bwd_saved_ex(Q, K, V, tau, saved, dO, km, causal, window, scale, alpha=alpha)
    assert entmax_attn_device_status() == 0
    return O, tau, grads


@pytest.mark.parametrize("alpha,B,H,Hkv,L,scale,causal,window,lens", CASES)
def test_alpha_small_full_parity(alpha, B, H, Hkv, L, scale, causal, window, lens):
    w = Workload(0, "alpha", B, H, L, 64, scale, causal, window, lens, H_kv=Hkv)
    inp = make_inputs(w, seed=41 + L + H)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    O, tau, grads = _run(inp, alpha, causal, window, scale)
    O_ref, tau_ref = orc.attn_fwd_gqa(d["Q"], d["K"], d["V"], km, causal, window, scale, alpha=alpha)
    Og, tg = to64(O), to64(tau)
    assert np.array_equal(np.isfinite(tg), np.isfinite(tau_ref))
    assert np.max(np.abs(Og - O_ref)) <= O_TOL
    Kr = orc.repeat_kv(d["K"], H // Hkv)
    check_rows(d["Q"], Kr, np.arange(B * H * L), tg.reshape(-1), tau_ref.reshape(-1), km, causal, window, scale, H,
               L, alpha=alpha)
    refs = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], km, causal, window, scale, alpha=alpha)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, refs):
        err = np.max(np.abs(to64(g) - r))
        assert err <= GRAD_TOL, (name, err)


def test_generic_kernels_next_to_one_point_five():
    """alpha = 1.5 + 2^-20 runs the generic kernels (powers, Newton finish); alpha = 1.5 the
    specialised ones (squares, closed-form finish).  The two agree far inside the tolerances."""
    w = Workload(0, "alpha", 2, 3, 600, 64, 1 / 8, True, 0, (300, 600))
    inp = make_inputs(w, seed=43)
    Q, K, V, dO, km = _dev(inp)
    O, tau, saved = entmax_attn_fwd_train(Q, K, V, km, True, 0, 1 / 8, out_dtype=torch.float32)
    gs = entmax_attn_bwd_saved(Q, K, V, tau, saved, dO, km, True, 0, 1 / 8)
    a = 1.5 + 2.0 ** -20
    Og, tg, gg = _run(inp, a, True, 0, 1 / 8)
    assert torch.max(torch.abs(Og - O)).item() < 1e-4
    assert torch.max(torch.abs(tg - tau)).item() < 1e-4
    for x, y in zip(gg, gs):
        assert torch.max(torch.abs(x - y)).item() < 1e-3


@pytest.mark.parametrize("alpha,L", [(1.1, 300), (1.25, 1000)])
def test_large_supports_take_the_exact_paths(alpha, L):
    """Small alpha - 1 spreads each row over many keys: rows overflow the forward's candidate lists
    (redone on CUDA cores) and the saved lists (the backward's exact pass)."""
    w = Workload(0, "alpha-dense", 1, 2, L, 64, 1 / 8)
    inp = make_inputs(w, seed=44)
    d = inputs_f64(inp, False)
    O, tau, grads = _run(inp, alpha, False, 0, 1 / 8)
    O_ref, tau_ref = orc.attn_fwd(d["Q"], d["K"], d["V"], None, False, 0, 1 / 8, alpha=alpha)
    assert np.max(np.abs(to64(O) - O_ref)) <= O_TOL
    check_rows(d["Q"], d["K"], np.arange(2 * L), to64(tau).reshape(-1), tau_ref.reshape(-1), None, False, 0, 1 / 8,
               2, L, alpha=alpha)
    refs = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], None, False, 0, 1 / 8, alpha=alpha)
    for g, r in zip(grads, refs):
        assert np.max(np.abs(to64(g) - r)) <= GRAD_TOL


def test_sparsemax_long_context_sampled():
    """alpha = 2 (sparsemax) at L = 4096 with temperature 2 (streamed key blocks): sampled rows for
    the forward, one whole head for the backward."""
    w = Workload(0, "sparsemax-long", 2, 4, 4096, 64, 2 / 8)
    inp = make_inputs(w, seed=45)
    d = inputs_f64(inp, False)
    O, tau, grads = _run(inp, 2.0, False, 0, 2 / 8, out_dtype=torch.bfloat16)
    O32, tau32, _ = _run(inp, 2.0, False, 0, 2 / 8, out_dtype=torch.float32)
    assert_bf16_is_rounded(O, O32)
    assert torch.equal(tau, tau32)
    rng = np.random.default_rng(45)
    ids = np.unique(np.concatenate([rng.integers(0, 8 * 4096, size=128), [0, 4095, 8 * 4096 - 1]]))
    O_ref, tau_ref = orc.attn_fwd_rows(d["Q"], d["K"], d["V"], ids, None, False, 0, 2 / 8, alpha=2.0)
    assert np.max(np.abs(to64(O32).reshape(-1, 64)[ids] - O_ref)) <= O_TOL
    check_rows(d["Q"], d["K"], ids, to64(tau).reshape(-1)[ids], tau_ref, None, False, 0, 2 / 8, 4, 4096, alpha=2.0)
    rQ, rK, rV = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], [6], None, False, 0, 2 / 8, alpha=2.0)
    for g, r in zip(grads, (rQ, rK, rV)):
        assert np.max(np.abs(to64(g).reshape(8, 4096, 64)[6] - r[0])) <= GRAD_TOL


def test_alpha_autograd():
    w = Workload(0, "alpha", 1, 4, 200, 64, 1 / 8, True, 0, H_kv=2)
    inp = make_inputs(w, seed=46)
    d = inputs_f64(inp, False)
    Q, K, V, dO, _ = _dev(inp)
    for x in (Q, K, V):
        x.requires_grad_(True)
    O = EntmaxAttention.apply(Q, K, V, None, True, 0, 1 / 8, 1.75)
    O.backward(dO)
    O_ref, _ = orc.attn_fwd_gqa(d["Q"], d["K"], d["V"], None, True, 0, 1 / 8, alpha=1.75)
    # the autograd wrapper returns O and the gradients in the inputs' dtype (bf16): each value is the
    # kernels' fp32 result (checked at the flat bounds by the tests above) rounded once to bf16, so
    # the bound here adds half a bf16 ulp of the value
    assert np.all(np.abs(to64(O) - O_ref) <= O_TOL + np.abs(O_ref) * 2.0 ** -9)
    refs = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], None, True, 0, 1 / 8, alpha=1.75)
    for g, r in zip((Q.grad, K.grad, V.grad), refs):
        assert np.all(np.abs(to64(g) - r) <= GRAD_TOL + np.abs(r) * 2.0 ** -8)
