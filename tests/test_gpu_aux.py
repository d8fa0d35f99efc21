"""The forward's auxiliary rows (entmax_attn_fwd_aux) and the backward that takes them
(entmax_attn_bwd_aux) against the fp64 oracle.

Otil_i = sum_j sqrt(p_ij) V_j and r_i = sum_j sqrt(p_ij) give the backward's row scalar
u_i = dO_i . Otil_i / r_i (page "svd-sst2-roberta-adasplash", section 2.4).  The forward's O and tau
must be those of entmax_attn_fwd (bit for bit where both run the gather forward, to 1e-4 where
entmax_attn_fwd runs the tensor-core one); Otil and r are compared with the oracle's attn_aux_rows,
the gradients with its attn_bwd.  Shapes cover the tensor-core configurations (L <= 512, causal
windows) and the others, ragged tails, padding down to one key and a fully padded batch.
"""
import numpy as np
import pytest
import torch

import entmax_tcgen05_tma_b200 as E
from entmax_tcgen05_tma_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import oracle as orc
from tests.gpu_helpers import GRAD_TOL, O_TOL, inputs_f64, to64

pytestmark = pytest.mark.gpu

R_TOL = 1e-3  # r_i = sum sqrt(p_ij): its error is that of tau, times the support size


def _dev(inp):
    Q, K, V, dO = (inp[k].cuda() for k in ("Q", "K", "V", "dO"))
    km = None if inp["key_mask"] is None else inp["key_mask"].cuda()
    return Q, K, V, dO, km


CASES = [
    # B, H, L, scale, causal, window, len_range
    (1, 2, 64, 1 / 8, False, 0, None),
    (2, 2, 129, 1 / 8, False, 0, None),
    (3, 2, 300, 1 / 8, False, 0, (1, 300)),
    (2, 2, 300, 2 / 8, True, 32, None),
    (1, 2, 513, 1 / 8, True, 0, (200, 513)),
    (1, 1, 700, 2 / 8, True, 5, None),
    (1, 2, 1000, 2 / 8, False, 0, None),
]


@pytest.mark.parametrize("B,H,L,scale,causal,window,lens", CASES)
def test_aux_rows_and_backward(B, H, L, scale, causal, window, lens):
    w = Workload(0, "aux", B, H, L, 64, scale, causal, window, lens)
    inp = make_inputs(w, seed=61 + L + B)
    d = inputs_f64(inp, False)
    km = None if inp["key_mask"] is None else inp["key_mask"].numpy()
    Q, K, V, dO, kmd = _dev(inp)
    O, tau, Ot, rs = E.entmax_attn_fwd_aux(Q, K, V, kmd, causal, window, scale, out_dtype=torch.float32)
    O2, tau2 = E.entmax_attn_fwd(Q, K, V, kmd, causal, window, scale, out_dtype=torch.float32)
    assert E.entmax_attn_device_status() == 0
    if L <= 512 or (causal and 0 < window <= 128):
        # entmax_attn_fwd runs the tensor-core forward here, the auxiliary rows the gather forward:
        # the same O and tau up to the order of their sums
        assert torch.allclose(O, O2, atol=1e-4, rtol=0) and torch.allclose(tau, tau2, atol=1e-4, rtol=0)
    else:
        assert torch.equal(O, O2) and torch.equal(tau, tau2)
    O_ref, tau_ref = orc.attn_fwd(d["Q"], d["K"], d["V"], km, causal, window, scale)
    assert np.max(np.abs(to64(O) - O_ref)) <= O_TOL
    ids = np.arange(B * H * L)
    Ot_ref, r_ref = orc.attn_aux_rows(d["Q"], d["K"], d["V"], ids, km, causal, window, scale)
    assert np.max(np.abs(to64(Ot).reshape(-1, 64) - Ot_ref)) <= O_TOL
    assert np.max(np.abs(to64(rs).reshape(-1) - r_ref)) <= R_TOL
    grads = E.entmax_attn_bwd_aux(Q, K, V, tau, Ot, rs, dO, kmd, causal, window, scale)
    assert E.entmax_attn_device_status() == 0
    refs = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], km, causal, window, scale)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, refs):
        err = np.max(np.abs(to64(g) - r))
        assert err <= GRAD_TOL, (name, err)
    # the same gradients as the backward that derives u_i itself, up to the order of the sums
    plain = E.entmax_attn_bwd(Q, K, V, tau, dO, kmd, causal, window, scale)
    for g, p in zip(grads, plain):
        assert torch.allclose(g, p, atol=1e-3, rtol=0), float((g - p).abs().max())


def test_aux_fully_padded_batch():
    w = Workload(0, "aux-empty", 2, 2, 200, 64, 1 / 8, len_range=(50, 50))
    inp = make_inputs(w, seed=67)
    inp["key_mask"][1] = 0
    Q, K, V, dO, kmd = _dev(inp)
    O, tau, Ot, rs = E.entmax_attn_fwd_aux(Q, K, V, kmd, False, 0, w.scale)
    assert torch.all(Ot[1] == 0) and torch.all(rs[1] == 0) and torch.all(torch.isinf(tau[1]))
    dQ, dK, dV = E.entmax_attn_bwd_aux(Q, K, V, tau, Ot, rs, dO, kmd, False, 0, w.scale)
    assert E.entmax_attn_device_status() == 0
    for g in (dQ, dK, dV):
        assert torch.all(g[1] == 0) and torch.isfinite(g).all()


@pytest.mark.parametrize("wid", [3, 5])
def test_aux_full_size_workloads(wid):
    """Full-size workloads: the auxiliary rows on sampled rows, gradients on the first and last heads."""
    w = WORKLOADS[wid]
    inp = make_inputs(w)
    d = inputs_f64(inp, False)
    km = None if inp["key_mask"] is None else inp["key_mask"].numpy()
    Q, K, V, dO, kmd = _dev(inp)
    O, tau, Ot, rs = E.entmax_attn_fwd_aux(Q, K, V, kmd, w.causal, w.window, w.scale)
    rng = np.random.default_rng(wid)
    BH = w.B * w.H
    ids = np.unique(np.concatenate([rng.integers(0, BH * w.L, size=160), [0, w.L - 1, BH * w.L - 1]]))
    Ot_ref, r_ref = orc.attn_aux_rows(d["Q"], d["K"], d["V"], ids, km, w.causal, w.window, w.scale)
    assert np.max(np.abs(to64(Ot).reshape(-1, 64)[ids] - Ot_ref)) <= O_TOL
    assert np.max(np.abs(to64(rs).reshape(-1)[ids] - r_ref)) <= R_TOL
    grads = E.entmax_attn_bwd_aux(Q, K, V, tau, Ot, rs, dO, kmd, w.causal, w.window, w.scale)
    assert E.entmax_attn_device_status() == 0
    heads = [0, BH - 1]
    refs = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], heads, km, w.causal, w.window, w.scale)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, refs):
        err = np.max(np.abs(to64(g).reshape(BH, w.L, 64)[heads] - r))
        assert err <= GRAD_TOL, (name, err)
