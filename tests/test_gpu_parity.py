"""GPU (sm_100a kernels through the C ABI) vs the fp64 oracle, element by element.

Small shapes span several 128-row tiles and ragged tails and are compared in full; the five
workloads at full size run in the launch configuration bench.py times and are compared on
sampled rows (forward) and sampled heads (backward).  Tolerances: tests/gpu_helpers.py.
"""
import math

import numpy as np
import pytest
import torch

from entmax_tcgen05_tma_b200 import (
    entmax_attn_bwd,
    entmax_attn_bwd_saved,
    entmax_attn_device_status,
    entmax_attn_fwd,
    entmax_attn_fwd_train,
)
import entmax_tcgen05_tma_b200 as E
from entmax_tcgen05_tma_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import oracle as orc
from tests.gpu_helpers import GRAD_TOL, O_TOL, assert_bf16_is_rounded, check_rows, inputs_f64, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _gpu_fwd(inp, w: Workload, out_dtype=torch.float32):
    Q, K, V = (inp[k].to(DEV) for k in ("Q", "K", "V"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(DEV)
    O, tau = entmax_attn_fwd(Q, K, V, km, w.causal, w.window, w.scale, out_dtype=out_dtype)
    assert entmax_attn_device_status() == 0
    return O, tau, (Q, K, V, km)


def _gpu_bwd(dev_inp, tau, dO, w: Workload):
    Q, K, V, km = dev_inp
    dQ, dK, dV = entmax_attn_bwd(Q, K, V, tau, dO.to(DEV), km, w.causal, w.window, w.scale)
    assert entmax_attn_device_status() == 0
    return dQ, dK, dV


def _mask_np(inp):
    return None if inp["key_mask"] is None else inp["key_mask"].numpy()


SMALL = [
    # B, H, L, scale, causal, window, len_range
    (1, 2, 64, 1 / 8, False, 0, None),
    (2, 2, 1, 1 / 8, False, 0, None),
    (2, 3, 17, 1 / 8, False, 0, None),
    (1, 2, 127, 1 / 8, False, 0, None),
    (1, 2, 128, 1 / 8, False, 0, None),
    (2, 1, 129, 1 / 8, False, 0, None),
    (3, 2, 300, 1 / 8, False, 0, (1, 300)),
    (2, 2, 300, 2 / 8, False, 0, None),
    (2, 2, 300, 1 / 8, True, 0, None),
    (2, 2, 300, 1 / 8, True, 32, None),
    (1, 2, 513, 1 / 8, True, 0, (200, 513)),
    (1, 1, 700, 2 / 8, True, 5, None),
]


@pytest.mark.parametrize("B,H,L,scale,causal,window,lens", SMALL)
def test_small_fwd_bwd_full_parity(B, H, L, scale, causal, window, lens):
    w = Workload(0, "small", B, H, L, 64, scale, causal, window, lens)
    inp = make_inputs(w, seed=7 + L + B + window)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    O, tau, dev = _gpu_fwd(inp, w)
    O_ref, tau_ref = orc.attn_fwd(d["Q"], d["K"], d["V"], km, causal, window, scale)
    Og, tg = to64(O), to64(tau)
    finite = np.isfinite(tau_ref)
    assert np.array_equal(np.isfinite(tg), finite)
    assert np.max(np.abs(Og - O_ref)) <= O_TOL
    ids = np.arange(B * H * L)
    check_rows(d["Q"], d["K"], ids, tg.reshape(-1), tau_ref.reshape(-1), km, causal, window, scale, H, L)
    # backward
    dQ, dK, dV = _gpu_bwd(dev, tau, inp["dO"], w)
    rQ, rK, rV = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], km, causal, window, scale)
    for name, g, r in (("dQ", dQ, rQ), ("dK", dK, rK), ("dV", dV, rV)):
        err = np.max(np.abs(to64(g) - r))
        assert err <= GRAD_TOL, (name, err)


def test_fp32_inputs_bf16_output_workload1():
    """Workload 1: fp32 inputs rounded to bf16 at the boundary.  The fp32 output meets the flat
    bound; the bf16 output is that fp32 output rounded to bf16, bit for bit."""
    w = WORKLOADS[1]
    inp = make_inputs(w)
    d = inputs_f64(inp, True)
    O32, tau, _ = _gpu_fwd(inp, w, out_dtype=torch.float32)
    O, tau16, _ = _gpu_fwd(inp, w, out_dtype=torch.bfloat16)
    O_ref, tau_ref = orc.attn_fwd(d["Q"], d["K"], d["V"], None, False, 0, w.scale)
    assert np.max(np.abs(to64(O32) - O_ref)) <= O_TOL
    assert_bf16_is_rounded(O, O32)
    assert torch.equal(tau, tau16)
    assert np.max(np.abs(to64(tau) - tau_ref)) <= 1e-3
    # and the fp32-input backward path
    w2 = w.with_shape()
    Q, K, V = (inp[k].to(DEV) for k in ("Q", "K", "V"))
    dQ, dK, dV = entmax_attn_bwd(Q, K, V, tau, inp["dO"].to(DEV), None, False, 0, w.scale)
    assert entmax_attn_device_status() == 0
    rQ, rK, rV = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], None, False, 0, w2.scale)
    for g, r in ((dQ, rQ), (dK, rK), (dV, rV)):
        assert np.max(np.abs(to64(g) - r)) <= GRAD_TOL


def _sample_rows(w: Workload, inp, rng, n=192):
    L, BH = w.L, w.B * w.H
    ids = set(rng.integers(0, BH * L, size=n).tolist())
    for bh in (0, BH - 1):
        for i in (0, 1, L // 2, L - 1):
            ids.add(bh * L + i)
    if inp["lengths"] is not None:
        b = int(torch.argmin(inp["lengths"]))
        for i in (0, L - 1):
            ids.add((b * w.H) * L + i)
    return np.array(sorted(ids), dtype=np.int64)


def _grad_heads(w: Workload):
    """Heads whose gradients are compared in full at the large sizes: the first and the last, plus
    two more at workload 4 (one head there is 4096 x 4096 oracle pairs)."""
    BH = w.B * w.H
    return [0, BH // 3, (2 * BH) // 3, BH - 1] if w.L >= 4096 else [0, BH - 1]


def _check_fwd_rows(w: Workload, inp, d, O32, tau, rng):
    """Sampled rows of a full-size forward against the oracle: the flat O bound on the fp32 output,
    tau, the simplex and the support band."""
    km = _mask_np(inp)
    ids = _sample_rows(w, inp, rng)
    O_ref, tau_ref = orc.attn_fwd_rows(d["Q"], d["K"], d["V"], ids, km, w.causal, w.window, w.scale)
    Og = to64(O32).reshape(-1, w.D)[ids]
    err = np.max(np.abs(Og - O_ref))
    assert err <= O_TOL, err
    check_rows(d["Q"], d["K"], ids, to64(tau).reshape(-1)[ids], tau_ref, km, w.causal, w.window, w.scale, w.H, w.L)
    # every row: finite tau (no row is empty in these workloads), O finite
    assert torch.isfinite(tau).all() and torch.isfinite(O32).all()


@pytest.mark.parametrize("wid", [2, 3, 4, 5])
def test_full_size_workloads(wid):
    """Full-size workloads in the bench launch configuration.  The fp32 output meets the flat O
    bound on sampled rows; the bf16 output (as timed) is the fp32 output rounded, bit for bit."""
    w = WORKLOADS[wid]
    inp = make_inputs(w)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    O32, tau, dev = _gpu_fwd(inp, w, out_dtype=torch.float32)
    O, tau16, _ = _gpu_fwd(inp, w, out_dtype=torch.bfloat16)
    assert_bf16_is_rounded(O, O32)
    assert torch.equal(tau, tau16)
    _check_fwd_rows(w, inp, d, O32, tau, np.random.default_rng(wid))
    if not w.backward:
        return
    dQ, dK, dV = _gpu_bwd(dev, tau, inp["dO"], w)
    heads = _grad_heads(w)
    rQ, rK, rV = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], heads, km, w.causal, w.window, w.scale)
    for name, g, r in (("dQ", dQ, rQ), ("dK", dK, rK), ("dV", dV, rV)):
        gh = to64(g).reshape(w.B * w.H, w.L, w.D)[heads]
        err = np.max(np.abs(gh - r))
        assert err <= GRAD_TOL, (name, err)
    for g in (dQ, dK, dV):
        assert torch.isfinite(g).all()


def test_empty_rows_and_masked_batches():
    """A batch whose keys are all padding: O = 0, tau = +inf, zero gradients."""
    w = Workload(0, "empty", 2, 2, 200, 64, 1 / 8, len_range=(50, 50))
    inp = make_inputs(w, seed=3)
    inp["key_mask"][1] = 0
    O, tau, dev = _gpu_fwd(inp, w)
    assert torch.all(O[1] == 0) and torch.all(torch.isinf(tau[1]))
    dQ, dK, dV = _gpu_bwd(dev, tau, inp["dO"], w)
    assert torch.all(dQ[1] == 0) and torch.all(dK[1] == 0) and torch.all(dV[1] == 0)
    d = inputs_f64(inp, False)
    rQ, rK, rV = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], inp["key_mask"].numpy(), False, 0, w.scale)
    assert np.max(np.abs(to64(dK) - rK)) <= GRAD_TOL


@pytest.mark.parametrize("L", [100, 300, 1000])
def test_uniform_rows_take_the_exact_redo_path(L):
    """Q = 0 makes every allowed score equal: the support is the whole row, larger than the
    candidate capacity once L > 128, so the rows are redone exactly on CUDA cores.  O is the
    plain mean of V and tau = -2/sqrt(n)."""
    w = Workload(0, "uniform", 1, 2, L, 64, 1 / 8)
    inp = make_inputs(w, seed=11)
    inp["Q"].zero_()
    O, tau, dev = _gpu_fwd(inp, w)
    V = to64(inp["V"])
    np.testing.assert_allclose(to64(O), np.broadcast_to(V.mean(axis=2, keepdims=True), V.shape), atol=1e-4)
    np.testing.assert_allclose(to64(tau), -2 / math.sqrt(L), atol=1e-6)
    dQ, dK, dV = _gpu_bwd(dev, tau, inp["dO"], w)
    d = inputs_f64(inp, False)
    rQ, rK, rV = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], None, False, 0, w.scale)
    for g, r in ((dQ, rQ), (dK, rK), (dV, rV)):
        assert np.max(np.abs(to64(g) - r)) <= GRAD_TOL


@pytest.mark.parametrize("causal", [False, True])
def test_rows_past_the_candidate_lists(causal):
    """Rows whose candidates do not fit the tensor-core forward's lists (32 per half row): a zero query
    row ties every allowed key, so all of them are candidates.  Tile 0 of head 0 has two such rows
    and tile 1 of head 0 one: their extra candidates fit the CTA's spill area, and a warp solves each
    row from its lists and its spill entries.  Tile 0 of head 1 has eight: without the causal mask
    (256 candidates a row) they overflow the spill area and tau comes from the rows' scores
    recomputed on CUDA cores; with it (about 100 a row) they fit.  Everything is compared with the
    oracle."""
    w = Workload(0, "spill", 1, 2, 256, 64, 1 / 8, causal=causal)
    inp = make_inputs(w, seed=13)
    Q = inp["Q"]
    for h, rows in ((0, (90, 117, 200)), (1, range(100, 108))):
        for r in rows:
            Q[0, h, r].zero_()
    d = inputs_f64(inp, False)
    O, tau, dev = _gpu_fwd(inp, w)
    O_ref, tau_ref = orc.attn_fwd(d["Q"], d["K"], d["V"], None, causal, 0, w.scale)
    assert np.max(np.abs(to64(O) - O_ref)) <= O_TOL
    check_rows(d["Q"], d["K"], np.arange(2 * 256), to64(tau).reshape(-1), tau_ref.reshape(-1), None, causal, 0,
               w.scale, 2, 256)
    dQ, dK, dV = _gpu_bwd(dev, tau, inp["dO"], w)
    refs = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], None, causal, 0, w.scale)
    for g, r in zip((dQ, dK, dV), refs):
        assert np.max(np.abs(to64(g) - r)) <= GRAD_TOL


@pytest.mark.parametrize("causal", [False, True])
def test_recompute_backward_both_workspaces(causal):
    """Long rows through entmax_attn_bwd: with the full workspace the supports are rebuilt by the
    training forward and the support-list backward runs; with the minimum one float per row the
    recompute kernels run.  Both against the oracle, and against each other."""
    w = Workload(0, "recompute", 2, 2, 900, 64, 1 / 8, causal=causal, len_range=(500, 900))
    inp = make_inputs(w, seed=29)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    O, tau, dev = _gpu_fwd(inp, w)
    Q, K, V, kmd = dev
    dO = inp["dO"].to(DEV)
    full = entmax_attn_bwd(Q, K, V, tau, dO, kmd, causal, 0, w.scale)
    ws = torch.empty(E.bwd_min_workspace_size(w.B, w.H, w.L), dtype=torch.uint8, device=DEV)
    small = entmax_attn_bwd(Q, K, V, tau, dO, kmd, causal, 0, w.scale, workspace=ws)
    assert entmax_attn_device_status() == 0
    refs = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], km, causal, 0, w.scale)
    for name, a, b, r in zip(("dQ", "dK", "dV"), full, small, refs):
        assert np.max(np.abs(to64(a) - r)) <= GRAD_TOL, name
        assert np.max(np.abs(to64(b) - r)) <= GRAD_TOL, name
        assert torch.allclose(a, b, atol=1e-4, rtol=0), (name, float((a - b).abs().max()))


EXTRACT_CASES = [
    # B, H, L, scale, causal, window, len_range: streamed tiles with padding; causal; a causal
    # window of 200 keys (tiles of at most three key blocks, scored once); near-uniform rows whose
    # supports overflow the lists (every row takes the unsaved-row kernel)
    (2, 2, 1100, 1 / 8, False, 0, (600, 1100)),
    (1, 3, 900, 2 / 8, True, 0, None),
    (2, 2, 1000, 1 / 8, True, 200, None),
    (1, 2, 700, 1e-3, False, 0, None),
]


@pytest.mark.parametrize("B,H,L,scale,causal,window,lens", EXTRACT_CASES)
def test_support_extraction_backward(B, H, L, scale, causal, window, lens):
    """entmax_attn_bwd with its full workspace lists each row's support from the caller's tau (one
    score pass cut at tau_i) and runs the support-list backward.  Against the oracle, and against
    the training path (entmax_attn_fwd_train + entmax_attn_bwd_saved), whose lists hold the same
    supports: the two differ only by the rounding of sqrt(p_ij) (one fused step from tau against
    the forward's two from the row max) and by the atomic order of the dK, dV sums."""
    w = Workload(0, "extract", B, H, L, 64, scale, causal, window, lens)
    inp = make_inputs(w, seed=41 + L + window)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    O, tau, dev = _gpu_fwd(inp, w)
    got = _gpu_bwd(dev, tau, inp["dO"], w)
    _, tau_t, saved = _gpu_train(inp, w)
    assert torch.equal(tau, tau_t)
    refs = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], km, causal, window, w.scale)
    for name, a, b, r in zip(("dQ", "dK", "dV"), got, saved, refs):
        assert np.max(np.abs(to64(a) - r)) <= GRAD_TOL, name
        bound = 1e-5 * max(1.0, float(b.abs().max()))
        assert float((a - b).abs().max()) <= bound, (name, float((a - b).abs().max()))


def test_one_hot_rows():
    """A key aligned with every query and far above the rest takes all the weight."""
    w = Workload(0, "onehot", 1, 1, 256, 64, 1.0)
    inp = make_inputs(w, seed=5)
    inp["Q"] = torch.zeros_like(inp["Q"])
    inp["K"] = torch.zeros_like(inp["K"])
    inp["Q"][..., 0] = 1.0
    inp["K"][0, 0, 77, 0] = 8.0
    O, tau, _ = _gpu_fwd(inp, w)
    V = to64(inp["V"])
    np.testing.assert_allclose(to64(O)[0, 0], np.broadcast_to(V[0, 0, 77], (256, 64)), atol=1e-6)
    np.testing.assert_allclose(to64(tau), 6.0, atol=1e-6)


def test_repeat_calls_are_deterministic():
    """Every output of both backward paths is the same bit for bit from run to run where they run on
    the tensor-core kernels (here L = 512 and a causal window of 32; no atomics, fixed sum order); the
    recompute backward is deterministic everywhere."""
    for w in (WORKLOADS[3].with_shape(B=2), WORKLOADS[5].with_shape(B=2)):
        inp = make_inputs(w)
        O1, t1, dev = _gpu_fwd(inp, w)
        O2, t2, _ = _gpu_fwd(inp, w)
        assert torch.equal(O1, O2) and torch.equal(t1, t2)
        g1 = _gpu_bwd(dev, t1, inp["dO"], w)
        g2 = _gpu_bwd(dev, t1, inp["dO"], w)
        for a, b in zip(g1, g2):
            assert torch.equal(a, b)
        _, _, s1 = _gpu_train(inp, w)
        _, _, s2 = _gpu_train(inp, w)
        for a, b in zip(s1, s2):
            assert torch.equal(a, b)


def test_saved_backward_repeatability_on_support_lists():
    """Beyond the tensor-core configurations (here L = 2048) the saved backward buckets support
    entries by key with atomic slot counters, so dK and dV are summed in a scheduling-dependent
    order: run to run they agree to fp32 rounding of those sums (bound stated here), dQ, O and tau
    exactly."""
    w = Workload(0, "long", 1, 4, 2048, 64, 2 / 8)
    inp = make_inputs(w, seed=81)
    O1, t1, g1 = _gpu_train(inp, w)
    O2, t2, g2 = _gpu_train(inp, w)
    assert torch.equal(O1, O2) and torch.equal(t1, t2) and torch.equal(g1[0], g2[0])
    for a, b in zip(g1[1:], g2[1:]):
        assert torch.allclose(a, b, atol=1e-5, rtol=1e-5), float((a - b).abs().max())


# ----------------------------------------------------------------------------------- training path
def _gpu_train(inp, w: Workload, out_dtype=torch.float32):
    Q, K, V, dO = (inp[k].to(DEV) for k in ("Q", "K", "V", "dO"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(DEV)
    O, tau, saved = entmax_attn_fwd_train(Q, K, V, km, w.causal, w.window, w.scale, out_dtype=out_dtype)
    dQ, dK, dV = entmax_attn_bwd_saved(Q, K, V, tau, saved, dO, km, w.causal, w.window, w.scale)
    assert entmax_attn_device_status() == 0
    return O, tau, (dQ, dK, dV)


@pytest.mark.parametrize("B,H,L,scale,causal,window,lens", SMALL)
def test_training_path_small_full_parity(B, H, L, scale, causal, window, lens):
    """entmax_attn_fwd_train + entmax_attn_bwd_saved against the oracle, every element."""
    w = Workload(0, "small", B, H, L, 64, scale, causal, window, lens)
    inp = make_inputs(w, seed=7 + L + B + window)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    O, tau, grads = _gpu_train(inp, w)
    O_ref, tau_ref = orc.attn_fwd(d["Q"], d["K"], d["V"], km, causal, window, scale)
    assert np.max(np.abs(to64(O) - O_ref)) <= O_TOL
    # the training forward computes exactly what the plain forward computes
    O2, tau2, _ = _gpu_fwd(inp, w)
    assert torch.equal(O, O2) and torch.equal(tau, tau2)
    rQ, rK, rV = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], km, causal, window, scale)
    for name, g, r in (("dQ", grads[0], rQ), ("dK", grads[1], rK), ("dV", grads[2], rV)):
        err = np.max(np.abs(to64(g) - r))
        assert err <= GRAD_TOL, (name, err)


@pytest.mark.parametrize("wid", [3, 4, 5])
def test_training_path_full_size_workloads(wid):
    """The step bench.py times (training forward with bf16 O, then the saved backward) at full size:
    its forward against the oracle on sampled rows (the bf16 O it times is the fp32 O rounded, bit
    for bit; the fp32 O meets the flat bound), its gradients on whole heads."""
    w = WORKLOADS[wid]
    inp = make_inputs(w)
    d = inputs_f64(inp, False)
    km = _mask_np(inp)
    O, tau, grads = _gpu_train(inp, w, out_dtype=torch.bfloat16)
    O32, tau32, _ = _gpu_train(inp, w, out_dtype=torch.float32)
    assert_bf16_is_rounded(O, O32)
    assert torch.equal(tau, tau32)
    _check_fwd_rows(w, inp, d, O32, tau, np.random.default_rng(100 + wid))
    heads = _grad_heads(w)
    rQ, rK, rV = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], heads, km, w.causal, w.window, w.scale)
    for name, g, r in (("dQ", grads[0], rQ), ("dK", grads[1], rK), ("dV", grads[2], rV)):
        gh = to64(g).reshape(w.B * w.H, w.L, w.D)[heads]
        err = np.max(np.abs(gh - r))
        assert err <= GRAD_TOL, (name, err)
    for g in grads:
        assert torch.isfinite(g).all()


@pytest.mark.parametrize("L", [100, 300])
def test_training_path_unsaved_rows(L):
    """Uniform rows (Q = 0) have supports larger than the saved lists once L > 64: the backward's
    exact pass recomputes them and adds their dK/dV terms."""
    w = Workload(0, "uniform", 1, 2, L, 64, 1 / 8)
    inp = make_inputs(w, seed=11)
    inp["Q"].zero_()
    O, tau, grads = _gpu_train(inp, w)
    d = inputs_f64(inp, False)
    rQ, rK, rV = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], None, False, 0, w.scale)
    for g, r in zip(grads, (rQ, rK, rV)):
        assert np.max(np.abs(to64(g) - r)) <= GRAD_TOL


def test_training_path_empty_batch():
    w = Workload(0, "empty", 2, 2, 200, 64, 1 / 8, len_range=(50, 50))
    inp = make_inputs(w, seed=3)
    inp["key_mask"][1] = 0
    O, tau, grads = _gpu_train(inp, w)
    assert torch.all(O[1] == 0) and torch.all(torch.isinf(tau[1]))
    for g in grads:
        assert torch.all(g[1] == 0)


# ----------------------------------------------------------------------------------- size limits
@pytest.mark.parametrize("causal,window,scale", [(False, 0, 2 / 8), (True, 32, 1 / 8)])
def test_maximum_sequence_length(causal, window, scale):
    """L = 16384, the longest sequence the library takes (128 streamed key blocks per query tile):
    forward on sampled rows, both backward paths on the whole head."""
    w = Workload(0, "max-L", 1, 1, 16384, 64, scale, causal=causal, window=window)
    inp = make_inputs(w, seed=21)
    d = inputs_f64(inp, False)
    O, tau, dev = _gpu_fwd(inp, w, out_dtype=torch.float32)
    rng = np.random.default_rng(21)
    ids = np.unique(np.concatenate([rng.integers(0, w.L, size=96), [0, 1, 127, 128, w.L // 2, w.L - 1]]))
    O_ref, tau_ref = orc.attn_fwd_rows(d["Q"], d["K"], d["V"], ids, None, causal, window, scale)
    assert np.max(np.abs(to64(O).reshape(-1, w.D)[ids] - O_ref)) <= O_TOL
    check_rows(d["Q"], d["K"], ids, to64(tau).reshape(-1)[ids], tau_ref, None, causal, window, scale, w.H, w.L)
    rQ, rK, rV = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], [0], None, causal, window, scale)
    grads = [_gpu_bwd(dev, tau, inp["dO"], w)]
    _, _, g_saved = _gpu_train(inp, w)
    grads.append(g_saved)
    for g in grads:
        for name, x, r in zip(("dQ", "dK", "dV"), g, (rQ, rK, rV)):
            err = np.max(np.abs(to64(x).reshape(1, w.L, w.D) - r))
            assert err <= GRAD_TOL, (name, err)


def test_maximum_head_count():
    """B * H = 65535 heads (the grid's limit), two rows each, with key padding down to one key."""
    w = Workload(0, "max-heads", 65535, 1, 2, 64, 1 / 8, len_range=(1, 2))
    inp = make_inputs(w, seed=22)
    d = inputs_f64(inp, False)
    km = inp["key_mask"].numpy()
    O, tau, dev = _gpu_fwd(inp, w, out_dtype=torch.float32)
    ids = np.array(sorted({0, 1, 2, 3, 65533 * 2, 65534 * 2, 65534 * 2 + 1} | set(range(40000, 40040))), dtype=np.int64)
    O_ref, tau_ref = orc.attn_fwd_rows(d["Q"], d["K"], d["V"], ids, km, False, 0, w.scale)
    assert np.max(np.abs(to64(O).reshape(-1, w.D)[ids] - O_ref)) <= O_TOL
    check_rows(d["Q"], d["K"], ids, to64(tau).reshape(-1)[ids], tau_ref, km, False, 0, w.scale, w.H, w.L)
    heads = [0, 1, 20000, 65534]
    rQ, rK, rV = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], heads, km, False, 0, w.scale)
    for g in (_gpu_bwd(dev, tau, inp["dO"], w), _gpu_train(inp, w)[2]):
        for name, x, r in zip(("dQ", "dK", "dV"), g, (rQ, rK, rV)):
            err = np.max(np.abs(to64(x).reshape(-1, w.L, w.D)[heads] - r))
            assert err <= GRAD_TOL, (name, err)
