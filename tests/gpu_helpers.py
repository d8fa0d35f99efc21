"""Shared helpers for the GPU-vs-oracle parity tests.

Tolerances (fixed by the specification of the hot path):
  * O:      max |O_gpu - O_ref| <= 1e-2, flat, on the fp32 output.  The bf16 output the bench
            times must equal that fp32 output rounded to bf16 (round to nearest even) bit for bit,
            so it carries no error beyond the output format's own rounding.
  * tau:    |tau_gpu - tau_ref| <= 1e-3
  * simplex: |sum_j A_ij - 1| <= 1e-3 with A recomputed in fp64 from the GPU's tau
  * support: (S_ij > tau_gpu) differs from (S_ij > tau_ref) only where |S_ij - tau_ref| < 1e-3
  * grads:  max |dX_gpu - dX_ref| <= 2e-2 for dQ, dK, dV
"""
from __future__ import annotations

import numpy as np
import torch

O_TOL = 1e-2
TAU_TOL = 1e-3
SUM_TOL = 1e-3
SUPPORT_BAND = 1e-3
GRAD_TOL = 2e-2


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def inputs_f64(inp: dict, fp32_inputs: bool):
    """Oracle view of the inputs: the bf16 values both sides compute with, widened to fp64."""
    from oracle import oracle as orc
    out = {}
    for k in ("Q", "K", "V", "dO"):
        t = inp[k]
        out[k] = orc.round_bf16(t.numpy()) if fp32_inputs else to64(t)
    return out


def allowed_matrix(L, causal, window, mask_row):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    a = np.ones((L, L), bool)
    if causal:
        a &= j <= i
    if window:
        a &= j >= i - window + 1
    if mask_row is not None:
        a &= np.asarray(mask_row, bool)[None, :]
    return a


def check_rows(Qd, Kd, row_ids, tau_gpu_rows, tau_ref_rows, key_mask, causal, window, scale, H, L, alpha=1.5):
    """Simplex and support checks for the listed rows, in fp64 from the GPU's tau
    (p = max(0, (alpha-1)(s - tau))^(1/(alpha-1)); alpha 1.5: ((s - tau)/2)^2; alpha 1: softmax,
    p = exp(s - tau), every allowed key in the support)."""
    a1 = alpha - 1.0
    worst_sum = 0.0
    for r, rid in enumerate(row_ids):
        i = rid % L
        bh = rid // L
        b, h = divmod(bh, H)
        mrow = None if key_mask is None else key_mask[b]
        a = allowed_matrix(L, causal, window, mrow)[i]
        if not a.any():
            assert np.isinf(tau_gpu_rows[r]) and np.isinf(tau_ref_rows[r])
            continue
        s = scale * (Kd[b, h][a] @ Qd[b, h, i])
        tg, tr = tau_gpu_rows[r], tau_ref_rows[r]
        assert abs(tg - tr) <= TAU_TOL, (rid, tg, tr)
        if alpha == 1.0:
            worst_sum = max(worst_sum, abs(np.exp(s - tg).sum() - 1.0))
            continue
        p = np.clip(a1 * (s - tg), 0, None) ** (1.0 / a1)
        worst_sum = max(worst_sum, abs(p.sum() - 1.0))
        differ = (s > tg) != (s > tr)
        assert np.all(np.abs(s[differ] - tr) < SUPPORT_BAND), (rid, s[differ], tr)
    assert worst_sum <= SUM_TOL, worst_sum
    return worst_sum


def assert_bf16_is_rounded(o_bf16: torch.Tensor, o_f32: torch.Tensor) -> None:
    """The bf16 output equals the fp32 output of the same kernel rounded to nearest even."""
    assert o_bf16.dtype == torch.bfloat16 and o_f32.dtype == torch.float32
    assert torch.equal(o_bf16, o_f32.to(torch.bfloat16))
