"""[B, L, H, 64] memory layout on the GPU (the _ex entry points with ENTMAX_LAYOUT_BLHD).

The attention layer of the AdaSplash pages projects to [B, L, H, d] and views it as [B, H, L, d]
through a transpose; the library reads that memory directly.  The kernels do the same arithmetic
in both layouts, so O, tau and dQ must agree bit for bit with the [B, H, L, 64] run of the same
values, dK and dV up to the order of their sums; one case is also checked against the oracle.
Ragged L makes the last tile of each batch run into the next batch's rows (masked) and, after the
last batch, into the tensor map's zero fill.
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
from tests.gpu_helpers import GRAD_TOL, O_TOL, inputs_f64, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _blhd(x: torch.Tensor) -> torch.Tensor:
    """The same values as x [B,H,L,D], held in [B,L,H,D] memory (a transpose(1, 2) view)."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


def _run(Q, K, V, dO, km, w, alpha):
    O, tau, saved = entmax_attn_fwd_ex(Q, K, V, km, w.causal, w.window, w.scale, alpha=alpha, save=True,
                                       out_dtype=torch.float32)
    O2, tau2 = entmax_attn_fwd_ex(Q, K, V, km, w.causal, w.window, w.scale, alpha=alpha, out_dtype=torch.float32)
    assert torch.equal(O, O2) and torch.equal(tau, tau2)
    g = entmax_attn_bwd_saved_ex(Q, K, V, tau, saved, dO, km, w.causal, w.window, w.scale, alpha=alpha)
    assert entmax_attn_device_status() == 0
    return O, tau, g


CASES = [
    # alpha, B, H, H_kv, L, scale, causal, window, len_range
    (1.5, 2, 3, 3, 300, 1 / 8, False, 0, (1, 300)),
    (1.5, 3, 4, 2, 129, 2 / 8, True, 0, None),
    (1.5, 2, 2, 2, 700, 1 / 8, True, 32, None),
    (1.5, 1, 4, 1, 1000, 2 / 8, False, 0, None),
    (2.0, 2, 4, 2, 513, 1 / 8, False, 0, (100, 513)),
    (1.25, 2, 2, 2, 17, 1 / 8, False, 0, None),
]


@pytest.mark.parametrize("alpha,B,H,Hkv,L,scale,causal,window,lens", CASES)
def test_blhd_matches_bhld(alpha, B, H, Hkv, L, scale, causal, window, lens):
    w = Workload(0, "layout", B, H, L, 64, scale, causal, window, lens, H_kv=Hkv)
    inp = make_inputs(w, seed=51 + L + H)
    Q, K, V, dO = (inp[k].to(DEV) for k in ("Q", "K", "V", "dO"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(DEV)
    O0, t0, g0 = _run(Q, K, V, dO, km, w, alpha)
    Qs, Ks, Vs, dOs = (_blhd(x) for x in (Q, K, V, dO))
    O1, t1, g1 = _run(Qs, Ks, Vs, dOs, km, w, alpha)
    # outputs come back in the inputs' layout
    for x in (O1, *g1):
        assert x.transpose(1, 2).is_contiguous()  # (with one head both layouts are contiguous)
    assert torch.equal(O1, O0) and torch.equal(t1, t0)
    assert torch.equal(g1[0], g0[0])
    for a, b in zip(g1[1:], g0[1:]):
        assert torch.allclose(a, b, atol=1e-5, rtol=1e-5), (a - b).abs().max().item()


def test_blhd_against_the_oracle():
    w = Workload(0, "layout", 2, 4, 384, 64, 1 / 8, True, 0, (150, 384), H_kv=2)
    inp = make_inputs(w, seed=52)
    d = inputs_f64(inp, False)
    km_np = inp["key_mask"].numpy()
    Q, K, V, dO = (_blhd(inp[k].to(DEV)) for k in ("Q", "K", "V", "dO"))
    km = inp["key_mask"].to(DEV)
    O, tau, g = _run(Q, K, V, dO, km, w, 1.5)
    O_ref, tau_ref = orc.attn_fwd_gqa(d["Q"], d["K"], d["V"], km_np, True, 0, 1 / 8)
    assert np.max(np.abs(to64(O) - O_ref)) <= O_TOL
    assert np.max(np.abs(to64(tau) - tau_ref)) <= 1e-3
    refs = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], km_np, True, 0, 1 / 8)
    for x, r in zip(g, refs):
        assert np.max(np.abs(to64(x) - r)) <= GRAD_TOL


def test_blhd_autograd_views():
    """The pages' layer: q = proj(x).view(B, L, H, d).transpose(1, 2) goes in as is."""
    B, L, H, D = 2, 200, 4, 64
    g = torch.Generator(device="cpu").manual_seed(53)
    x = [torch.randn(B, L, H, D, generator=g).to(torch.bfloat16).to(DEV).requires_grad_(True) for _ in range(3)]
    q, k, v = (t.transpose(1, 2) for t in x)
    O = EntmaxAttention.apply(q, k, v, None, True, 0, 1 / 8)
    assert O.transpose(1, 2).is_contiguous()
    dO = torch.randn(B, H, L, D, generator=g).to(torch.bfloat16).to(DEV)
    O.backward(dO)
    # the same through contiguous [B, H, L, D] copies
    y = [t.detach().transpose(1, 2).contiguous().requires_grad_(True) for t in x]
    O2 = EntmaxAttention.apply(y[0], y[1], y[2], None, True, 0, 1 / 8)
    O2.backward(dO)
    assert torch.equal(O.float(), O2.float())
    for a, b in zip(x, y):
        assert torch.allclose(a.grad.transpose(1, 2).float(), b.grad.float(), atol=1e-2, rtol=1e-2)


def test_variants_at_the_size_limits():
    """L = 16384 (the longest sequence) with sparsemax, two query heads on one key/value head and
    [B, L, H, 64] memory, causal window 32: sampled rows forward, the whole key/value head backward."""
    B, H, Hkv, L = 1, 2, 1, 16384
    w = Workload(0, "limits", B, H, L, 64, 1 / 8, True, 32, H_kv=Hkv)
    inp = make_inputs(w, seed=54)
    d = inputs_f64(inp, False)
    Q, K, V, dO = (_blhd(inp[k].to(DEV)) for k in ("Q", "K", "V", "dO"))
    O, tau, g = _run(Q, K, V, dO, None, w, 2.0)
    rng = np.random.default_rng(54)
    ids = np.unique(np.concatenate([rng.integers(0, B * H * L, size=96), [0, 31, 32, L - 1, L, 2 * L - 1]]))
    O_ref, tau_ref = orc.attn_fwd_rows_gqa(d["Q"], d["K"], d["V"], ids, None, True, 32, 1 / 8, alpha=2.0)
    assert np.max(np.abs(to64(O).reshape(-1, 64)[ids] - O_ref)) <= O_TOL
    assert np.max(np.abs(to64(tau).reshape(-1)[ids] - tau_ref)) <= 1e-3
    refs = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], None, True, 32, 1 / 8, alpha=2.0)
    for x, r in zip(g, refs):
        assert np.max(np.abs(to64(x) - r)) <= GRAD_TOL


def test_blhd_at_the_head_limit():
    """B * H = 65535 heads of two positions in [B, L, H, 64] memory (H = 3), key padding down to one
    key: the tensor maps' third dimension is B * L = 43690 positions."""
    B, H, L = 21845, 3, 2
    w = Workload(0, "head-limit", B, H, L, 64, 1 / 8, len_range=(1, 2))
    inp = make_inputs(w, seed=55)
    d = inputs_f64(inp, False)
    km_np = inp["key_mask"].numpy()
    Q, K, V, dO = (_blhd(inp[k].to(DEV)) for k in ("Q", "K", "V", "dO"))
    km = inp["key_mask"].to(DEV)
    O, tau, g = _run(Q, K, V, dO, km, w, 1.5)
    ids = np.array(sorted({0, 1, 2, 5, B * H * L - 1, B * H * L - 2} | set(range(70000, 70030))), dtype=np.int64)
    O_ref, tau_ref = orc.attn_fwd_rows(d["Q"], d["K"], d["V"], ids, km_np, False, 0, 1 / 8)
    assert np.max(np.abs(to64(O).reshape(-1, 64)[ids] - O_ref)) <= O_TOL
    assert np.max(np.abs(to64(tau).reshape(-1)[ids] - tau_ref)) <= 1e-3
    heads = [0, 1, 40000, B * H - 1]
    rQ, rK, rV = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], heads, km_np, False, 0, 1 / 8)
    for x, r in zip(g, (rQ, rK, rV)):
        assert np.max(np.abs(to64(x).reshape(-1, L, 64)[heads] - r)) <= GRAD_TOL


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25])
def test_fully_masked_batch_in_every_variant(alpha):
    """A batch whose keys are all padding, in [B, L, H, 64] memory with grouped heads: its rows have
    no allowed key, so O = 0, tau = +inf and every gradient of that batch is 0; the other batch
    against the oracle."""
    B, H, Hkv, L = 2, 4, 2, 200
    w = Workload(0, "masked", B, H, L, 64, 1 / 8, H_kv=Hkv)
    inp = make_inputs(w, seed=56)
    km_np = np.ones((B, L), dtype=np.uint8)
    km_np[1] = 0
    km_np[0, 150:] = 0
    d = inputs_f64(inp, False)
    Q, K, V, dO = (_blhd(inp[k].to(DEV)) for k in ("Q", "K", "V", "dO"))
    km = torch.from_numpy(km_np).to(DEV)
    O, tau, g = _run(Q, K, V, dO, km, w, alpha)
    assert torch.all(O[1] == 0) and torch.all(torch.isinf(tau[1])) and torch.all(tau[1] > 0)
    for x in g:
        assert torch.all(x[1] == 0)
    O_ref, tau_ref = orc.attn_fwd_gqa(d["Q"], d["K"], d["V"], km_np, False, 0, 1 / 8, alpha=alpha)
    assert np.array_equal(np.isfinite(to64(tau)), np.isfinite(tau_ref))
    assert np.max(np.abs(to64(O) - O_ref)) <= O_TOL
    assert np.max(np.abs(to64(tau)[0] - tau_ref[0])) <= 1e-3
    refs = orc.attn_bwd_gqa(d["Q"], d["K"], d["V"], d["dO"], km_np, False, 0, 1 / 8, alpha=alpha)
    for x, r in zip(g, refs):
        assert np.max(np.abs(to64(x) - r)) <= GRAD_TOL
