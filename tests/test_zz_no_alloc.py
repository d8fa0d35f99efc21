"""The allocation-free backward (entmax_attn_bwd_noalloc) against the workspace backward.

Callers that cannot allocate device memory when they run the backward pass (pre-planned memory
engines, code inside stream capture, latency-critical loops) use entmax_attn_bwd_noalloc, whose
scratch is a fixed array inside the library.  Its gradients must match entmax_attn_bwd's within the
gradient tolerance of the parity tests, on two calls in a row (the second sees the array as the
first left it).  This file is collected last on purpose, and passes alone in a fresh process too.
"""
import pytest
import torch

import entmax_tcgen05_tma_b200 as E
from entmax_tcgen05_tma_b200.workloads import Workload, make_inputs
from tests.gpu_helpers import GRAD_TOL

pytestmark = pytest.mark.gpu


def _run(w: Workload, seed: int):
    inp = make_inputs(w, seed=seed)
    Q, K, V, dO = (inp[k].cuda() for k in ("Q", "K", "V", "dO"))
    km = None if inp["key_mask"] is None else inp["key_mask"].cuda()
    O, tau = E.entmax_attn_fwd(Q, K, V, km, w.causal, w.window, w.scale)
    ref = E.entmax_attn_bwd(Q, K, V, tau, dO, km, w.causal, w.window, w.scale)
    got = E.entmax_attn_bwd_noalloc(Q, K, V, tau, dO, km, w.causal, w.window, w.scale)
    assert E.entmax_attn_device_status() == 0
    for a, b in zip(ref, got):
        err = float((a - b).abs().max())
        assert err <= GRAD_TOL, err
        assert torch.isfinite(b).all()
    return got


def test_noalloc_matches_workspace_backward_twice():
    first = _run(Workload(0, "noalloc-1", 2, 3, 300, 64, 1 / 8, len_range=(100, 300)), seed=21)
    # a second call with another shape and mask: the scratch still holds the first call's values
    second = _run(Workload(0, "noalloc-2", 1, 4, 520, 64, 1 / 8, causal=True, window=32), seed=22)
    assert first[0].shape != second[0].shape


def test_noalloc_rejects_oversized_and_fp32():
    x = torch.zeros(1, 1, 8, 64, dtype=torch.float32, device="cuda")
    t = torch.zeros(1, 1, 8, dtype=torch.float32, device="cuda")
    with pytest.raises(E.EntmaxError) as ei:
        E.entmax_attn_bwd_noalloc(x, x, x, t, x)
    assert ei.value.status == E.ENTMAX_ERR_UNSUPPORTED
    p = 0x10000  # never dereferenced: the size check fails first
    st = E.lib.entmax_attn_bwd_noalloc(p, p, p, 0, None, 0, 0, 0.125, 64, 128, 129, 64, p, p, p, p, p, None)
    assert st == E.ENTMAX_ERR_UNSUPPORTED
