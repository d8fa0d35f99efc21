"""The allocation-free backward (entmax_attn_bwd_noalloc) against the workspace backward.

Callers that cannot allocate device memory when they run the backward pass (pre-planned memory
engines, code inside stream capture, latency-critical loops) use entmax_attn_bwd_noalloc, whose
scratch is a fixed array inside the library.  It launches the same kernels as entmax_attn_bwd, which
sum in a fixed order (no atomics), so its gradients must equal entmax_attn_bwd's bit for bit.  The
larger call runs first and a smaller one second, so the second call starts from an array that
still holds the first call's values beyond its own rows.  One case is also checked against the fp64
oracle.  This file is collected last on purpose, and passes alone in a fresh process too.
"""
import numpy as np
import pytest
import torch

import entmax_tcgen05_tma_b200 as E
from entmax_tcgen05_tma_b200.workloads import Workload, make_inputs
from oracle import oracle as orc
from tests.gpu_helpers import GRAD_TOL, inputs_f64, to64

pytestmark = pytest.mark.gpu


def _run(w: Workload, seed: int):
    inp = make_inputs(w, seed=seed)
    Q, K, V, dO = (inp[k].cuda() for k in ("Q", "K", "V", "dO"))
    km = None if inp["key_mask"] is None else inp["key_mask"].cuda()
    O, tau = E.entmax_attn_fwd(Q, K, V, km, w.causal, w.window, w.scale)
    # the minimum workspace: entmax_attn_bwd then runs the kernels the allocation-free entry point
    # runs at every length (with the full workspace, long rows list their supports from tau)
    ws = torch.empty(E.bwd_min_workspace_size(w.B, w.H, w.L), dtype=torch.uint8, device="cuda")
    ref = E.entmax_attn_bwd(Q, K, V, tau, dO, km, w.causal, w.window, w.scale, workspace=ws)
    got = E.entmax_attn_bwd_noalloc(Q, K, V, tau, dO, km, w.causal, w.window, w.scale)
    assert E.entmax_attn_device_status() == 0
    for a, b in zip(ref, got):
        assert torch.equal(a, b), float((a - b).abs().max())
    return inp, got


def test_noalloc_matches_workspace_backward_twice():
    big = Workload(0, "noalloc-1", 1, 4, 520, 64, 1 / 8, causal=True, window=32)
    small = Workload(0, "noalloc-2", 2, 3, 300, 64, 1 / 8, len_range=(100, 300))
    long = Workload(0, "noalloc-3", 1, 2, 700, 64, 1 / 8)  # long rows: the recompute kernels
    assert big.B * big.H * big.L > small.B * small.H * small.L
    _run(long, seed=23)
    _run(big, seed=22)
    # the second, smaller call: the array still holds the first call's values past its rows
    inp, got = _run(small, seed=21)
    d = inputs_f64(inp, False)
    km = inp["key_mask"].numpy()
    refs = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], km, small.causal, small.window, small.scale)
    for name, g, r in zip(("dQ", "dK", "dV"), got, refs):
        err = np.max(np.abs(to64(g) - r))
        assert err <= GRAD_TOL, (name, err)


def test_noalloc_rejects_oversized_and_fp32():
    x = torch.zeros(1, 1, 8, 64, dtype=torch.float32, device="cuda")
    t = torch.zeros(1, 1, 8, dtype=torch.float32, device="cuda")
    with pytest.raises(E.EntmaxError) as ei:
        E.entmax_attn_bwd_noalloc(x, x, x, t, x)
    assert ei.value.status == E.ENTMAX_ERR_UNSUPPORTED
    p = 0x10000  # never dereferenced: the size check fails first
    st = E.lib.entmax_attn_bwd_noalloc(p, p, p, 0, None, 0, 0, 0.125, 64, 128, 129, 64, p, p, p, p, p, None)
    assert st == E.ENTMAX_ERR_UNSUPPORTED
