"""The device-side timeout path, exercised on purpose without faulting or hanging the GPU.

Every mbarrier wait in the tcgen05 kernels is bounded by entmax_attn_set_wait_timeout_ns.  With a
bound of 1 ns a wait gives up after its first 128 polls: the CTA records ENTMAX_ERR_TIMEOUT in the
device status word, every role stops, the CTA drains the TMA loads and MMAs it issued and frees its
tensor memory, and the kernel returns.  The test checks that the status reports the timeout, that
the CUDA context stays usable, and that with the default bound restored the next calls match the
fp64 oracle again.
"""
import numpy as np
import pytest
import torch

import entmax_tcgen05_tma_b200 as E
from entmax_tcgen05_tma_b200.workloads import Workload, make_inputs
from oracle import oracle as orc
from tests.gpu_helpers import GRAD_TOL, O_TOL, inputs_f64, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L,causal", [(300, False), (2048, True)])
def test_forced_timeout_then_recovery(L, causal):
    w = Workload(0, "timeout", 2, 2, L, 64, 1 / 8, causal=causal)
    inp = make_inputs(w, seed=71 + L)
    Q, K, V, dO = (inp[k].cuda() for k in ("Q", "K", "V", "dO"))
    assert E.entmax_attn_device_status() == 0
    try:
        E.entmax_attn_set_wait_timeout_ns(1)
        O, tau = E.entmax_attn_fwd(Q, K, V, None, causal, 0, w.scale, out_dtype=torch.float32)
        assert E.entmax_attn_device_status() == E.ENTMAX_ERR_TIMEOUT
        # the recompute backward runs the same bounded pipeline (score passes on tcgen05)
        E.entmax_attn_bwd(Q, K, V, torch.zeros_like(tau), dO, None, causal, 0, w.scale)
        assert E.entmax_attn_device_status() == E.ENTMAX_ERR_TIMEOUT
    finally:
        E.entmax_attn_set_wait_timeout_ns(0)
    # the status word was cleared by the read, and the context still works
    assert E.entmax_attn_device_status() == 0
    torch.cuda.synchronize()
    O, tau = E.entmax_attn_fwd(Q, K, V, None, causal, 0, w.scale, out_dtype=torch.float32)
    dQ, dK, dV = E.entmax_attn_bwd(Q, K, V, tau, dO, None, causal, 0, w.scale)
    assert E.entmax_attn_device_status() == 0
    d = inputs_f64(inp, False)
    O_ref, tau_ref = orc.attn_fwd(d["Q"], d["K"], d["V"], None, causal, 0, w.scale)
    assert np.max(np.abs(to64(O) - O_ref)) <= O_TOL
    assert np.max(np.abs(to64(tau) - tau_ref)) <= 1e-3
    heads = [0, w.B * w.H - 1]
    rQ, rK, rV = orc.attn_bwd_heads(d["Q"], d["K"], d["V"], d["dO"], heads, None, causal, 0, w.scale)
    for name, g, r in zip(("dQ", "dK", "dV"), (dQ, dK, dV), (rQ, rK, rV)):
        err = np.max(np.abs(to64(g).reshape(w.B * w.H, L, 64)[heads] - r))
        assert err <= GRAD_TOL, (name, err)


def test_saved_backward_after_a_forward_that_gave_up():
    """A training forward whose waits give up leaves its support lists half-written.  While that
    error is recorded (not yet read), the support-list backward reads none of them: the call returns,
    the status still reports the timeout, and the context works afterwards."""
    w = Workload(0, "timeout-train", 1, 2, 1000, 64, 1 / 8)
    inp = make_inputs(w, seed=73)
    Q, K, V, dO = (inp[k].cuda() for k in ("Q", "K", "V", "dO"))
    assert E.entmax_attn_device_status() == 0
    try:
        E.entmax_attn_set_wait_timeout_ns(1)
        O, tau, saved = E.entmax_attn_fwd_train(Q, K, V, None, False, 0, w.scale)
    finally:
        E.entmax_attn_set_wait_timeout_ns(0)
    E.entmax_attn_bwd_saved(Q, K, V, tau, saved, dO, None, False, 0, w.scale)
    assert E.entmax_attn_device_status() == E.ENTMAX_ERR_TIMEOUT
    torch.cuda.synchronize()
    O, tau, saved = E.entmax_attn_fwd_train(Q, K, V, None, False, 0, w.scale)
    grads = E.entmax_attn_bwd_saved(Q, K, V, tau, saved, dO, None, False, 0, w.scale)
    assert E.entmax_attn_device_status() == 0
    d = inputs_f64(inp, False)
    refs = orc.attn_bwd(d["Q"], d["K"], d["V"], d["dO"], None, False, 0, w.scale)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, refs):
        assert np.max(np.abs(to64(g) - r)) <= GRAD_TOL, name
