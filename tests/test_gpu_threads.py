"""Several host threads calling the library at once, each on its own CUDA stream: every thread's
forward and saved backward equal a single-threaded run of the same inputs (O, tau and dQ bit for
bit; dK and dV up to the order of their sums), and the device status stays clear."""
import threading

import pytest
import torch

from entmax_tcgen05_tma_b200 import (
    entmax_attn_bwd_saved_gqa,
    entmax_attn_device_status,
    entmax_attn_fwd_train_gqa,
)
from entmax_tcgen05_tma_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _step(Q, K, V, dO, km):
    O, tau, saved = entmax_attn_fwd_train_gqa(Q, K, V, km, True, 0, 1 / 8, out_dtype=torch.float32)
    return O, tau, entmax_attn_bwd_saved_gqa(Q, K, V, tau, saved, dO, km, True, 0, 1 / 8)


def test_concurrent_host_threads():
    w = Workload(0, "threads", 2, 4, 300, 64, 1 / 8, True, 0, (100, 300), H_kv=2)
    inp = make_inputs(w, seed=57)
    Q, K, V, dO = (inp[k].to(DEV) for k in ("Q", "K", "V", "dO"))
    km = inp["key_mask"].to(DEV)
    O0, t0, g0 = _step(Q, K, V, dO, km)
    torch.cuda.synchronize()
    n = 4
    results, errors = [None] * n, []
    start = threading.Barrier(n)

    def work(k):
        try:
            s = torch.cuda.Stream()
            start.wait(timeout=60)
            with torch.cuda.stream(s):
                out = _step(Q, K, V, dO, km)
            s.synchronize()
            results[k] = out
        except Exception as e:  # reported below, on the main thread
            errors.append(e)

    threads = [threading.Thread(target=work, args=(k,)) for k in range(n)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads)
    assert not errors, errors
    assert entmax_attn_device_status() == 0
    for O, tau, g in results:
        assert torch.equal(O, O0) and torch.equal(tau, t0)
        assert torch.equal(g[0], g0[0])
        for a, b in zip(g[1:], g0[1:]):
            assert torch.allclose(a, b, atol=1e-5, rtol=1e-5), (a - b).abs().max().item()


def test_first_cuda_work_of_a_new_thread():
    """A host thread whose first CUDA work is a call into the library (no context current yet: a
    new thread, or an autograd worker): the calls that encode tensor maps -- the 1.5-entmax forward,
    the tensor-core backward, softmax -- must run there as on the main thread, bit for bit (the
    support-list backward of alpha 1.75: dK, dV to the order of their atomically bucketed sums)."""
    from entmax_tcgen05_tma_b200 import EntmaxAttention, entmax_attn_bwd_saved_ex, entmax_attn_fwd_ex

    w = Workload(0, "new-thread", 1, 2, 200, 64, 1 / 8, True, 0)
    inp = make_inputs(w, seed=89)
    Q, K, V, dO = (inp[k].to(DEV) for k in ("Q", "K", "V", "dO"))

    def step(alpha):
        O, tau, saved = entmax_attn_fwd_ex(Q, K, V, None, True, 0, w.scale, alpha=alpha, save=True)
        g = entmax_attn_bwd_saved_ex(Q, K, V, tau, saved, dO, None, True, 0, w.scale, alpha=alpha)
        torch.cuda.synchronize()
        return (O, tau) + tuple(g)

    for alpha in (1.5, 1.0, 1.75):
        ref = step(alpha)
        out, errors = [], []

        def work():
            try:
                out.append(step(alpha))
            except Exception as e:  # noqa: BLE001 -- reported below
                errors.append(e)

        t = threading.Thread(target=work)
        t.start()
        t.join(timeout=120)
        assert not errors, (alpha, errors)
        assert entmax_attn_device_status() == 0
        for k, (x, y) in enumerate(zip(out[0], ref)):
            if alpha == 1.75 and k >= 3:
                assert torch.allclose(x, y, atol=1e-5, rtol=1e-5), alpha
            else:
                assert torch.equal(x, y), (alpha, k)
    # the autograd wrapper: its backward runs on the autograd engine's worker thread
    for alpha in (1.5, 1.0):
        q, k, v = (x.clone().requires_grad_(True) for x in (Q, K, V))
        O = EntmaxAttention.apply(q, k, v, None, True, 0, w.scale, alpha)
        O.backward(dO)
        assert entmax_attn_device_status() == 0
        assert all(torch.isfinite(x.grad).all() for x in (q, k, v))
