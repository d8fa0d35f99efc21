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
