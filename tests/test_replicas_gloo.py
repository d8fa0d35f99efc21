"""Host-side logic of bench.py's multi-GPU replicas, on CPU with two gloo ranks.

The operation has no exchange step, so N GPUs run N independent replicas; the only cross-rank work
is the barrier around the timed region and the max of the step time over ranks, which these tests
exercise without a GPU.
"""
import os
import socket
import sys
from pathlib import Path

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        bench.dist_barrier(world)
        # each rank reports its own step time; every rank must see the slowest one
        mine = 10.0 + 5.0 * rank
        worst = bench.dist_max(mine, world, torch.device("cpu"))
        value = bench.aggregate_value(1e12, world, worst)
        Path(out_dir, "r%d.txt" % rank).write_text("%r %r" % (worst, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_whole_job_value(tmp_path, world):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = [Path(tmp_path, "r%d.txt" % r).read_text().split() for r in range(world)]
    slowest = 10.0 + 5.0 * (world - 1)
    for worst, value in got:
        assert float(worst) == slowest
        # whole-job throughput: every rank's work over the slowest rank's time (TFLOP/s)
        assert abs(float(value) - world * 1e12 / (slowest * 1e-3) / 1e12) < 1e-9


def test_single_process_helpers_need_no_process_group():
    sys.path.insert(0, str(ROOT))
    import bench

    bench.dist_barrier(1)
    assert bench.dist_max(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.aggregate_value(2e12, 1, 1000.0) == pytest.approx(2.0)


def test_allowed_pairs_by_brute_force():
    """bench.py's dense-equivalent FLOP count rests on the number of (query, key) pairs the masks
    allow: checked against a direct count over every pair."""
    sys.path.insert(0, str(ROOT))
    import bench
    from entmax_tcgen05_tma_b200.workloads import Workload

    for causal, window, lens in ((False, 0, None), (False, 0, (3, 17)), (True, 0, None), (True, 5, (4, 17))):
        w = Workload(0, "pairs", 3, 2, 17, 64, 0.125, causal, window, lens)
        km = None
        if lens is not None:
            km = torch.zeros(3, 17, dtype=torch.uint8)
            for b, n in enumerate((lens[0], 9, lens[1])):
                km[b, :n] = 1
        want = 0
        for b in range(3):
            for i in range(17):
                for j in range(17):
                    ok = (km is None or km[b, j] == 1) and (not causal or j <= i) and (window == 0 or j >= i - window + 1)
                    want += int(ok)
        assert bench.allowed_pairs(w, km) == want * 2
        assert bench.dense_equiv_flops(w, want * 2) == 14.0 * 64 * want * 2


def test_min_hbm_bytes_counts_each_tensor_once():
    sys.path.insert(0, str(ROOT))
    import bench
    from entmax_tcgen05_tma_b200.workloads import Workload

    w = Workload(0, "bytes", 2, 3, 10, 64, 0.125, len_range=(4, 10), H_kv=1)
    km = torch.zeros(2, 10, dtype=torch.uint8)
    km[0, :4] = 1
    km[1, :7] = 1
    rows, kv_rows = 2 * 3 * 10, (4 + 7) * 1
    fwd = rows * 64 * 2 + 2 * kv_rows * 64 * 2 + rows * 64 * 2 + rows * 4
    bwd = 2 * rows * 64 * 2 + 2 * kv_rows * 64 * 2 + rows * 4 + rows * 64 * 4 + 2 * 2 * 1 * 10 * 64 * 4
    assert bench.min_hbm_bytes(w, km) == fwd + bwd
    assert bench.min_hbm_bytes(w.with_shape(backward=False), km) == fwd


def test_reference_arm_under_torchrun_prints_one_line():
    """`bench.py --impl reference` launched as two ranks: rank 0 alone times the oracle and prints
    the one JSON line (with the launch's n_gpus), the other rank exits 0 without work."""
    import json
    import subprocess

    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), str(ROOT / "bench.py"),
           "--gpus", "2", "--impl", "reference", "--workload", "2", "--steps", "1", "--warmup", "3",
           "--ref-step-seconds", "0.5"]
    r = subprocess.run(cmd, capture_output=True, text=True, cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == 2 and out["steps"] == 1 and out["warmup"] == 3
    assert out["value"] > 0 and out["e2e"]["value"] == out["value"]
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["cpu_baseline"]["kind"] == "oracle"
    assert out["config"]["workload_id"] == 2


def test_link_bound_takes_the_slower_direction():
    import bench

    r = bench.link_bound({"h2d_gbs": 50.0, "d2h_gbs": 40.0}, 100_000_000, 200_000_000, 10.0)
    # 100 MB at 50 GB/s = 2 ms in, 200 MB at 40 GB/s = 5 ms out: the step cannot beat 5 ms
    assert r["copy_bound_ms"] == pytest.approx(5.0) and r["frac"] == pytest.approx(0.5)
    assert r["h2d_gbs"] == 50.0 and r["d2h_gbs"] == 40.0
    r = bench.link_bound({"h2d_gbs": 10.0, "d2h_gbs": 40.0}, 100_000_000, 200_000_000, 20.0)
    assert r["copy_bound_ms"] == pytest.approx(10.0) and r["frac"] == pytest.approx(0.5)
    assert bench.link_bound({"error": "x"}, 1, 1, 1.0) == {"error": "x"}
    # both directions at once at 50 GB/s in total: 300 MB take 6 ms, above either direction alone
    r = bench.link_bound({"h2d_gbs": 50.0, "d2h_gbs": 40.0, "duplex_gbs": 50.0}, 100_000_000, 200_000_000, 12.0)
    assert r["copy_bound_ms"] == pytest.approx(6.0) and r["frac"] == pytest.approx(0.5)
    # a full-duplex link leaves the slower direction as the bound
    r = bench.link_bound({"h2d_gbs": 50.0, "d2h_gbs": 40.0, "duplex_gbs": 90.0}, 100_000_000, 200_000_000, 10.0)
    assert r["copy_bound_ms"] == pytest.approx(5.0)


def test_link_rates_report_failure_instead_of_raising():
    import bench

    if torch.cuda.is_available():
        pytest.skip("checks the failure path, which needs a machine without a GPU")
    r = bench.host_link_rates(torch.device("cpu"), None, nbytes=1 << 10, reps=1)
    assert set(r) == {"error"}


def test_link_bound_never_divides_by_zero():
    import bench

    assert bench.link_bound({"h2d_gbs": 0.0, "d2h_gbs": 40.0}, 1, 1, 1.0) == {"h2d_gbs": 0.0, "d2h_gbs": 40.0}
    assert "copy_bound_ms" not in bench.link_bound({"h2d_gbs": 1.0, "d2h_gbs": 1.0}, 1, 1, 0.0)
