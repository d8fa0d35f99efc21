#!/usr/bin/env python3
"""Benchmark of 1.5-entmax attention forward+backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload {2,3,4,5}] [--impl {b200,reference}]

One step = entmax_attn_fwd_train + entmax_attn_bwd_saved (the training path: forward with saved
supports, then the closed-form backward from them) over one batch of synthetic inputs resident in
HBM; forward-only workloads run entmax_attn_fwd.  Prints ONE JSON line (rank 0).

Metric: dense-equivalent TFLOP/s = 14 * d * P / t_step (fwd+bwd; 4 * d * P for forward-only
workloads), where P counts the (query, key) pairs the masks allow -- entmax zeros are never
subtracted.  ms_per_step is reported beside it.  Default workload: 4 (B=4, H=12, L=4096, d=64,
scale 2/8, no mask), the tensor-bound fwd+bwd configuration.

Multi-GPU: the operation does not shard (every (b, h) is independent and the workloads fit one
GPU), so --gpus N runs N independent replicas, one per rank, with no data-path collective;
value = total work of all ranks / max step time over ranks ("scaling": "weak").

--impl reference times the fp64 CPU oracle on the host cores (bounded sample per step).

Variants (side measurements, not the headline line): --alpha A runs alpha-entmax for A in (1, 2],
--hkv N grouped-query attention with N key/value heads and --blhd keeps Q, K, V, dO (and the
outputs) in [B, L, H, 64] memory, all through entmax_attn_fwd_ex / entmax_attn_bwd_saved_ex; the
dense-equivalent FLOP count is unchanged (it counts query heads).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

import torch  # noqa: E402

from entmax_tcgen05_tma_b200.workloads import WORKLOADS, Workload, make_inputs  # noqa: E402

METRIC = "1.5-entmax attn fwd+bwd ms & dense-equiv TFLOP/s vs bf16 peak, 1 B200"
L2_FLUSH_BYTES = 256 << 20


def allowed_pairs(w: Workload, key_mask) -> int:
    """(query, key) pairs allowed by key padding, causal and window, over all (b, h)."""
    L = w.L
    i = torch.arange(L).unsqueeze(1)
    j = torch.arange(L).unsqueeze(0)
    band = torch.ones(L, L, dtype=torch.bool)
    if w.causal:
        band &= j <= i
    if w.window > 0:
        band &= j >= i - w.window + 1
    if key_mask is None:
        per_b = torch.full((w.B,), int(band.sum()), dtype=torch.int64)
    else:
        per_b = (band.unsqueeze(0) & key_mask.bool().unsqueeze(1)).sum(dim=(1, 2))
    return int(per_b.sum()) * w.H


def dense_equiv_flops(w: Workload, pairs: int) -> float:
    return (14.0 if w.backward else 4.0) * w.D * pairs


def min_hbm_bytes(w: Workload, key_mask) -> float:
    """Bytes a step must move at least, each tensor once: the forward reads Q and the K, V rows of
    valid keys and writes O (bf16) and tau; the backward reads Q, K, V (valid rows), dO and tau and
    writes dQ, dK, dV (fp32)."""
    D, in_b = w.D, (4 if w.fp32_inputs else 2)
    rows = w.B * w.H * w.L
    valid_keys = w.B * w.L if key_mask is None else int(key_mask.to(torch.int64).sum())
    kv_rows = valid_keys * w.kv_heads
    fwd = rows * D * in_b + 2 * kv_rows * D * in_b + rows * D * 2 + rows * 4
    if not w.backward:
        return float(fwd)
    bwd = 2 * rows * D * in_b + 2 * kv_rows * D * in_b + rows * 4 + rows * D * 4 + 2 * w.B * w.kv_heads * w.L * D * 4
    return float(fwd + bwd)


def workload_desc(w: Workload) -> str:
    s = "%s: B=%d H=%d L=%d d=%d scale=%g" % (w.name, w.B, w.H, w.L, w.D, w.scale)
    if w.len_range:
        s += " key-padding len U[%d,%d]" % w.len_range
    if w.causal:
        s += " causal"
    if w.window:
        s += " window=%d" % w.window
    return s


def load_peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            for line in Path(self.path).read_text().splitlines():
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        finally:
            if self.path:
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        smax = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ----------------------------------------------------------------------------- oracle
def oracle_baseline(w: Workload, inp: dict, budget_s: float = 12.0, max_heads: int = 64, alpha: float = 1.5,
                    threads: int = 0) -> dict:
    """Time the fp64 oracle (as it stands) on whole heads of the workload until ~budget_s; threads > 0
    limits its OpenMP threads for the call."""
    from oracle import oracle as orc

    if threads > 0:
        before = orc.num_threads()
        orc.set_num_threads(threads)
        try:
            return oracle_baseline(w, inp, budget_s, max_heads, alpha)
        finally:
            orc.set_num_threads(before)

    f64 = {k: inp[k].to(torch.float64).numpy() for k in ("Q", "K", "V", "dO")}
    if w.kv_heads != w.H:  # grouped heads: the oracle's repeat of K and V (outside the timed loop)
        for k in ("K", "V"):
            f64[k] = orc.repeat_kv(f64[k], w.H // w.kv_heads)
    km = None if inp["key_mask"] is None else inp["key_mask"].numpy()
    pairs_per_head = []
    full_pairs = allowed_pairs(w, inp["key_mask"])
    BH = w.B * w.H
    heads = 0
    t0 = time.perf_counter()
    while heads < min(max_heads, BH) and time.perf_counter() - t0 < budget_s:
        bh = (heads * 7919) % BH
        b = bh // w.H
        L = w.L
        rows = bh * L + torch.arange(L).numpy()
        orc.attn_fwd_rows(f64["Q"], f64["K"], f64["V"], rows, km, w.causal, w.window, w.scale, alpha=alpha)
        if w.backward:
            orc.attn_bwd_heads(f64["Q"], f64["K"], f64["V"], f64["dO"], [bh], km, w.causal, w.window, w.scale,
                               alpha=alpha)
        sub = w.with_shape(B=1)
        pairs_per_head.append(allowed_pairs(sub.with_shape(H=1), None if km is None else inp["key_mask"][b:b + 1]))
        heads += 1
    dt = time.perf_counter() - t0
    flops = dense_equiv_flops(w, sum(pairs_per_head))
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": "%d of %d heads (fwd%s) of the workload, %.1f s" % (heads, BH, "+bwd" if w.backward else "", dt),
            "seconds": dt, "heads": heads, "full_job_seconds_est": dt * full_pairs / max(1, sum(pairs_per_head))}


def host_link_rates(dev, stream, nbytes: int = 1 << 28, reps: int = 5) -> dict:
    """Pinned copy rates (GB/s) of this GPU's host link, timed with CUDA events: host-to-device and
    device-to-host one direction at a time, then both at once on two streams ("duplex_gbs", bytes
    of both directions over the time both took) -- the ceilings of the end-to-end copies.  Runs
    outside every timed region; any failure is reported instead of the rates."""
    try:
        h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
        d = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        h2 = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
        d2 = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        rates = {}
        with torch.cuda.stream(stream):
            for name, dst, src in (("h2d_gbs", d, h), ("d2h_gbs", h, d)):
                dst.copy_(src, non_blocking=True)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    dst.copy_(src, non_blocking=True)
                e1.record(stream)
                e1.synchronize()
                rates[name] = round(nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9, 2)
        other = torch.cuda.Stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        other.wait_event(e0)
        with torch.cuda.stream(stream):
            for _ in range(reps):
                d.copy_(h, non_blocking=True)
        with torch.cuda.stream(other):
            for _ in range(reps):
                h2.copy_(d2, non_blocking=True)
        stream.wait_stream(other)
        e1.record(stream)
        e1.synchronize()
        rates["duplex_gbs"] = round(2 * nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9, 2)
        return rates
    except Exception as exc:  # a measurement aid only: never fail the bench line for it
        return {"error": repr(exc)[:200]}


def link_bound(rates: dict, h2d_bytes: int, d2h_bytes: int, e2e_ms: float) -> dict:
    """The end-to-end step against its copy time: each direction's bytes over its own rate, and the
    bytes of both over the rate the link sustains with both directions busy; the bound is the
    largest of the three."""
    if not (rates.get("h2d_gbs", 0) > 0 and rates.get("d2h_gbs", 0) > 0 and e2e_ms > 0):
        return dict(rates)
    bound_ms = 1e3 * max(h2d_bytes / (rates["h2d_gbs"] * 1e9), d2h_bytes / (rates["d2h_gbs"] * 1e9))
    if rates.get("duplex_gbs", 0) > 0:
        bound_ms = max(bound_ms, 1e3 * (h2d_bytes + d2h_bytes) / (rates["duplex_gbs"] * 1e9))
    return {**rates, "copy_bound_ms": round(bound_ms, 4), "frac": round(bound_ms / e2e_ms, 4)}


# ----------------------------------------------------------------------------- GPU arm
def measured_sparsity(w: Workload, Q, K, tau, km) -> float:
    """Fraction of allowed pairs with A = 0 (scores recomputed in fp32 with torch, outside the timed
    region; only for reporting)."""
    zeros = 0
    allowed = 0
    L = w.L
    i = torch.arange(L, device=Q.device).unsqueeze(1)
    j = torch.arange(L, device=Q.device).unsqueeze(0)
    band = torch.ones(L, L, dtype=torch.bool, device=Q.device)
    if w.causal:
        band &= j <= i
    if w.window:
        band &= j >= i - w.window + 1
    rep = w.H // w.kv_heads
    for b in range(w.B):
        a = band if km is None else band & km[b].bool().unsqueeze(0)
        for h in range(w.H):
            S = w.scale * (Q[b, h].float() @ K[b, h // rep].float().T)
            supp = (S > tau[b, h].unsqueeze(1)) & a
            allowed += int(a.sum())
            zeros += int(a.sum()) - int(supp.sum())
    return zeros / max(1, allowed)


class _Flush:
    """Evicts L2 between timed steps, outside the step's events: a 256 MiB write (larger than the
    126 MB L2), then a 256 MiB read of a second buffer, so L2 is left holding clean lines and the
    timed kernels neither hit on their inputs nor write back the flush's dirty lines."""

    def __init__(self, dev):
        self.w = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device=dev)
        self.r = torch.ones((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self, k: int) -> None:
        self.w.fill_(float(k))
        torch.sum(self.r, dim=0, out=self.sink)


class _Prepared:
    """Device-resident inputs, outputs and the step's library calls for one workload."""

    def __init__(self, args, w: Workload, dev, alpha: float | None = None):
        import entmax_tcgen05_tma_b200 as E

        self.E, self.w, self.dev = E, w, dev
        alpha = args.alpha if alpha is None else alpha
        self.variant = variant = alpha != 1.5 or w.kv_heads != w.H or args.blhd  # the _ex entry points
        # entmax_attn_fwd + entmax_attn_bwd: with its full workspace, or with the minimum (one float per
        # row), which runs the recompute kernels at long rows
        self.recompute = recompute = args.bwd in ("recompute", "recompute-min")
        self.inp = inp = make_inputs(w)
        self.pairs = allowed_pairs(w, inp["key_mask"])
        self.flops = dense_equiv_flops(w, self.pairs)
        # --blhd: the same values held in [B, L, H, 64] memory, passed as transpose(1, 2) views
        lay = (lambda x: x.transpose(1, 2).contiguous().transpose(1, 2)) if args.blhd else (lambda x: x)
        self.Q, self.K, self.V, self.dO = (lay(inp[k].to(dev)) for k in ("Q", "K", "V", "dO"))
        self.km = None if inp["key_mask"] is None else inp["key_mask"].to(dev)
        B, H, L, D = w.B, w.H, w.L, w.D
        Hkv = w.kv_heads
        self.O = lay(torch.empty((B, H, L, D), dtype=torch.bfloat16, device=dev))
        self.tau = torch.empty((B, H, L), dtype=torch.float32, device=dev)
        self.dQ = lay(torch.empty((B, H, L, D), dtype=torch.float32, device=dev))
        self.dK, self.dV = (lay(torch.empty((B, Hkv, L, D), dtype=torch.float32, device=dev)) for _ in range(2))
        self.saved = torch.empty((E.entmax_attn_saved_bytes(B, H, L, D),), dtype=torch.uint8, device=dev)
        self.ws = torch.empty((E.entmax_attn_bwd_saved_workspace_size(B, H, L, D),), dtype=torch.uint8, device=dev)
        rws = E.bwd_min_workspace_size(B, H, L) if args.bwd == "recompute-min" else \
            E.entmax_attn_bwd_workspace_size(B, H, L, D)
        self.rws = torch.empty((max(rws, 1),), dtype=torch.uint8, device=dev)
        self.alpha = alpha

    def fwd_call(self):
        E, w = self.E, self.w
        Q, K, V, km, O, tau = self.Q, self.K, self.V, self.km, self.O, self.tau
        if self.recompute:
            E.entmax_attn_fwd(Q, K, V, km, w.causal, w.window, w.scale, O=O, tau=tau)
        elif self.variant:
            E.entmax_attn_fwd_ex(Q, K, V, km, w.causal, w.window, w.scale, alpha=self.alpha, save=w.backward, O=O,
                                 tau=tau, saved=self.saved if w.backward else None)
        elif w.backward:
            E.entmax_attn_fwd_train(Q, K, V, km, w.causal, w.window, w.scale, O=O, tau=tau, saved=self.saved)
        else:
            E.entmax_attn_fwd(Q, K, V, km, w.causal, w.window, w.scale, O=O, tau=tau)

    def bwd_call(self):
        E, w = self.E, self.w
        Q, K, V, km, tau, dO = self.Q, self.K, self.V, self.km, self.tau, self.dO
        if self.recompute:
            E.entmax_attn_bwd(Q, K, V, tau, dO, km, w.causal, w.window, w.scale, dQ=self.dQ, dK=self.dK, dV=self.dV,
                              workspace=self.rws)
        elif self.variant:
            E.entmax_attn_bwd_saved_ex(Q, K, V, tau, self.saved, dO, km, w.causal, w.window, w.scale,
                                       alpha=self.alpha, dQ=self.dQ, dK=self.dK, dV=self.dV, workspace=self.ws)
        else:
            E.entmax_attn_bwd_saved(Q, K, V, tau, self.saved, dO, km, w.causal, w.window, w.scale, dQ=self.dQ,
                                    dK=self.dK, dV=self.dV, workspace=self.ws)

    def step(self):
        self.fwd_call()
        if self.w.backward:
            self.bwd_call()


def tensor_core_backward(w: Workload, alpha: float = 1.5) -> bool:
    """Whether the library runs the backward on its tensor-core kernels (dq, dkdv): softmax (alpha 1)
    always, alpha 1.5 with L <= 512 or a causal window of at most 128 keys (the library's own
    dispatch rule; alpha 1.5's forward then runs its tensor-core kernel too)."""
    return alpha == 1.0 or (alpha == 1.5 and (w.L <= 512 or (w.causal and 0 < w.window <= 128)))


def launches_per_step(w: Workload, recompute: bool, alpha: float = 1.5, minimum: bool = False) -> int:
    """The library's kernel launches in one step: the forward kernel, then the backward's kernels
    (tensor-core configurations: dq and dkdv; otherwise the support-list backward: key scan, rows,
    keys and the exact pass for unsaved rows -- which entmax_attn_bwd, given its full workspace,
    precedes by the support extraction that lists each row's support from tau; with the minimum
    workspace its recompute kernels, rows and keys)."""
    if not w.backward:
        return 1
    if tensor_core_backward(w, alpha):
        return 3
    if recompute:
        return 1 + (2 if minimum else 5)
    return 1 + 4


def time_device(prep: _Prepared, flush: _Flush, steps: int, warmup: int, world: int) -> dict:
    """W warm-up steps, then `steps` timed steps: L2 evicted before each (outside the events), CUDA
    events on the launching stream around the forward and the backward, clocks sampled during the
    timed region.  Per-step lists in ms; `total_ms` is the max over ranks."""
    E, dev, w = prep.E, prep.dev, prep.w
    stream = torch.cuda.current_stream(dev)
    for k in range(warmup):
        flush(k)
        prep.step()
    torch.cuda.synchronize(dev)
    st = E.entmax_attn_device_status()
    if st != 0:
        raise RuntimeError("device status %d after warm-up" % st)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    dist_barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        wall0 = time.perf_counter()
        for k in range(steps):
            flush(k)
            ev[k][0].record(stream)
            prep.fwd_call()
            ev[k][1].record(stream)
            if w.backward:
                prep.bwd_call()
            ev[k][2].record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
    dist_barrier(world)
    st = E.entmax_attn_device_status()
    if st != 0:
        raise RuntimeError("device status %d after the timed steps" % st)
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    return {"fwd_ms": [a.elapsed_time(b) for a, b, _ in ev], "bwd_ms": [b.elapsed_time(c) for _, b, c in ev],
            "step_ms": step_ms, "total_ms": dist_max(sum(step_ms), world, dev), "wall_s": wall,
            "clocks": clk.summary()}


def step_roofline(w: Workload, km, flops: float, ms_per_step: float, peaks: dict) -> dict:
    """The whole step against its roofline time: max(dense-equivalent FLOPs / bf16 burst peak,
    minimum HBM bytes / HBM peak), as a fraction of the measured step time."""
    step_bytes = min_hbm_bytes(w, km)
    t_flop, t_byte = flops / (peaks["bf16_tflops"] * 1e12), step_bytes / (peaks["hbm_gbs"] * 1e9)
    return {"bound": "tensor" if t_flop >= t_byte else "hbm", "time_us": round(1e6 * max(t_flop, t_byte), 2),
            "frac": round(1e3 * max(t_flop, t_byte) / ms_per_step, 4), "min_hbm_bytes": step_bytes,
            "peaks": "bf16 %.1f TFLOP/s (burst), HBM %.1f GB/s (%s)" % (peaks["bf16_tflops"], peaks["hbm_gbs"],
                                                                     peaks["source"])}


def extra_workload(args, w: Workload, dev, world: int, flush: _Flush, peaks: dict, alpha: float = 1.5) -> dict:
    """Another fwd+bwd workload timed in the same process and the same way as the headline line
    (same library calls, L2 eviction, events, warm-up and step count)."""
    prep = _Prepared(args, w, dev, alpha)
    t = time_device(prep, flush, args.steps, args.warmup, world)
    ms = t["total_ms"] / args.steps
    # softmax keeps every allowed pair (no zeros to count)
    sparsity = 0.0 if alpha == 1.0 else measured_sparsity(w, prep.Q, prep.K, prep.tau, prep.km)
    out = {"workload": workload_desc(w), "alpha": alpha, "steps": args.steps, "warmup": args.warmup,
           "value": round(aggregate_value(prep.flops, world, ms), 3), "unit": "TFLOP/s",
           "ms_per_step": round(ms, 4), "fwd_ms": round(statistics.mean(t["fwd_ms"]), 4),
           "bwd_ms": round(statistics.mean(t["bwd_ms"]), 4) if w.backward else 0.0,
           "step_ms_median": round(statistics.median(t["step_ms"]), 4),
           "dense_equiv_gflop_per_step": prep.flops / 1e9, "allowed_pairs": prep.pairs,
           "sparsity": round(sparsity, 4), "step_roofline": step_roofline(w, prep.km, prep.flops, ms, peaks),
           "gpu_launches": launches_per_step(w, prep.recompute, alpha) * args.steps, "clocks": t["clocks"]}
    if alpha == 1.0:
        # softmax forward kernel: its algorithmic work is the dense 4 d P of S = Q K^T and P V (every
        # allowed pair is in the support); the tensor core issues 8 d P (S twice, P as two bf16 parts)
        fwd_ms = statistics.mean(t["fwd_ms"])
        alg = 4.0 * w.D * prep.pairs
        out["roofline"] = {"kernel": "softmax_fwd_kernel", "bound": "tensor",
                           "achieved": alg / (fwd_ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                           "unit": "TFLOP/s", "peak_source": "%s bf16 burst (MEASURED_PEAKS.json)" % peaks["source"],
                           "algorithmic_flops_per_launch": alg, "issued_mma_flops_per_launch": 2.0 * alg,
                           "traffic": None}
        out["roofline"]["frac"] = out["roofline"]["achieved"] / out["roofline"]["peak"]
        tr = ROOT / "profiles" / ("traffic_softmax_workload%d.txt" % w.wid)
        if tr.exists() and w.H == w.kv_heads and not args.blhd:
            t = json.loads(tr.read_text())
            if t.get("kernel") == "softmax_fwd_kernel" and t.get("source_hash") == source_hash("softmax_fwd_kernel"):
                out["roofline"]["traffic"] = t["bytes_per_launch"]
    del prep
    torch.cuda.empty_cache()
    return out


def run_gpu(args, rank: int, world: int) -> dict | None:
    import entmax_tcgen05_tma_b200 as E

    w = bench_workload(args)
    alpha = args.alpha
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    prep = _Prepared(args, w, dev)
    variant, recompute = prep.variant, prep.recompute
    inp, pairs, flops = prep.inp, prep.pairs, prep.flops
    Q, K, tau, km = prep.Q, prep.K, prep.tau, prep.km
    B, H, L, D = w.B, w.H, w.L, w.D
    Hkv = w.kv_heads
    O = prep.O
    stream = torch.cuda.current_stream(dev)
    flush = _Flush(dev)

    t = time_device(prep, flush, args.steps, args.warmup, world)
    fwd_ms, bwd_ms, step_ms, total_ms = t["fwd_ms"], t["bwd_ms"], t["step_ms"], t["total_ms"]
    clocks, wall = t["clocks"], t["wall_s"]
    # ---- end to end through the public API, host buffers, copies inside the timed region
    host_in = {k: inp[k].pin_memory() for k in ("Q", "K", "V", "dO")}
    if args.blhd:  # host tensors in [B, L, H, 64] memory too
        host_in = {k: v.transpose(1, 2).contiguous().pin_memory().transpose(1, 2) for k, v in host_in.items()}
    host_km = None if inp["key_mask"] is None else inp["key_mask"].pin_memory()
    def host_empty(shape, dtype):  # pinned, in the device tensors' memory layout
        if args.blhd:
            b_, h_, l_, d_ = shape
            return torch.empty((b_, l_, h_, d_), dtype=dtype).pin_memory().transpose(1, 2)
        return torch.empty(shape, dtype=dtype).pin_memory()

    host_out = {"O": host_empty(O.shape, O.dtype),
                "tau": torch.empty(tau.shape, dtype=tau.dtype).pin_memory()}
    if w.backward:
        for name in ("dQ", "dK", "dV"):
            host_out[name] = host_empty((B, H if name == "dQ" else Hkv, L, D), torch.float32)
    h2d = sum(t.numel() * t.element_size() for t in host_in.values()) + (
        0 if host_km is None else host_km.numel())
    if not w.backward:
        h2d -= host_in["dO"].numel() * host_in["dO"].element_size()
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    e2e_steps = max(3, min(args.steps, 20))
    # The step's batch in chunks, alternating over two streams: each chunk's host-to-device copies,
    # its calls and its device-to-host copies are queued on its stream, so one chunk's copies
    # overlap another's kernels (the two copy directions run on separate engines), and only the
    # first chunk's inputs and the last chunk's outputs cross PCIe with nothing beside them.  A chunk
    # is a run of whole sequences or, with fewer sequences than chunks, a group of heads of one
    # sequence (contiguous in [B, H, L, 64] memory; plain heads only).  Every byte of the step still
    # crosses PCIe inside the timed region.
    target = max(1, args.e2e_chunks)
    if w.B >= target or Hkv != H or args.blhd:
        nb_ = min(w.B, target)
        cuts = [w.B * c // nb_ for c in range(nb_ + 1)]
        chunks = [(cuts[c], cuts[c + 1], 0, H) for c in range(nb_)]
    else:
        ng = min(H, -(-target // w.B))
        hc = [H * g // ng for g in range(ng + 1)]
        chunks = [(b, b + 1, hc[g], hc[g + 1]) for b in range(w.B) for g in range(ng)]
    nchunk = len(chunks)
    e2e_streams = [torch.cuda.Stream(dev) for _ in range(2)]
    bmax = max(c[1] - c[0] for c in chunks)
    hmax = max(c[3] - c[2] for c in chunks)
    e2e_saved = [torch.empty((E.entmax_attn_saved_bytes(bmax, hmax, L, D),), dtype=torch.uint8, device=dev)
                 for _ in e2e_streams]
    e2e_ws = [torch.empty((E.entmax_attn_bwd_saved_workspace_size(bmax, hmax, L, D),), dtype=torch.uint8,
                          device=dev) for _ in e2e_streams]
    rws_bytes = (E.bwd_min_workspace_size(bmax, hmax, L) if args.bwd == "recompute-min"
                 else E.entmax_attn_bwd_workspace_size(bmax, hmax, L, D)) if recompute else 1
    e2e_rws = [torch.empty((max(rws_bytes, 1),), dtype=torch.uint8, device=dev) for _ in e2e_streams]

    def e2e_chunk(b0, b1, h0, h1, k):
        hin = {n: (t[b0:b1] if (h0, h1) == (0, H) else t[b0:b1, h0:h1]) for n, t in host_in.items()}
        Qd = hin["Q"].to(dev, non_blocking=True)
        Kd = hin["K"].to(dev, non_blocking=True)
        Vd = hin["V"].to(dev, non_blocking=True)
        kmd = None if host_km is None else host_km[b0:b1].to(dev, non_blocking=True)
        sv_buf, ws_buf = e2e_saved[k], e2e_ws[k]
        if recompute:
            Oo, to = E.entmax_attn_fwd(Qd, Kd, Vd, kmd, w.causal, w.window, w.scale)
            sv = None
        elif variant:
            r = E.entmax_attn_fwd_ex(Qd, Kd, Vd, kmd, w.causal, w.window, w.scale, alpha=alpha, save=w.backward,
                                     saved=sv_buf if w.backward else None)
            Oo, to, sv = r if w.backward else (r[0], r[1], None)
        elif w.backward:
            Oo, to, sv = E.entmax_attn_fwd_train(Qd, Kd, Vd, kmd, w.causal, w.window, w.scale, saved=sv_buf)
        else:
            Oo, to = E.entmax_attn_fwd(Qd, Kd, Vd, kmd, w.causal, w.window, w.scale)
        host_out["O"][b0:b1, h0:h1].copy_(Oo, non_blocking=True)
        host_out["tau"][b0:b1, h0:h1].copy_(to, non_blocking=True)
        if w.backward:
            dOd = hin["dO"].to(dev, non_blocking=True)
            if recompute:
                g = E.entmax_attn_bwd(Qd, Kd, Vd, to, dOd, kmd, w.causal, w.window, w.scale, workspace=e2e_rws[k])
            elif variant:
                g = E.entmax_attn_bwd_saved_ex(Qd, Kd, Vd, to, sv, dOd, kmd, w.causal, w.window, w.scale, alpha=alpha,
                                               workspace=ws_buf)
            else:
                g = E.entmax_attn_bwd_saved(Qd, Kd, Vd, to, sv, dOd, kmd, w.causal, w.window, w.scale,
                                            workspace=ws_buf)
            for name, t in zip(("dQ", "dK", "dV"), g):
                host_out[name][b0:b1, h0:h1].copy_(t, non_blocking=True)

    def e2e_step(start_event):
        for k, s in enumerate(e2e_streams):
            s.wait_event(start_event)
        for c, (b0, b1, h0, h1) in enumerate(chunks):
            k = c % len(e2e_streams)
            with torch.cuda.stream(e2e_streams[k]):
                e2e_chunk(b0, b1, h0, h1, k)
        for s in e2e_streams:
            stream.wait_stream(s)

    e_warm = torch.cuda.Event()
    e_warm.record(stream)
    e2e_step(e_warm)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(world)
    e0.record(stream)
    for _ in range(e2e_steps):
        e_go = torch.cuda.Event()
        e_go.record(stream)
        e2e_step(e_go)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = dist_max(e0.elapsed_time(e1), world, dev) / e2e_steps
    if E.entmax_attn_device_status() != 0:
        raise RuntimeError("device status after the end-to-end steps")
    link = host_link_rates(dev, stream)

    # the other fwd+bwd workloads the bf16-roofline target covers (L >= 512), timed the same way on
    # every rank (their timing takes the same barriers and max over ranks)
    extras = {}
    if not args.no_extra and not variant and not recompute and not w.fp32_inputs and args.workload == 4:
        peaks = load_peaks()
        extras = {str(k): extra_workload(args, WORKLOADS[k], dev, world, flush, peaks) for k in (3, 5)}
        # softmax attention (alpha = 1, the pages' alpha -> 1 branch) on the headline shape
        extras["softmax_4"] = extra_workload(args, WORKLOADS[4], dev, world, flush, peaks, alpha=1.0)
        # the backward from tau alone on the headline shape: entmax_attn_bwd with its full workspace
        # (support extraction, then the support-list backward), after entmax_attn_fwd
        try:
            rec = extra_workload(argparse.Namespace(**{**vars(args), "bwd": "recompute"}), WORKLOADS[4], dev, world,
                                 flush, peaks)
            rec["backward"] = "entmax_attn_bwd, full workspace (support extraction, then the support-list backward)"
            rec["bwd_vs_saved"] = round(rec["bwd_ms"] / statistics.mean(bwd_ms), 3)
        except Exception as exc:  # recorded, not fatal: the headline line still prints
            rec = {"error": "%s: %s" % (type(exc).__name__, exc)}
        extras["recompute_bwd_4"] = rec

    if rank != 0:
        return None

    # ---- dominant kernel roofline (forward kernel: one launch per entmax_attn_fwd call)
    peaks = load_peaks()
    sparsity = 0.0 if alpha == 1.0 else measured_sparsity(w, Q, K, tau, km)
    supp_pairs = (1.0 - sparsity) * pairs
    fwd_alg_flops = 2.0 * D * pairs + 2.0 * D * supp_pairs
    rows = B * H * L
    # Q, K, V read once, O (bf16) and tau written; the training forward also writes each row's
    # saved support: a count and a (u16 key, fp32 sqrt p) pair per entry
    kv_rows = B * Hkv * L
    fwd_alg_bytes = rows * D * 2 + 2.0 * kv_rows * D * 2 + rows * D * 2 + rows * 4
    if w.backward and not recompute and not tensor_core_backward(w, alpha):
        fwd_alg_bytes += rows * 4 + supp_pairs * 6
    fwd_mean = statistics.mean(fwd_ms)
    bwd_mean = statistics.mean(bwd_ms) if w.backward else 0.0
    ms_per_step = total_ms / args.steps
    # the forward kernel runs for well under a millisecond inside a sub-millisecond step: the burst
    # bf16 figure is its tensor peak
    t_tensor = fwd_alg_flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = fwd_alg_bytes / (peaks["hbm_gbs"] * 1e9)
    fwd_kernel = ("softmax_fwd_kernel" if alpha == 1.0 else
                  "entmax_dense_fwd_kernel" if alpha == 1.5 and tensor_core_backward(w, alpha) else "entmax_fwd_kernel")
    if t_tensor >= t_hbm:
        roof = {"kernel": fwd_kernel, "bound": "tensor",
                "achieved": fwd_alg_flops / (fwd_mean * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "peak_source": "%s bf16 burst (MEASURED_PEAKS.json)" % peaks["source"]}
    else:
        roof = {"kernel": fwd_kernel, "bound": "hbm",
                "achieved": fwd_alg_bytes / (fwd_mean * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "peak_source": "%s HBM copy (MEASURED_PEAKS.json)" % peaks["source"]}
    roof.update({"traffic": None, "algorithmic_flops_per_launch": fwd_alg_flops,
                 "algorithmic_bytes_per_launch": fwd_alg_bytes})
    roof["frac"] = roof["achieved"] / roof["peak"]
    tr = ROOT / "profiles" / ("traffic_workload%d.txt" % w.wid)
    if tr.exists() and not variant:
        t = json.loads(tr.read_text())
        if t.get("kernel") == fwd_kernel and t.get("source_hash") == source_hash(fwd_kernel):
            roof["traffic"] = t["bytes_per_launch"]

    step_roof = step_roofline(w, km, flops, ms_per_step, peaks)
    value = aggregate_value(flops, world, ms_per_step)
    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded i.i.d. N(0,1), bf16; stands in for GLUE SST-2 batches)",
        "config": {
            "workload": workload_desc(w),
            "workload_id": w.wid,
            "allowed_pairs": pairs,
            "dense_equiv_gflop_per_step": flops / 1e9,
            "dense_equiv_gflop_full_L2": dense_equiv_flops(w, w.B * w.H * w.L * w.L) / 1e9,
            "l2": "evicted before each timed step, outside its events: 256 MiB written, then another 256 MiB read "
                  "(L2 left holding clean lines)",
            "parallelism": "replicas" if world > 1 else "single GPU",
        },
        "variant": {"alpha": alpha, "H_kv": Hkv, "layout": "BLHD" if args.blhd else "BHLD",
                    "inputs": "fp32 (rounded to bf16 on the device)" if w.fp32_inputs else "bf16"}
        if variant or w.fp32_inputs else None,
        "backward": ("entmax_attn_bwd" if recompute else "entmax_attn_bwd_saved") + (
            " (tensor-core kernels: scores recomputed, every product on tcgen05)" if tensor_core_backward(w, alpha)
            else " (recompute kernels: minimum workspace)" if args.bwd == "recompute-min"
            else " (supports listed from tau by one score pass, then the support-list backward)" if recompute
            else " (saved supports)"),
        "fwd_ms": round(fwd_mean, 4),
        "bwd_ms": round(bwd_mean, 4),
        "step_ms_median": round(statistics.median(step_ms), 4),
        "wall_ms_per_step_incl_flush": round(wall * 1e3 / args.steps, 4),
        "sparsity": round(sparsity, 4),
        "roofline": roof,
        "step_roofline": step_roof,
        "gpu_launches": launches_per_step(w, recompute, alpha, args.bwd == "recompute-min") * args.steps,
        "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "chunks": "%d chunks (%s) on 2 streams (copies overlap kernels)" % (
                    nchunk, "whole sequences" if chunks[0][2:] == (0, H) else "head groups of one sequence"),
                "host_link": link_bound(link, h2d, d2h, e2e_ms)},
        "clocks": clocks,
    }
    if extras:
        out["workloads"] = extras
    if world == 1 and not args.no_cpu_baseline:
        cb = oracle_baseline(w, inp, budget_s=args.cpu_seconds, alpha=alpha)
        out["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        cb1 = oracle_baseline(w, inp, budget_s=args.cpu_seconds / 3, max_heads=8, alpha=alpha, threads=1)
        out["cpu_baseline_1thread"] = {k: cb1[k] for k in ("value", "unit", "cores", "kind", "sample")}
    return out


# The source files each profiled kernel is built from: a committed traffic figure counts only while
# the hash of its kernel's files is the one it was captured at.
KERNEL_SOURCES = {
    "entmax_fwd_kernel": ("fwd.cu", "tau15.cuh", "common.cuh", "ptx.cuh", "internal.h"),
    "softmax_fwd_kernel": ("fwd_softmax.cu", "dense.cuh", "common.cuh", "ptx.cuh", "internal.h"),
    "entmax_dense_fwd_kernel": ("fwd_dense.cu", "tau15.cuh", "dense.cuh", "common.cuh", "ptx.cuh", "internal.h"),
}


def source_hash(kernel: str | None = None) -> str:
    """sha256 (16 hex digits) of the kernel's source files, or of every file under csrc/."""
    import hashlib

    csrc = ROOT / "entmax_tcgen05_tma_b200" / "csrc"
    files = [csrc / f for f in KERNEL_SOURCES[kernel]] if kernel else sorted(csrc.glob("*"))
    h = hashlib.sha256()
    for p in files:
        h.update(p.read_bytes())
    return h.hexdigest()[:16]


def bench_workload(args) -> Workload:
    w = WORKLOADS[args.workload]
    if args.hkv:
        if args.hkv < 1 or w.H % args.hkv:
            raise SystemExit("--hkv must divide the workload's %d heads" % w.H)
        w = w.with_shape(H_kv=args.hkv)
    if getattr(args, "fp32_inputs", False):
        w = w.with_shape(fp32_inputs=True)
    return w


def run_reference(args) -> dict:
    w = bench_workload(args)
    inp = make_inputs(w)
    per = []
    cb = None
    for k in range(args.warmup + args.steps):
        cb = oracle_baseline(w, inp, budget_s=args.ref_step_seconds, max_heads=1 if k < args.warmup else 64,
                             alpha=args.alpha)
        if k >= args.warmup:
            per.append(cb)
    secs = sum(c["seconds"] for c in per)
    value = sum(c["value"] * c["seconds"] for c in per) / secs
    pairs = allowed_pairs(w, inp["key_mask"])
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": args.gpus,  # the launch's N; the oracle itself runs on host cores only
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * dense_equiv_flops(w, pairs) / (value * 1e12), 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded i.i.d. N(0,1), bf16-rounded)",
        "config": {"workload": workload_desc(w), "workload_id": w.wid,
                   "note": "each step times the fp64 CPU oracle on a bounded sample of whole heads; "
                           "ms_per_step extrapolates to the full workload; no GPU is used"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cb["cores"], "kind": "oracle",
                         "sample": "%d steps, each %s" % (args.steps, per[-1]["sample"])},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- dist helpers
def aggregate_value(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: the work of all ranks over the (max over ranks) step time."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def dist_barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def dist_max(x: float, world: int, dev) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=4, choices=[2, 3, 4, 5])
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=8.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the selected workload (the default workload-4 line also times 3 and 5)")
    ap.add_argument("--alpha", type=float, default=1.5, help="alpha-entmax variant, alpha in [1, 2] (1: softmax)")
    ap.add_argument("--hkv", type=int, default=0, help="grouped-query variant: key/value heads")
    ap.add_argument("--blhd", action="store_true", help="variant: tensors in [B, L, H, 64] memory")
    ap.add_argument("--fp32-inputs", action="store_true",
                    help="variant: Q, K, V, dO given as fp32 (the library rounds them to bf16 on the device)")
    ap.add_argument("--e2e-chunks", type=int, default=4,
                    help="end-to-end step: chunks of the batch whose copies overlap other chunks' kernels")
    ap.add_argument("--bwd", default="saved", choices=["saved", "recompute", "recompute-min"],
                    help="backward path: from the forward's saved supports, or entmax_attn_bwd with its full "
                         "workspace (long rows list their supports from tau) or with the minimum one (recompute kernels)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if not (args.alpha == 1.0 or 1.0 < args.alpha <= 2.0):
        ap.error("--alpha must be 1 (softmax) or lie in (1, 2]")
    if args.bwd != "saved" and (args.alpha != 1.5 or args.hkv or args.blhd):
        ap.error("--bwd recompute takes the plain path only (alpha 1.5, H_kv = H, [B, H, L, 64])")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        out = run_gpu(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
