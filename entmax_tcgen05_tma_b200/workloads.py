"""Seeded synthetic workloads for 1.5-entmax attention.

This module draws inputs only; it holds none of the method's arithmetic.  Both
the CUDA path (through the binding) and the fp64 oracle are fed from here.

The five workloads stand in for the GLUE/SST-2 evaluations the AdaSplash
pages measure on (model cards "roberta-base-adasplash" and
"distilbert-sst2-adasplash", empirical table: L=128, B=32, 12 heads of 64),
plus a long-context and a causal sliding-window decoder case.  Inputs are
i.i.d. N(0,1) drawn in fp32 from ``torch.Generator('cpu').manual_seed(1000+k)``
and rounded to bf16 (workload 1 stays fp32 at the library boundary).  Draw
order: Q, K, V, dO, lengths.  Key padding is right padding:
``mask[b, j] = j < len_b`` with ``len_b ~ U[lo, hi]``.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    B: int
    H: int
    L: int
    D: int
    scale: float
    causal: bool = False
    window: int = 0
    len_range: tuple[int, int] | None = None  # key-padding valid length U[lo, hi]
    backward: bool = True
    fp32_inputs: bool = False
    H_kv: int | None = None  # key/value heads (grouped-query attention); None: H

    @property
    def kv_heads(self) -> int:
        return self.H if self.H_kv is None else self.H_kv

    def with_shape(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: dict[int, Workload] = {
    1: Workload(1, "oracle-scale forward, fp32 inputs", 1, 2, 64, 64, 1.0 / 8, backward=False, fp32_inputs=True),
    2: Workload(2, "RoBERTa-base-shaped encoder forward, key padding", 32, 12, 128, 64, 1.0 / 8,
                len_range=(16, 128), backward=False),
    3: Workload(3, "DistilBERT-shaped encoder fwd+bwd, key padding", 32, 12, 512, 64, 1.0 / 8,
                len_range=(64, 512)),
    4: Workload(4, "long-context encoder fwd+bwd, temperature 2", 4, 12, 4096, 64, 2.0 / 8),
    5: Workload(5, "GPT-2-small-shaped decoder fwd+bwd, causal + window 32", 8, 12, 1024, 64, 1.0 / 8,
                causal=True, window=32),
}


def make_inputs(w: Workload, seed: int | None = None) -> dict:
    """Draw the workload's tensors on the CPU.

    Returns a dict with Q, dO [B,H,L,D] and K, V [B,H_kv,L,D] (bf16, or fp32 for fp32-input workloads),
    ``lengths`` (int64 [B] or None) and ``key_mask`` (uint8 [B, L] or None).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(1000 + w.wid if seed is None else seed)
    dt = torch.float32 if w.fp32_inputs else torch.bfloat16
    out = {}
    for name in ("Q", "K", "V", "dO"):
        heads = w.kv_heads if name in ("K", "V") else w.H
        out[name] = torch.randn((w.B, heads, w.L, w.D), generator=gen, dtype=torch.float32).to(dt)
    if w.len_range is not None:
        lo, hi = w.len_range
        lengths = torch.randint(lo, hi + 1, (w.B,), generator=gen, dtype=torch.int64)
        mask = (torch.arange(w.L).unsqueeze(0) < lengths.unsqueeze(1)).to(torch.uint8)
        out["lengths"] = lengths
        out["key_mask"] = mask.contiguous()
    else:
        out["lengths"] = None
        out["key_mask"] = None
    return out

