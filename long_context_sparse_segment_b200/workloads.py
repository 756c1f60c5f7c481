"""Seeded synthetic inputs for the permuted block-sparse attention prefill path.

This module only draws random tensors: it holds none of the method's
arithmetic, so that both the CPU oracle (test infrastructure) and the CUDA
path can be fed from it.

The real workloads of "Sparser Block-Sparse Attention via Token Permutation"
(LongBench / LongBenchv2 prompts through Llama-3.1-8B, Experiments section)
are not available, so these tensors stand in for them. They have the
attention shape of Llama-3.1-8B (32 query heads, 8 KV heads, head dim 128)
and a planted structure of "heavy hitter" keys, the kind of structure the
method's key permutation is meant to cluster (gist.science summary,
"Globale-Importanz-basierte Key-Permutation").

Recipe, per (batch, KV head), with one ``torch.Generator`` seeded once:

1. Q, K, V drawn in that order as fp32 N(0, 1).
2. u drawn as fp32 N(0, I) per (batch, KV head), scaled to unit length.
3. Salient key positions (see ``Workload.salient``).
4. K[salient] += 3 u; every query of the KV head's group gets Q += u.
5. Q, K, V rounded to bf16.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    hq: int
    hkv: int
    n: int
    d: int
    block: int      # B: block size of the block-sparse attention
    segment: int    # S: permutation segment size
    mode: str       # "threshold" | "topk_frac" | "all" | "dense_causal"
    param: float    # tau for threshold, fraction for topk_frac
    salient: str    # "uniform" | "per_segment" | "bursts"
    salient_rate: float
    layers: int = 1
    seed: int = 0
    burst: int = 16
    strength: float = 3.0  # planted keys get K += strength * u

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def nb(self) -> int:
        return self.n // self.block

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # 1 head, N=1024, d=64, 5% planted keys uniform over the sequence.
    "tiny": Workload("tiny", 1, 1, 1, 1024, 64, 64, 256, "threshold", 0.9,
                     "uniform", 0.05),
    # Llama-3.1-8B attention shape at 8K, 2% planted keys per segment.
    "llama8k": Workload("llama8k", 1, 32, 8, 8192, 128, 128, 1024, "threshold",
                        0.9, "per_segment", 0.02),
    # 32K, planted keys in bursts of 16 contiguous tokens.
    "llama32k": Workload("llama32k", 1, 32, 8, 32768, 128, 128, 2048,
                         "threshold", 0.9, "bursts", 0.02),
    # 128K, fixed top-k of 25% of the causal key blocks per query block.
    "llama128k": Workload("llama128k", 1, 32, 8, 131072, 128, 128, 4096,
                          "topk_frac", 0.25, "per_segment", 0.02),
    # Longer contexts with the 128K recipe (the pages name 256K and 512K as
    # the lengths of their largest speedups, without a selection setting).
    "llama256k": Workload("llama256k", 1, 32, 8, 262144, 128, 128, 4096,
                          "topk_frac", 0.25, "per_segment", 0.02),
    "llama512k": Workload("llama512k", 1, 32, 8, 524288, 128, 128, 4096,
                          "topk_frac", 0.25, "per_segment", 0.02),
    # 32 independent layers at 64K, batch 2; layer l is seeded with l.
    "stack64k": Workload("stack64k", 2, 32, 8, 65536, 128, 128, 2048,
                         "threshold", 0.9, "per_segment", 0.02, layers=32),
}


def salient_mask(w: Workload, gen: torch.Generator, device) -> torch.Tensor:
    """Boolean [batch, hkv, n] marking the planted heavy-hitter keys."""
    b, h, n = w.batch, w.hkv, w.n
    mask = torch.zeros(b, h, n, dtype=torch.bool, device=device)
    if w.salient == "uniform":
        count = round(w.salient_rate * n)
        order = torch.rand(b, h, n, generator=gen, device=device).argsort(-1)
        mask.scatter_(-1, order[..., :count], True)
    elif w.salient == "per_segment":
        nseg = n // w.segment
        count = round(w.salient_rate * w.segment)
        order = torch.rand(b, h, nseg, w.segment, generator=gen,
                           device=device).argsort(-1)[..., :count]
        base = (torch.arange(nseg, device=device) * w.segment).view(1, 1, nseg, 1)
        mask.scatter_(-1, (order + base).reshape(b, h, -1), True)
    elif w.salient == "bursts":
        count = round(w.salient_rate * n / w.burst)
        starts = torch.randint(0, n - w.burst + 1, (b, h, count), generator=gen,
                               device=device)
        pos = starts.unsqueeze(-1) + torch.arange(w.burst, device=device)
        mask.scatter_(-1, pos.reshape(b, h, -1), True)
    else:
        raise ValueError(f"unknown salient structure {w.salient!r}")
    return mask


def make_inputs(w: Workload, device="cpu", layer: int = 0, seed: int | None = None):
    """Draw (q, k, v) as bf16 tensors [batch, heads, n, d] on ``device``.

    The seed is ``w.seed + layer`` unless given. Draws happen on ``device``
    with a generator of that device, so CPU and CUDA draws differ but each is
    reproducible.
    """
    device = torch.device(device)
    s = (w.seed + layer) if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(s)
    shp_q = (w.batch, w.hq, w.n, w.d)
    shp_kv = (w.batch, w.hkv, w.n, w.d)
    q = torch.randn(shp_q, generator=gen, device=device, dtype=torch.float32)
    k = torch.randn(shp_kv, generator=gen, device=device, dtype=torch.float32)
    v = torch.randn(shp_kv, generator=gen, device=device, dtype=torch.float32)
    u = torch.randn(w.batch, w.hkv, w.d, generator=gen, device=device,
                    dtype=torch.float32)
    u = u / u.norm(dim=-1, keepdim=True)
    sal = salient_mask(w, gen, device)
    k += w.strength * sal.unsqueeze(-1).float() * u.unsqueeze(2)
    q += u.repeat_interleave(w.group, dim=1).unsqueeze(2)
    out = (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))
    del q, k, v
    return out + (sal,)
