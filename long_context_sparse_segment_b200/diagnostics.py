"""Attention-coverage and block-density diagnostics ("Sparser Block-Sparse
Attention via Token Permutation", sciencestack.ai Figure 2 caption and
Figure 4; gist.science summary, "Experimentelle Ergebnisse", Sparsity).

For a workload, with and without the segment-local permutation: the exact
attention mass of every (query block, key block) pair (pbs_block_mass),
the coverage of the block lists the selection keeps, and the fewest blocks
that reach a target coverage (pbs_coverage). Density is a block count over
the dense-causal block count, as for the path.
"""
from __future__ import annotations

import ctypes

import torch

from . import ops
from ._lib import check, lib


def block_mass(q, k_perm, kpos, block, segment, scale=0.0):
    """[b, hq, nb, nb] fp32: the attention mass of each (query block, key
    block) pair; kpos None is the unpermuted sequence."""
    b, hq, n, d = q.shape
    shp = ops.shape_of(q, k_perm, block, segment)
    mass = torch.empty(b, hq, n // block, n // block, dtype=torch.float32, device=q.device)
    check(lib().pbs_block_mass(ops._ptr(q), ops._ptr(k_perm), ops._ptr(kpos), ops._ptr(mass),
                               shp, scale, ops._stream(q.device)), "pbs_block_mass")
    return mass


def coverage(mass, shape, idx=None, cnt=None, target=None):
    """(coverage [b, hq, nb] fp32 of the lists, or None; blocks needed for
    `target` [b, hq, nb] int32, or None)."""
    b, hq, nb, _ = mass.shape
    cov = torch.empty(b, hq, nb, dtype=torch.float32, device=mass.device) if idx is not None else None
    need = (torch.empty(b, hq, nb, dtype=torch.int32, device=mass.device)
            if target is not None else None)
    check(lib().pbs_coverage(ops._ptr(mass), ops._ptr(idx), ops._ptr(cnt),
                             ctypes.c_double(target if target is not None else 1.0),
                             ops._ptr(cov), ops._ptr(need), shape, ops._stream(mass.device)),
          "pbs_coverage")
    return cov, need


def report(q, k, v, block, segment, mode, param, target=0.975, scale=0.0):
    """Coverage and density of the selection, and the density an ideal
    selection needs for `target` coverage, with and without permutation."""
    b, hq, n, d = q.shape
    nb = n // block
    dense = b * hq * nb * (nb + 1) / 2
    shp = ops.shape_of(q, k, block, segment)
    res = ops.pbs_attention(q, k, v, block, segment, mode, param, scale, keep=True)
    m_perm = block_mass(q, res["k_perm"], res["kpos"], block, segment, scale)
    cov, need_perm = coverage(m_perm, shp, res["idx"], res["cnt"], target)
    m_nat = block_mass(q, k, None, block, segment, scale)
    _, need_nat = coverage(m_nat, shp, target=target)
    # the same selection rule on the unpermuted sequence
    idx0, cnt0, _ = ops.select_blocks(q, k, None, block, segment, mode, param, scale)
    cov0, _ = coverage(m_nat, shp, idx0, cnt0)
    out = {
        "selection": f"{mode} {param}",
        "coverage_perm": float(cov.double().mean()),
        "density_perm": float(res["cnt"].double().sum()) / dense,
        "coverage_noperm": float(cov0.double().mean()),
        "density_noperm": float(cnt0.double().sum()) / dense,
        "target_coverage": target,
        "ideal_density_perm": float(need_perm.double().sum()) / dense,
        "ideal_density_noperm": float(need_nat.double().sum()) / dense,
    }
    out["ideal_block_reduction"] = 1.0 - out["ideal_density_perm"] / out["ideal_density_noperm"]
    return out


def _main():
    import argparse
    import json

    from .workloads import WORKLOADS, make_inputs

    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--config", default="llama32k", choices=sorted(WORKLOADS))
    ap.add_argument("--target", type=float, default=0.975)
    ap.add_argument("--strength", type=float, default=None,
                    help="planted-key strength (K += strength * u) instead of the workload's")
    args = ap.parse_args()
    w = WORKLOADS[args.config]
    if args.strength is not None:
        w = w.with_(strength=args.strength)
    dev = torch.device("cuda", 0)
    q, k, v, _ = make_inputs(w, dev)
    out = {"workload": w.name, "strength": w.strength, **report(q, k, v, w.block, w.segment, w.mode, w.param,
                                       args.target)}
    # time the block-mass pass on the permuted keys (tensor work: two QK
    # products per admissible (head, key block) pair)
    res = ops.pbs_attention(q, k, v, w.block, w.segment, w.mode, w.param, keep=True)
    block_mass(q, res["k_perm"], res["kpos"], w.block, w.segment)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    block_mass(q, res["k_perm"], res["kpos"], w.block, w.segment)
    e1.record()
    torch.cuda.synchronize()
    nb, spb = w.n // w.block, w.segment // w.block
    pairs = w.batch * w.hq * sum(min(nb, (i // spb + 1) * spb) for i in range(nb))
    ms = e0.elapsed_time(e1)
    out["block_mass_ms"] = round(ms, 3)
    out["block_mass_tflops"] = round(2 * 2.0 * w.block * w.block * w.d * pairs / ms / 1e9, 1)
    out["status"] = ops.device_status()
    print(json.dumps(out))


if __name__ == "__main__":
    _main()
