#!/usr/bin/env python
"""Benchmark of the permuted block-sparse attention (PBS-Attn) prefill path.

One step = the whole path over one synthetic input (every layer of it):
importance scoring, segment-local permutation, block selection and the
block-sparse forward (the inverse permutation is a no-op in the default
natural-query mode). Inputs are resident in HBM before timing and larger
than L2. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Under torchrun every rank runs its own replica of the workload (the units of
the path are independent per batch and head, so there is no collective on the
data path): weak scaling, value = all ranks' work / the slowest rank's time.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import long_context_sparse_segment_b200 as pbs  # noqa: E402
from long_context_sparse_segment_b200._lib import OP_HOST_PATH  # noqa: E402
from long_context_sparse_segment_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "PBS-Attn prefill ms and effective TFLOP/s (% BF16 peak) at N=32K–128K vs dense"
UNIT = "TFLOP/s"
L2_BYTES = 126 << 20  # B200
LAUNCHES_PER_LAYER = 9  # score 3, permute 2, select 3 (pooling, scores, lists), forward 1
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="llama128k", choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: every rank runs the whole workload (weak scaling), or "
                         "the KV groups of one workload are split over the ranks (strong)")
    ap.add_argument("--queries", choices=["natural", "fused", "separate"], default="natural",
                    help="natural query order (the default path), or queries permuted with "
                         "the keys and the inverse permutation fused into the forward's "
                         "epilogue or run as its own step")
    ap.add_argument("--gather-output", choices=["none", "nccl", "fused"], default="none",
                    help="with --shard heads on N > 1 GPUs: the whole output on every rank, "
                         "inside the timed step, by an NCCL all-gather after the forward or "
                         "by the forward itself writing into every rank's buffer "
                         "(pbs_attn_fwd_bcast over symmetric memory)")
    ap.add_argument("--gather-kv", action="store_true",
                    help="the forward reads K, V through the key order (pbs_attn_fwd_gather); "
                         "the permutation writes only the order and block sums")
    ap.add_argument("--block", type=int, choices=[64, 128], default=None,
                    help="the workload with another block size B (the method's free "
                         "parameter; its segment size and selection unchanged)")
    ap.add_argument("--graph", action="store_true",
                    help="capture each layer's step as one CUDA graph after the warm-up and "
                         "replay it in the timed region: the same kernels without the host's "
                         "per-launch overhead, which bounds the small configs")
    ap.add_argument("--profile", action="store_true",
                    help="time the steps only (no dense, end-to-end or CPU legs), for ncu")
    return ap.parse_args()


def workload_of(args):
    w = WORKLOADS[args.config]
    if args.block and args.block != w.block:
        w = w.with_(name=f"{w.name}_b{args.block}", block=args.block)
    return w


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


RANK_SEED_STRIDE = 1000  # rank r draws its replica's inputs with seed + 1000 r


def rank_seed_offset(rank):
    return RANK_SEED_STRIDE * rank


def shard_heads(w, rank, world):
    """The rank's share of one sequence when the KV groups are split over the
    ranks (the path is independent per KV group, so no data crosses ranks):
    KV heads [rank * hkv / world, (rank + 1) * hkv / world) with their query
    heads. Returns (workload of the share, first KV head)."""
    if w.hkv % world:
        raise ValueError(f"{w.hkv} KV heads do not split over {world} ranks")
    per = w.hkv // world
    return w.with_(hkv=per, hq=per * w.group), rank * per


def gather_heads(o_local, dist, world, out=None):
    """With the KV groups split over the ranks, each rank holds the output of
    its own query heads, [b, hq / world, n, d]; this all-gathers them into
    the whole output [b, hq, n, d] on every rank (one collective, NCCL over
    NVLink on GPUs; gloo on the CPU in the tests). Rank r's heads come r-th,
    as shard_heads assigns them."""
    b, h, n, d = o_local.shape
    parts = torch.empty((world * b, h, n, d), dtype=o_local.dtype, device=o_local.device)
    dist.all_gather_into_tensor(parts, o_local.contiguous())  # rank r's slice r-th
    full = parts.view(world, b, h, n, d).permute(1, 0, 2, 3, 4).reshape(b, world * h, n, d)
    if out is not None:
        out.copy_(full)
        return out
    return full


def job_throughput(flops_rank, ms_rank, dist=None, device="cpu"):
    """Whole-job TFLOP/s: the flops of all ranks over the slowest rank's time.

    Returns (TFLOP/s, slowest ms, total flops). Every rank must call it (it
    holds two collectives when dist is given)."""
    if dist is None:
        return flops_rank / (ms_rank * 1e-3) / 1e12, ms_rank, flops_rank
    t = torch.tensor([ms_rank], dtype=torch.float64, device=device)
    f = torch.tensor([flops_rank], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(f, op=dist.ReduceOp.SUM)
    ms, flops = float(t.item()), float(f.item())
    return flops / (ms * 1e-3) / 1e12, ms, flops


def block_flops(w, total_blocks):
    return 4.0 * w.block * w.block * w.d * total_blocks


# ------------------------------------------------------------------ clocks
REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x2: "applications_clocks_setting", 0x1: "gpu_idle"}


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while timing."""

    def __init__(self, device):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", ident, "--query-gpu=clocks.sm,clocks.max.sm,power.draw,"
                 "clocks_event_reasons.active", "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 4:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                    mask = int(parts[3], 16)
                except ValueError:
                    continue
                for bit, name in REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- GPU arm
class Layer:
    def __init__(self, w, dev, layer, seed_offset, gather_kv=False, queries="natural"):
        self.w = w
        self.gather_kv = gather_kv  # the forward reads K, V through the key order
        # "natural", or permuted queries with the inverse permutation "fused"
        # into the forward or run as its own step ("separate")
        self.queries = queries
        self.q, self.k, self.v, _ = make_inputs(w, dev, layer=layer, seed=w.seed + layer + seed_offset)
        self.out = None
        self.o_perm = None
        # (output buffers of every rank, this rank's index, first head): the
        # forward writes its heads into all of them (pbs_attn_fwd_bcast)
        self.bcast = None


def run_layer(layer, ev=None):
    """The five steps on one layer; returns (o, blk_cnt). ev: dict of event
    pairs recorded around score / permute / select / forward / unpermute."""
    w = layer.w
    B, S = w.block, w.segment
    permuted_q = layer.queries != "natural"

    def mark(name, i):
        if ev is not None:
            ev[name][i].record()

    mark("score", 0)
    imp = pbs.score(layer.q, layer.k, B, S)
    mark("score", 1)
    mark("permute", 0)
    perm = pbs.permute(imp, layer.k, layer.v, B, S, q=layer.q if permuted_q else None, hq=w.hq,
                       materialize=not layer.gather_kv)
    mark("permute", 1)
    q_used = perm["q_perm"] if permuted_q else layer.q
    qpos = perm["kpos"] if permuted_q else None
    mark("select", 0)
    idx, cnt, _ = pbs.select_blocks(q_used, perm["k_perm"], perm["kbar_sum"], B, S, w.mode,
                                    w.param)
    mark("select", 1)
    fused = layer.queries == "fused"
    mark("attn", 0)
    if layer.bcast is not None:
        outs, me, first_head = layer.bcast
        pbs.attn_fwd_bcast(q_used, perm["k_perm"], perm["v_perm"], perm["kpos"], idx, cnt, B, S,
                           outs, head_offset=first_head)
        o = outs[me]
    elif layer.gather_kv:
        o = pbs.attn_fwd_gather(q_used, layer.k, layer.v, perm["kpos"], qpos, idx, cnt, B, S,
                                out=layer.o_perm if layer.queries == "separate" else layer.out,
                                unpermute=fused)
    else:
        fwd_out = layer.o_perm if layer.queries == "separate" else layer.out
        o = pbs.attn_fwd(q_used, perm["k_perm"], perm["v_perm"], perm["kpos"], qpos, idx, cnt,
                         B, S, out=fwd_out, unpermute=fused)
    mark("attn", 1)
    mark("unpermute", 0)
    if layer.queries == "separate":
        layer.o_perm = o
        o = pbs.unpermute(o, qpos, w.hkv, B, S, out=layer.out)
    mark("unpermute", 1)
    layer.out = o
    return o, cnt


def time_dense(layer, reps=3):
    """Plain causal attention (identity order, blocks J <= I) on the same
    forward kernel, for the speedup."""
    w = layer.w
    idx, cnt, _ = pbs.select_blocks(layer.q, layer.k, None, w.block, w.segment, "dense_causal")
    for _ in range(2):
        pbs.attn_fwd(layer.q, layer.k, layer.v, None, None, idx, cnt, w.block, w.segment,
                     out=layer.out)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        pbs.attn_fwd(layer.q, layer.k, layer.v, None, None, idx, cnt, w.block, w.segment,
                     out=layer.out)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps, float(cnt.sum().item())


def e2e_run(w, layers, steps):
    """The same metric through the public call on host buffers
    (pbs_attention_host): every step copies each layer's inputs from
    page-locked host memory and its output back, the copies overlapped with
    the compute one KV group at a time; the timed region covers the copies."""
    host = []
    for L in layers:
        host.append(tuple(t.cpu().pin_memory() for t in (L.q, L.k, L.v)))
    o_host = torch.empty(layers[0].q.shape, dtype=torch.bfloat16).pin_memory()
    dev = layers[0].q.device
    ws = torch.empty(max(16, pbs.workspace_bytes(pbs.shape_of(layers[0].q, layers[0].k, w.block,
                                                              w.segment), OP_HOST_PATH)),
                     dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host[0]) * len(layers)
    d2h = o_host.numel() * o_host.element_size() * len(layers)

    def one():
        for hq_, hk_, hv_ in host:
            pbs.attention_host(hq_, hk_, hv_, w.block, w.segment, w.mode, w.param, out=o_host,
                               device=dev, ws=ws)

    one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, h2d, d2h


def gpu_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    w = workload_of(args)
    sharded = args.shard == "heads" and world > 1
    w_full = w
    if sharded:
        # one sequence: rank r draws the inputs of its own KV groups
        w, first = shard_heads(w, rank, world)
        seed_offset = first
    else:
        seed_offset = rank_seed_offset(rank)
    layers = [Layer(w, dev, l, seed_offset=seed_offset, gather_kv=args.gather_kv,
                    queries=args.queries) for l in range(w.layers)]
    torch.cuda.synchronize()

    gathering = args.gather_output if sharded else "none"
    if gathering == "fused":
        # every rank's whole-output buffer, mapped into every rank (symmetric
        # memory: plain peer stores, no multicast); each rank's forward
        # writes its heads into all of them
        if args.queries != "natural" or args.gather_kv:
            raise SystemExit("--gather-output fused runs the natural-order path only")
        import torch.distributed._symmetric_memory as symm_mem
        shape = (w_full.batch, w_full.hq, w_full.n, w_full.d)
        mine = symm_mem.empty(shape, dtype=torch.bfloat16, device=dev)
        hdl = symm_mem.rendezvous(mine, dist.group.WORLD.group_name)
        peers = [hdl.get_buffer(r, shape, torch.bfloat16) for r in range(world)]
        for L in layers:
            L.bcast = (peers, rank, first * w.group)
        step_done = torch.zeros(1, device=dev)

    def step_layer(L, ev=None):
        o, cnt = run_layer(L, ev)
        if ev is not None:
            ev["gather"][0].record()
        if gathering == "nccl":  # the whole output on every rank
            gather_heads(o, dist, world)
        elif gathering == "fused":  # every rank's stores have landed
            dist.all_reduce(step_done)
        if ev is not None:
            ev["gather"][1].record()
        return o, cnt

    # warm-up (also fixes the kept-block counts of this input)
    for _ in range(max(3, args.warmup)):
        total_blocks = 0.0
        for L in layers:
            _, cnt = step_layer(L)
            total_blocks += float(cnt.sum().item())
    flops_per_step = block_flops(w, total_blocks)

    names = ("score", "permute", "select", "attn", "unpermute", "gather")
    graphs = None
    if args.graph:
        if gathering != "none":
            raise SystemExit("--graph runs the path without --gather-output")
        # one graph per layer, with event-record nodes around its steps
        # (external events: replays record them, read after each step)
        gevs = [{n: (torch.cuda.Event(enable_timing=True, external=True),
                     torch.cuda.Event(enable_timing=True, external=True)) for n in names}
                for _ in layers]
        graphs = []
        for L, ge in zip(layers, gevs):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step_layer(L, ge)
            graphs.append(g)
        for g in graphs:
            g.replay()
        torch.cuda.synchronize()
    evs = [{n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for n in names} for _ in range(0 if graphs else args.steps * len(layers))]
    # inputs that fit in L2 (the small configs) would stay there from one
    # step to the next: then each step is timed on its own and a 256 MB
    # write between steps, outside the timed events, flushes L2
    input_bytes = sum(t.numel() * t.element_size() for L in layers for t in (L.q, L.k, L.v))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) \
        if input_bytes < 2 * L2_BYTES else None
    marks = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    per_sum = {n: 0.0 for n in names}
    i = 0
    for k in range(args.steps):
        if flush is not None:
            flush.fill_(k & 0xff)
        marks[k][0].record()
        if graphs is None:
            for L in layers:
                step_layer(L, evs[i])
                i += 1
        else:
            for g in graphs:
                g.replay()
        marks[k][1].record()
        if graphs is not None:  # the graphs' events hold this step's times
            torch.cuda.synchronize()
            for ge in gevs:
                for n in names:
                    per_sum[n] += ge[n][0].elapsed_time(ge[n][1])
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    if dist:
        dist.barrier()
    if flush is None and graphs is None:  # back to back: the whole region
        ms = marks[0][0].elapsed_time(marks[-1][1]) / args.steps
    else:  # each step bracketed by its own events
        ms = sum(a.elapsed_time(b) for a, b in marks) / args.steps
    if graphs is None:
        per_sum = {n: sum(e[n][0].elapsed_time(e[n][1]) for e in evs) for n in names}
    per = {n: v / args.steps for n, v in per_sum.items()}
    attn_launch_ms = per["attn"] / len(layers)
    value, ms, _ = job_throughput(flops_per_step, ms, dist, dev)
    pk, pk_kind = peaks()
    # the burst GEMM figure for a forward timed in steps of well under a
    # second; the sustained one (a seconds-long loop under the power cap) for
    # steps of a second or more, such as the 32-layer stack
    long_step = ms >= 1000.0
    peak_burst = pk.get("bf16_tflops", pk.get("bf16_tflops_sustained"))
    peak_sust = pk.get("bf16_tflops_sustained", peak_burst)
    peak = peak_sust if long_step else peak_burst
    attn_tflops = flops_per_step / len(layers) / (attn_launch_ms * 1e-3) / 1e12

    if args.profile:
        dense_ms, dense_blocks, e2e_ms, h2d, d2h = float("nan"), float("nan"), float("nan"), 0, 0
    else:
        dense_ms, dense_blocks = time_dense(layers[0])
        e2e_ms, h2d, d2h = e2e_run(w, layers, max(1, args.e2e_steps))
    e2e_value, e2e_ms, _ = job_throughput(flops_per_step, e2e_ms, dist, dev)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "strong" if sharded else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 with planted salient keys)",
        "config": {"workload": w.name, "batch": w.batch, "hq": w_full.hq, "hkv": w_full.hkv,
                   "n": w.n,
                   "d": w.d, "block": w.block, "segment": w.segment, "layers": w.layers,
                   "selection": f"{w.mode} {w.param}",
                   "l2": ("flushed between steps (256 MB write)" if flush is not None
                          else "inputs larger than L2"),
                   "parallelism": (f"heads/{world}" + {"none": "", "nccl": " + NCCL all-gather of O",
                                                        "fused": " + O written to every rank by "
                                                                 "the forward"}[gathering])
                   if sharded else f"replicas x{world}",
                   "kv": "gathered inside the forward" if args.gather_kv else "permuted copies",
                   "queries": {"natural": "natural order",
                               "fused": "permuted, inverse fused into the forward",
                               "separate": "permuted, inverse as its own step"}[args.queries],
                   **({"launch": "one CUDA graph per layer, replayed"} if graphs else {})},
        "density": round(total_blocks / (len(layers) * w.batch * w.hq * w.nb * (w.nb + 1) / 2), 4),
        "breakdown_ms": {n: round(v, 4) for n, v in per.items()},
        "dense_attn_ms": round(dense_ms * len(layers), 4),
        "speedup_vs_dense": {"attn": round(dense_ms / attn_launch_ms, 3),
                             "path": round(dense_ms * len(layers) / ms, 3)},
        "clocks": clock_info,
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "ms_per_step": round(e2e_ms, 3),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": (LAUNCHES_PER_LAYER + (args.queries == "separate")) * len(layers)
                        * args.steps,
        "roofline": {"kernel": "pbs_attn_fwd", "bound": "tensor",
                     "achieved": round(attn_tflops, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(attn_tflops / peak, 4), "peak_kind":
                     f"{pk_kind} bf16 dense, {'sustained' if long_step else 'burst'}",
                     "frac_of_sustained": round(attn_tflops / peak_sust, 4),
                     "traffic": None if args.gather_kv else traffic_for(w)},
    }
    if rank == 0 and world == 1 and not (args.no_cpu_baseline or args.profile):
        line["cpu_baseline"] = cpu_baseline(w, layers[0], total_blocks / len(layers))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def traffic_for(w):
    """DRAM bytes per forward launch from the committed ncu summary, if one
    exists for this workload."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_dram_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 2 and parts[0] == w.name:
                try:
                    return float(parts[1])
                except ValueError:
                    return None
    return None


# ---------------------------------------------------------- the CPU oracle
def oracle_sample(w, q, k, v, blocks_total_hint=None, attn_blocks=8):
    """Time the oracle on one KV group of the workload and scale it up.

    q: [1, G, n, d], k, v: [1, 1, n, d] bf16 CPU tensors of one KV group.
    Score, permutation and selection of the group are timed in full and
    scaled by the number of (batch, KV head) groups; the forward is timed on
    `attn_blocks` query blocks of the first head and scaled by kept blocks.
    Returns (seconds for the whole workload, total kept blocks, sample text).
    """
    import numpy as np

    from oracle import pbs_oracle as orc
    B, S = w.block, w.segment
    groups = w.batch * w.hkv * w.layers
    q64, k64, v64 = (t.double().numpy() for t in (q, k, v))
    t0 = time.perf_counter()
    imp = orc.score(q64, k64, B)
    t1 = time.perf_counter()
    perm = orc.permute(imp, k64, v64, S)
    t2 = time.perf_counter()
    idx, cnt, _ = orc.select_blocks(orc.block_means(q64, B), orc.block_means(perm["k_perm"], B),
                                    S // B, w.mode, w.param, None, w.group)
    t3 = time.perf_counter()
    nb = w.nb
    picks = sorted({int(round(x)) for x in np.linspace(0, nb - 1, attn_blocks)})
    blocks = [(0, 0, i) for i in picks]
    orc.attend_blocks(q64, perm["k_perm"], perm["v_perm"], perm["kpos"], None, idx, cnt, B,
                      blocks)
    t4 = time.perf_counter()
    sampled = float(sum(cnt[0, 0, i] for i in picks))
    group_blocks = float(cnt.sum())
    total_blocks = group_blocks * groups
    per_block = (t4 - t3) / sampled
    seconds = (t3 - t0) * groups + per_block * total_blocks
    text = (f"KV group 0 at full n={w.n}: score {t1 - t0:.2f}s, permute {t2 - t1:.2f}s, "
            f"select {t3 - t2:.2f}s timed in full and scaled x{groups} groups; forward on "
            f"{len(picks)} query blocks of head 0 ({int(sampled)} kept blocks, {t4 - t3:.2f}s) "
            f"scaled to {int(total_blocks)} kept blocks")
    return seconds, total_blocks, text


# Workloads whose whole oracle run stays within about half a minute on the
# host (b * hq * n^2 * d multiply-adds of the attention): timed in full.
ORACLE_FULL_LIMIT = 4e11


def oracle_fits_whole(w):
    return w.layers == 1 and w.batch * w.hq * float(w.n) ** 2 * w.d <= ORACLE_FULL_LIMIT


def oracle_whole(w, q, k, v):
    """Time the oracle's whole pipeline on the whole workload (all batches and
    heads). Returns (seconds, total kept blocks, sample text)."""
    from oracle import pbs_oracle as orc
    q64, k64, v64 = (t.double().numpy() for t in (q, k, v))
    t0 = time.perf_counter()
    res = orc.pbs_attention(q64, k64, v64, w.block, w.segment, w.mode, w.param)
    seconds = time.perf_counter() - t0
    blocks = float(res["cnt"].sum())
    return seconds, blocks, (f"the whole workload ({w.batch} x {w.hq} heads, n={w.n}), all "
                             f"five steps, timed in full")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def host_cores():
    """Cores this process may run on (the host's, unless restricted)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(w, layer, blocks_per_layer):
    if oracle_fits_whole(w):
        seconds, total_blocks, text = oracle_whole(w, layer.q.cpu(), layer.k.cpu(),
                                                   layer.v.cpu())
        extrapolated = False
    else:
        G = w.group
        seconds, total_blocks, text = oracle_sample(w, layer.q[:1, :G].cpu(),
                                                    layer.k[:1, :1].cpu(), layer.v[:1, :1].cpu())
        extrapolated = True
    value = block_flops(w, total_blocks) / seconds / 1e12
    out = {"value": value, "unit": UNIT, "cores": host_cores(), "blas_threads": blas_threads(),
           "kind": "oracle", "sample": text}
    out["ms_per_step_extrapolated" if extrapolated else "ms_per_step"] = round(seconds * 1e3, 1)
    return out


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = workload_of(args)
    whole = oracle_fits_whole(w)
    if whole:   # the whole workload, drawn on the host with the same recipe
        q, k, v, _ = make_inputs(w)
    else:       # one KV group of the workload, the rest extrapolated
        q, k, v, _ = make_inputs(w.with_(batch=1, hq=w.group, hkv=1, layers=1))
    times, text, blocks = [], "", 0.0
    for i in range(args.warmup + args.steps):
        sec, blocks, text = oracle_whole(w, q, k, v) if whole else oracle_sample(w, q, k, v)
        if i >= args.warmup:
            times.append(sec)
    sec = statistics.mean(times)
    value = block_flops(w, blocks) / sec / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": int(os.environ.get(
            "WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3,
        # with a sample, each step times one KV group and scales it to the
        # whole workload: ms_per_step is then an extrapolation, not a clock
        "ms_per_step_extrapolated": not whole,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "batch": w.batch, "hq": w.hq, "hkv": w.hkv, "n": w.n,
                   "d": w.d, "block": w.block, "segment": w.segment, "layers": w.layers,
                   "selection": f"{w.mode} {w.param}"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(),
                         "blas_threads": blas_threads(), "kind": "oracle", "sample": text},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
