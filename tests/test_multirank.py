"""Host-side logic of the N > 1 bench path, on two gloo ranks on the CPU.

Under torchrun every rank runs its own replica of the workload (the path's
units are independent, so no collective touches the data). What the ranks
share is the reporting: the whole-job throughput is all ranks' work over the
slowest rank's time, and every rank draws different inputs.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from long_context_sparse_segment_b200.workloads import WORKLOADS, make_inputs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        flops = 1e12 * (rank + 1)
        ms = 10.0 * (rank + 1)
        value, ms_max, total = bench.job_throughput(flops, ms, dist, "cpu")
        w = WORKLOADS["tiny"]
        q, _, _, _ = make_inputs(w, seed=w.seed + bench.rank_seed_offset(rank))
        digests = [None] * world
        dist.all_gather_object(digests, float(q.float().sum()))
        out.put((rank, value, ms_max, total, digests))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_whole_job_throughput_over_distinct_replicas():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms_max, total, digests in results:
        assert ms_max == 20.0                      # the slowest rank
        assert total == 3e12                       # both ranks' work
        assert value == pytest.approx(150.0)       # 3e12 flop / 20 ms
        assert digests[0] != digests[1]            # replicas draw different inputs


def test_single_process_throughput_needs_no_collective():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.job_throughput(2e12, 4.0) == (500.0, 4.0, 2e12)
    assert bench.rank_seed_offset(0) == 0 and bench.rank_seed_offset(3) == 3000


def test_head_sharding_covers_every_kv_group_once():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from long_context_sparse_segment_b200.workloads import WORKLOADS
    w = WORKLOADS["llama512k"]
    for world in (1, 2, 4, 8):
        heads = []
        for rank in range(world):
            ws, first = bench.shard_heads(w, rank, world)
            assert ws.hq == ws.hkv * w.group and ws.n == w.n
            heads += list(range(first, first + ws.hkv))
        assert heads == list(range(w.hkv))
    with pytest.raises(ValueError):
        bench.shard_heads(w, 0, 3)


def _sharded_worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from long_context_sparse_segment_b200.workloads import WORKLOADS

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = WORKLOADS["llama128k"]
        ws, _ = bench.shard_heads(w, rank, world)
        # each rank's flops are its share of the sequence; strong scaling:
        # the job's throughput is the whole sequence's flops over the slowest rank
        flops = 1e12 * ws.hq / w.hq
        value, ms, total = bench.job_throughput(flops, 5.0 + rank, dist, "cpu")
        out.put((rank, value, ms, total))
    finally:
        dist.destroy_process_group()


def test_two_ranks_head_sharded_throughput_counts_the_sequence_once():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms, total in results:
        assert total == pytest.approx(1e12)      # the sequence's flops, once
        assert ms == 6.0                         # the slower rank
        assert value == pytest.approx(1e12 / 6e-3 / 1e12)


def _gather_worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from long_context_sparse_segment_b200.workloads import WORKLOADS

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ok = []
        for batch in (1, 2):
            w = WORKLOADS["llama8k"].with_(batch=batch, n=256)
            ws, first = bench.shard_heads(w, rank, world)
            # a stand-in for the whole output whose every element names its place
            full = torch.arange(batch * w.hq * w.n * 8, dtype=torch.float32).reshape(
                batch, w.hq, w.n, 8)
            mine = full[:, first * w.group:(first + ws.hkv) * w.group].clone()
            got = bench.gather_heads(mine, dist, world)
            ok.append(bool(torch.equal(got, full)))
            into = torch.empty_like(full)
            ok.append(bench.gather_heads(mine, dist, world, out=into) is into
                      and bool(torch.equal(into, full)))
        out.put((rank, ok))
    finally:
        dist.destroy_process_group()


def test_all_gather_of_sharded_output_heads():
    """With --shard heads --gather-output every rank ends with the whole
    output: the ranks' head slices all-gathered in shard order."""
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok in results:
        assert all(ok), (rank, ok)
