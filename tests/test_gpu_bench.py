"""bench.py on the GPU: every timed mode computes the path's result, and the
JSON line carries the fields of its contract."""
import json
import os
import subprocess
import sys

import pytest
import torch

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200.workloads import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda", 0)


@pytest.mark.parametrize("queries", ["natural", "fused", "separate"])
@pytest.mark.parametrize("gather_kv", [False, True])
@pytest.mark.parametrize("block", [128, 64])
def test_timed_step_computes_the_path(queries, gather_kv, block, dev):
    """The step bench.py times gives, in every mode and for both block
    sizes, the output of the path's own entry point in the matching query
    and key-fetch mode."""
    sys.path.insert(0, ROOT)
    import bench

    w = Workload("bench2k", 1, 8, 2, 2048, 128, block, 512, "topk_frac", 0.3, "per_segment",
                 0.02)
    layer = bench.Layer(w, dev, 0, seed_offset=0, gather_kv=gather_kv, queries=queries)
    for _ in range(2):  # the second step reuses the first one's buffers
        o, cnt = bench.run_layer(layer)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    ref = pbs.pbs_attention(layer.q, layer.k, layer.v, w.block, w.segment, w.mode, w.param,
                            permute_q=queries != "natural", gather_kv=gather_kv)
    assert torch.equal(o, ref)
    assert int(cnt.sum()) > 0


def run_bench(*args, timeout=600):
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=timeout)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_line_contract(dev):
    d = run_bench("--config", "llama8k", "--steps", "2", "--warmup", "3", "--no-cpu-baseline",
                  "--e2e-steps", "1")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "clocks", "gpu_launches"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] >= 3
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "llama8k"
    assert d["config"]["l2"].startswith("flushed")  # 100 MB of inputs fit in L2
    assert d["gpu_launches"] == 9 * 2
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert 0 < r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-3)
    e = d["e2e"]
    w = WORKLOADS["llama8k"]
    assert e["value"] > 0
    assert e["h2d_bytes_per_step"] == 2 * w.batch * (w.hq + 2 * w.hkv) * w.n * w.d
    assert e["d2h_bytes_per_step"] == 2 * w.batch * w.hq * w.n * w.d


def test_bench_block_option(dev):
    """--block 64 runs the workload with 64-key blocks (same segment and
    selection) and says so in its config."""
    d = run_bench("--config", "llama8k", "--block", "64", "--steps", "2", "--warmup", "3",
                  "--no-cpu-baseline", "--e2e-steps", "1")
    assert d["config"]["workload"] == "llama8k_b64" and d["config"]["block"] == 64
    assert d["config"]["segment"] == WORKLOADS["llama8k"].segment
    assert d["value"] > 0 and d["roofline"]["achieved"] > 0


@pytest.mark.parametrize("queries", ["natural", "fused", "separate"])
@pytest.mark.parametrize("gather_kv", [False, True])
def test_graph_of_the_timed_step_computes_the_path(queries, gather_kv, dev):
    """The step captured as a CUDA graph the way `bench.py --graph` does
    (events around each step inside the graph) gives the path's output when
    replayed, also after new inputs are copied into the layer's tensors."""
    sys.path.insert(0, ROOT)
    import bench

    w = Workload("bench2k", 1, 8, 2, 2048, 128, 128, 512, "topk_frac", 0.3, "per_segment",
                 0.02)
    layer = bench.Layer(w, dev, 0, seed_offset=0, gather_kv=gather_kv, queries=queries)
    bench.run_layer(layer)  # the warm-up step: output buffers, kernel attributes
    names = ("score", "permute", "select", "attn", "unpermute")
    ev = {n: (torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True)) for n in names}
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        o, _ = bench.run_layer(layer, ev)
    fresh = bench.Layer(w, dev, 1, seed_offset=0)
    for turn in range(2):
        if turn:
            for t, src in ((layer.q, fresh.q), (layer.k, fresh.k), (layer.v, fresh.v)):
                t.copy_(src)
        g.replay()
        ref = pbs.pbs_attention(layer.q, layer.k, layer.v, w.block, w.segment, w.mode, w.param,
                                permute_q=queries != "natural", gather_kv=gather_kv)
        torch.cuda.synchronize()
        assert pbs.device_status() == 0
        assert torch.equal(o, ref), f"replay {turn}"
        assert ev["attn"][0].elapsed_time(ev["attn"][1]) > 0


def test_bench_graph_option(dev):
    """--graph replays one CUDA graph per layer in the timed region and says
    so in its config; its per-step breakdown comes from the graph's events."""
    d = run_bench("--config", "tiny", "--graph", "--steps", "20", "--warmup", "3",
                  "--no-cpu-baseline", "--e2e-steps", "1")
    assert d["config"]["launch"] == "one CUDA graph per layer, replayed"
    assert d["value"] > 0 and d["breakdown_ms"]["attn"] > 0
    assert d["breakdown_ms"]["attn"] <= d["ms_per_step"]
