"""The whole path captured once as a CUDA graph (PathGraph) and replayed.

A replay launches the same kernels with the same arguments as the eager
calls, so every intermediate and the output must equal the eager path's bit
for bit: on the captured inputs, and again after new inputs have been copied
into the captured tensors (the graph reads whatever they hold). Block lists
are compared on their valid entries (the count of each row) only.
"""
import pytest
import torch

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": WORKLOADS["tiny"],  # B = 64, d = 64, one head
    "gqa": Workload("gqa_graph", 1, 8, 2, 2048, 128, 128, 512, "topk_frac", 0.3, "per_segment",
                    0.02),
    "b64": Workload("b64_graph", 1, 4, 2, 1280, 128, 64, 256, "threshold", 0.9, "uniform", 0.05),
}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda", 0)


def assert_same(got, want, what):
    for key in ("imp", "kpos", "k_perm", "v_perm", "kbar_sum", "q_perm", "cnt", "o"):
        if key in want and want[key] is not None:
            assert torch.equal(got[key], want[key]), f"{what}: {key}"
    cnt = want["cnt"].long()
    valid = torch.arange(want["idx"].shape[-1], device=cnt.device) < cnt.unsqueeze(-1)
    assert torch.equal(torch.where(valid, got["idx"], 0), torch.where(valid, want["idx"], 0)), \
        f"{what}: idx"


@pytest.mark.parametrize("permute_q", [False, True])
@pytest.mark.parametrize("name", sorted(CASES))
def test_replay_equals_eager(name, permute_q, dev):
    w = CASES[name]
    B, S = w.block, w.segment
    q, k, v, _ = make_inputs(w, dev)
    graph = pbs.PathGraph(q, k, v, B, S, w.mode, w.param, permute_q=permute_q, keep=True)
    for turn in range(3):
        if turn == 1:  # new inputs copied into the captured tensors
            q2, k2, v2, _ = make_inputs(w, dev, seed=w.seed + 100)
            q.copy_(q2), k.copy_(k2), v.copy_(v2)
        got = graph.replay()
        want = pbs.pbs_attention(q, k, v, B, S, w.mode, w.param, permute_q=permute_q, keep=True)
        torch.cuda.synchronize()
        assert pbs.device_status() == 0
        assert_same(got, want, f"{name} replay {turn}")


def test_replays_back_to_back(dev):
    """Ten replays queued without a host wait in between give the eager
    output of the inputs they last saw."""
    w = CASES["gqa"]
    q, k, v, _ = make_inputs(w, dev)
    graph = pbs.PathGraph(q, k, v, w.block, w.segment, w.mode, w.param)
    for _ in range(10):
        o = graph.replay()
    want = pbs.pbs_attention(q, k, v, w.block, w.segment, w.mode, w.param)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    assert torch.equal(o, want)
