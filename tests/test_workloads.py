"""The seeded input generator: shapes, reproducibility, planted structure."""
import torch

from long_context_sparse_segment_b200.workloads import WORKLOADS, make_inputs, salient_mask


def test_tiny_shapes_and_determinism():
    w = WORKLOADS["tiny"]
    q, k, v, sal = make_inputs(w)
    assert q.shape == (1, 1, 1024, 64) and q.dtype == torch.bfloat16
    assert k.shape == v.shape == (1, 1, 1024, 64)
    q2, k2, v2, sal2 = make_inputs(w)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    assert int(sal.sum()) == 51          # 5 % of 1024, without replacement


def test_per_segment_and_burst_counts():
    w = WORKLOADS["llama8k"].with_(n=2048, hq=4, hkv=2)
    gen = torch.Generator().manual_seed(0)
    sal = salient_mask(w, gen, "cpu")
    per_seg = sal.view(1, 2, 2, 1024).sum(-1)
    assert torch.all(per_seg == 20)
    w = WORKLOADS["llama32k"].with_(hq=4, hkv=2)
    gen = torch.Generator().manual_seed(0)
    sal = salient_mask(w, gen, "cpu")
    assert 16 <= int(sal[0, 0].sum()) <= 41 * 16


def test_planted_keys_share_direction_with_queries():
    w = WORKLOADS["tiny"]
    q, k, _, sal = make_inputs(w)
    kf = k.float()[0, 0]
    qm = q.float()[0, 0].mean(0)
    s = kf @ qm
    assert s[sal[0, 0]].mean() > s[~sal[0, 0]].mean() + 1.0
