"""The forward that reads K and V through the carried key positions
(pbs_attn_fwd_gather) and the order-only permutation that feeds it.

A segment-local permutation only decides which rows of K and V make up each
key block, so the forward may fetch those rows by index instead of from
gathered copies. The tensor cores then see the same tiles in the same order:
the output must equal the forward on K' = K[kpos], V' = V[kpos] bit for bit
(on each kernel: the tcgen05 ones for B = 128 and B = 64, and the warp-MMA
one), and the CPU oracle fed the GPU's order and lists within the forward's
tolerance.
"""
import numpy as np
import pytest
import torch

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200 import _lib
from long_context_sparse_segment_b200.workloads import Workload, make_inputs
from oracle import pbs_oracle as orc
from pbs_testutil import assert_outputs_close, f64, i64

pytestmark = pytest.mark.gpu

CASES = {
    "gqa2k": Workload("gqa2k", 1, 8, 2, 2048, 128, 128, 512, "threshold", 0.9,
                      "per_segment", 0.02),
    "ragged": Workload("ragged", 2, 4, 2, 1280, 128, 128, 512, "topk_frac", 0.3,
                       "per_segment", 0.02),
    "d64_b128": Workload("d64_b128", 1, 4, 1, 1024, 64, 128, 256, "threshold", 0.7,
                         "uniform", 0.05),
    "d128_b64": Workload("d128_b64", 1, 4, 4, 1024, 128, 64, 256, "topk_frac", 0.25,
                         "uniform", 0.05),
    "odd_items": Workload("odd_items", 1, 3, 1, 1152, 128, 128, 384, "topk_frac", 0.4,
                          "uniform", 0.05),
    "s_eq_n": Workload("s_eq_n", 1, 2, 1, 1024, 64, 64, 1024, "threshold", 0.5,
                       "uniform", 0.05),
}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda", 0)


def prepared(w, dev, permute_q):
    q, k, v, _ = make_inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, q=qd if permute_q else None, hq=w.hq)
    q_used = perm["q_perm"] if permute_q else qd
    idx, cnt, _ = pbs.select_blocks(q_used, perm["k_perm"], perm["kbar_sum"], B, S, w.mode,
                                    w.param)
    return (q, k, v), (qd, kd, vd), perm, q_used, idx, cnt


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("forward", ["default", "mma"])
@pytest.mark.parametrize("permute_q", [False, True])
def test_gather_forward_equals_forward_on_gathered_copies(name, forward, permute_q, dev,
                                                          monkeypatch):
    w = CASES[name]
    if forward != "default":
        monkeypatch.setenv("PBS_FORWARD", forward)
    _, (qd, kd, vd), perm, q_used, idx, cnt = prepared(w, dev, permute_q)
    B, S = w.block, w.segment
    qpos = perm["kpos"] if permute_q else None
    o_ref, lse_ref = pbs.attn_fwd(q_used, perm["k_perm"], perm["v_perm"], perm["kpos"], qpos,
                                  idx, cnt, B, S, lse=True)
    o, lse = pbs.attn_fwd_gather(q_used, kd, vd, perm["kpos"], qpos, idx, cnt, B, S, lse=True)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)
    if permute_q:  # the inverse permutation fused into the same call
        o_nat = pbs.attn_fwd_gather(q_used, kd, vd, perm["kpos"], qpos, idx, cnt, B, S,
                                    unpermute=True)
        assert torch.equal(o_nat, pbs.unpermute(o_ref, qpos, w.hkv, B, S))
        assert pbs.device_status() == 0


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d128_b64", "odd_items"])
def test_gather_forward_against_oracle(name, dev):
    """The oracle's attention on K, V gathered on the CPU by the GPU's key
    order, with the GPU's lists."""
    w = CASES[name]
    (q, k, v), (qd, kd, vd), perm, _, idx, cnt = prepared(w, dev, False)
    B = w.block
    o = pbs.attn_fwd_gather(qd, kd, vd, perm["kpos"], None, idx, cnt, B, w.segment)
    kpos = i64(perm["kpos"])
    kp = np.take_along_axis(f64(k), kpos[..., None], axis=2)
    vp = np.take_along_axis(f64(v), kpos[..., None], axis=2)
    ref = orc.attend(f64(q), kp, vp, kpos, None, i64(idx), i64(cnt), B)
    assert_outputs_close(f64(o), ref, name)


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d128_b64"])
@pytest.mark.parametrize("permute_q", [False, True])
def test_order_only_permutation(name, permute_q, dev):
    """pbs_permute with no K'/V' outputs writes the same order and key block
    sums (and Q' in permuted-query mode)."""
    w = CASES[name]
    _, (qd, kd, vd), perm, _, _, _ = prepared(w, dev, permute_q)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    lean = pbs.permute(imp, kd, vd, B, S, q=qd if permute_q else None, hq=w.hq,
                       materialize=False)
    assert lean["k_perm"] is None and lean["v_perm"] is None
    assert torch.equal(lean["kpos"], perm["kpos"])
    assert torch.equal(lean["kbar_sum"], perm["kbar_sum"])
    if permute_q:
        assert torch.equal(lean["q_perm"], perm["q_perm"])
    assert pbs.device_status() == 0


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d64_b128", "d128_b64"])
@pytest.mark.parametrize("permute_q", [False, True])
def test_path_with_gathering_forward(name, permute_q, dev):
    w = CASES[name]
    _, (qd, kd, vd), _, _, _, _ = prepared(w, dev, permute_q)
    B, S = w.block, w.segment
    o_ref = pbs.pbs_attention(qd, kd, vd, B, S, w.mode, w.param, permute_q=permute_q)
    o = pbs.pbs_attention(qd, kd, vd, B, S, w.mode, w.param, permute_q=permute_q,
                          gather_kv=True)
    assert torch.equal(o, o_ref)
    assert pbs.device_status() == 0


@pytest.mark.parametrize("forward", ["default", "mma"])
def test_gather_reports_a_position_outside_its_segment(forward, dev, monkeypatch):
    """A carried position from another segment (still a row of the same head,
    so every read stays in bounds) is reported; the key's own row is read
    instead."""
    if forward != "default":
        monkeypatch.setenv("PBS_FORWARD", forward)
    w = CASES["gqa2k"]
    _, (qd, kd, vd), perm, _, _, _ = prepared(w, dev, False)
    B, S = w.block, w.segment
    kpos = perm["kpos"].clone()
    kpos[0, 0, S + 5] = 3  # slot of segment 1 pointing into segment 0
    idx, cnt, _ = pbs.select_blocks(qd, None, perm["kbar_sum"], B, S, "all")
    pbs.attn_fwd_gather(qd, kd, vd, kpos, None, idx, cnt, B, S)
    assert pbs.device_status() == _lib.ERR_DEVICE_ASSERT
    assert pbs.device_status() == 0


def test_gather_argument_checks(dev):
    w = CASES["gqa2k"]
    _, (qd, kd, vd), perm, _, idx, cnt = prepared(w, dev, True)
    B, S = w.block, w.segment
    with pytest.raises(pbs.PbsError):  # the carried positions are required
        shp = pbs.shape_of(qd, kd, B, S)
        pbs.ops.check(pbs.lib().pbs_attn_fwd_gather(
            pbs.ops._ptr(qd), pbs.ops._ptr(kd), pbs.ops._ptr(vd), None, None,
            pbs.ops._ptr(idx), pbs.ops._ptr(cnt), pbs.ops._ptr(torch.empty_like(qd)), None, shp,
            0.0, 0, None), "pbs_attn_fwd_gather")
    with pytest.raises(pbs.PbsError):  # written in place over an input still being read
        pbs.attn_fwd_gather(perm["q_perm"], kd, vd, perm["kpos"], perm["kpos"], idx, cnt, B, S,
                            out=perm["q_perm"], unpermute=True)
    with pytest.raises(pbs.PbsError):  # K' without V'
        imp = pbs.score(qd, kd, B)
        shp = pbs.shape_of(qd, kd, B, S)
        kpos = torch.empty_like(perm["kpos"])
        pbs.ops.check(pbs.lib().pbs_permute(
            pbs.ops._ptr(imp), pbs.ops._ptr(kd), pbs.ops._ptr(vd), None,
            pbs.ops._ptr(torch.empty_like(kd)), None, None, pbs.ops._ptr(kpos), None, shp, None),
            "pbs_permute")
