"""Parity at the full workload sizes, in the launch configuration bench.py times.

The oracle cannot run whole 32K-128K problems, so at full size the checks are
exact where the result is integer or a gather (key order of every head from
the GPU's own importance, K'/V' gathers, fp64 block sums of sampled heads,
block lists of sampled heads), and sampled for the floating-point results
(the importance of one KV head in full, output rows of sampled query blocks
of sampled heads against the oracle). llama128k is also run with every
admissible block kept and compared with dense causal attention on the same
forward (Theorem 3.3) and with the oracle's dense attention on sampled rows.
Inputs are drawn on the GPU with the same seeded recipe as the bench.
"""
import numpy as np
import pytest
import torch

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200.workloads import WORKLOADS, make_inputs
from oracle import pbs_oracle as orc
from pbs_testutil import assert_importance_close, assert_outputs_close, compare_lists, f64, i64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda", 0)


def run_path(w, dev, layer=0):
    q, k, v, _ = make_inputs(w, dev, layer=layer)
    res = pbs.pbs_attention(q, k, v, w.block, w.segment, w.mode, w.param, keep=True)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    return q, k, v, res


def check_full_size(w, dev, heads, blocks, layer=0):
    B, S, G = w.block, w.segment, w.group
    q, k, v, res = run_path(w, dev, layer)
    imp, kpos = res["imp"], res["kpos"]
    # importance: every row sums to one; one KV head in full against the oracle
    sums = imp.double().sum(-1)
    assert torch.allclose(sums, torch.ones_like(sums), atol=1e-3)
    bi, h = 0, heads[0] // G
    qg = f64(q[bi:bi + 1, h * G:(h + 1) * G])
    kg = f64(k[bi:bi + 1, h:h + 1])
    assert_importance_close(f64(imp[bi:bi + 1, h:h + 1]), orc.score(qg, kg, B))
    # key order of every head, exactly, from the GPU's own importance
    np.testing.assert_array_equal(i64(kpos), orc.segment_order(f64(imp), S))
    # gathers, exactly, on the device
    idx = kpos.long().unsqueeze(-1).expand(-1, -1, -1, w.d)
    assert torch.equal(res["k_perm"], torch.gather(k, 2, idx))
    assert torch.equal(res["v_perm"], torch.gather(v, 2, idx))
    # block sums and lists of the sampled heads
    for g in heads:
        hk = g // G
        kp = f64(res["k_perm"][bi:bi + 1, hk:hk + 1])
        np.testing.assert_array_equal(f64(res["kbar_sum"][bi:bi + 1, hk:hk + 1]),
                                      orc.block_means(kp, B) * B)
        qb, kb = orc.block_means(f64(q[bi:bi + 1, g:g + 1]), B), orc.block_means(kp, B)
        ref_idx, ref_cnt, margin = orc.select_blocks(qb, kb, S // B, w.mode, w.param, None, 1)
        n_amb = compare_lists(res["idx"][bi:bi + 1, g:g + 1], res["cnt"][bi:bi + 1, g:g + 1],
                              ref_idx, ref_cnt, margin, scores=orc.block_scores(qb, kb, None, 1),
                              spb=S // B, mode=w.mode, param=w.param)
        print(f"{w.name} head {g}: {n_amb} near-tie selections checked for validity")
        # sampled output blocks of this head against the oracle
        kpos_h = i64(kpos[bi:bi + 1, hk:hk + 1])
        idx_g, cnt_g = i64(res["idx"][bi:bi + 1, g:g + 1]), i64(res["cnt"][bi:bi + 1, g:g + 1])
        qh = f64(q[bi:bi + 1, g:g + 1])
        vp = f64(res["v_perm"][bi:bi + 1, hk:hk + 1])
        ref = orc.attend_blocks(qh, kp, vp, kpos_h, None, idx_g, cnt_g, B,
                                [(0, 0, I) for I in blocks])
        got = np.stack([f64(res["o"][bi, g, I * B:(I + 1) * B]) for I in blocks])
        assert_outputs_close(got, ref, f"{w.name} head {g}")
    return q, k, v, res


def sample_blocks(nb, spb):
    return sorted({0, 1, spb - 1, spb, nb // 2, nb - spb, nb - 2, nb - 1})


def test_llama8k_full_size(dev):
    """The 8K layer in full: every KV head's importance against the oracle,
    every head's block lists against the oracle (bit for bit on decided rows),
    and eight sampled query blocks of each of the 32 heads."""
    w = WORKLOADS["llama8k"]
    B, S, G = w.block, w.segment, w.group
    q, k, v, res = check_full_size(w, dev, heads=list(range(w.hq)),
                                   blocks=sample_blocks(w.nb, S // B))
    assert_importance_close(f64(res["imp"]), orc.score(f64(q), f64(k), B))


def test_llama32k_block64_full_size(dev):
    """The 32K layer with 64-key blocks (the B = 64 tcgen05 scoring and
    forward) at full size: key orders of every head, lists and sampled
    output blocks of three heads against the oracle."""
    w = WORKLOADS["llama32k"].with_(name="llama32k_b64", block=64)
    check_full_size(w, dev, heads=[0, 17, 31], blocks=sample_blocks(w.nb, w.segment // w.block))


def test_llama32k_full_size(dev):
    w = WORKLOADS["llama32k"]
    check_full_size(w, dev, heads=[0, 13, 31], blocks=sample_blocks(w.nb, w.segment // w.block))


def test_llama128k_top25_full_size(dev):
    w = WORKLOADS["llama128k"]
    q, k, v, res = check_full_size(w, dev, heads=[0, 21],
                                   blocks=sample_blocks(w.nb, w.segment // w.block))
    # the top-k rule fixes every count: own segment, plus k - own earlier blocks
    I = torch.arange(w.nb, device=dev)
    spb = w.segment // w.block
    k_i = torch.clamp((0.25 * (I + 1).double()).floor().long(), min=1)
    own = torch.clamp(w.nb - (I // spb) * spb, max=spb)
    earlier = (I // spb) * spb
    want = own + torch.minimum(earlier, torch.clamp(k_i - own, min=0))
    assert torch.equal(res["cnt"][0].long(), want.expand(w.hq, -1))


def test_llama512k_full_size(dev):
    """The largest context the bench runs (524,288 keys): Q and O hold 2^31
    bf16 values (4 GiB) and the block lists 2^29 entries, so byte offsets
    leave the 32-bit range. Orders of every head exact, gathers exact, one
    KV head's importance, two heads' lists and sampled output blocks against
    the oracle, the top-k counts of every row, and the last query block of
    the last head (the last rows of O)."""
    w = WORKLOADS["llama512k"]
    B, S = w.block, w.segment
    q, k, v, res = check_full_size(w, dev, heads=[0, 29], blocks=sample_blocks(w.nb, S // B))
    I = torch.arange(w.nb, device=dev)
    spb = S // B
    k_i = torch.clamp((float(np.float32(w.param)) * (I + 1).double()).floor().long(), min=1)
    own = torch.clamp(w.nb - (I // spb) * spb, max=spb)
    earlier = (I // spb) * spb
    want = own + torch.minimum(earlier, torch.clamp(k_i - own, min=0))
    assert torch.equal(res["cnt"][0].long(), want.expand(w.hq, -1))
    # the last query block of the last head: the last rows of O
    g, hk = w.hq - 1, (w.hq - 1) // w.group
    kp = f64(res["k_perm"][0:1, hk:hk + 1])
    vp = f64(res["v_perm"][0:1, hk:hk + 1])
    ref = orc.attend_blocks(f64(q[0:1, g:g + 1]), kp, vp, i64(res["kpos"][0:1, hk:hk + 1]), None,
                            i64(res["idx"][0:1, g:g + 1]), i64(res["cnt"][0:1, g:g + 1]), B,
                            [(0, 0, w.nb - 1)])
    got = f64(res["o"][0, g, (w.nb - 1) * B:w.nb * B])[None]
    assert_outputs_close(got, ref, "llama512k last block of the last head")


def test_llama128k_all_blocks_is_dense_causal(dev):
    w = WORKLOADS["llama128k"]
    B, S = w.block, w.segment
    q, k, v, _ = make_inputs(w, dev)
    imp = pbs.score(q, k, B, S)
    perm = pbs.permute(imp, k, v, B, S, hq=w.hq)
    idx, cnt, _ = pbs.select_blocks(q, perm["k_perm"], perm["kbar_sum"], B, S, "all")
    o_all = pbs.attn_fwd(q, perm["k_perm"], perm["v_perm"], perm["kpos"], None, idx, cnt, B, S)
    del idx
    didx, dcnt, _ = pbs.select_blocks(q, k, None, B, S, "dense_causal")
    o_dense = pbs.attn_fwd(q, k, v, None, None, didx, dcnt, B, S)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    err = (o_all.float() - o_dense.float()).abs()
    assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3
    # sampled rows of head 5 against the oracle's dense causal attention
    g, hk = 5, 5 // w.group
    rows = [0, 1, 4095, 4096, 65537, w.n - 1]
    q64, k64, v64 = f64(q[0, g]), f64(k[0, hk]), f64(v[0, hk])
    sigma = 1.0 / np.sqrt(w.d)
    for r in rows:
        logits = sigma * (k64[:r + 1] @ q64[r])
        p = np.exp(logits - logits.max())
        want = (p / p.sum()) @ v64[:r + 1]
        assert_outputs_close(f64(o_dense[0, g, r])[None], want[None], f"dense row {r}")
        assert_outputs_close(f64(o_all[0, g, r])[None], want[None], f"all-blocks row {r}")


def test_stack64k_one_layer_batch2(dev):
    w = WORKLOADS["stack64k"]
    check_full_size(w, dev, heads=[7], blocks=sample_blocks(w.nb, w.segment // w.block), layer=3)


@pytest.mark.parametrize("name", ["llama32k", "llama128k"])
def test_gathering_forward_full_size(name, dev):
    """At full size the forward that reads K, V through the key order gives
    the forward on the gathered copies bit for bit, and the order-only
    permutation the same order and block sums."""
    w = WORKLOADS[name]
    B, S = w.block, w.segment
    q, k, v, res = run_path(w, dev)
    imp = pbs.score(q, k, B, S)
    lean = pbs.permute(imp, k, v, B, S, hq=w.hq, materialize=False)
    assert torch.equal(lean["kpos"], res["kpos"])
    assert torch.equal(lean["kbar_sum"], res["kbar_sum"])
    o = pbs.attn_fwd_gather(q, k, v, lean["kpos"], None, res["idx"], res["cnt"], B, S)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    assert torch.equal(o, res["o"])
