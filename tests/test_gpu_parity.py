"""GPU parity of every step of the path against the CPU oracle, through the
C ABI, on seeded synthetic inputs (sizes the oracle finishes in seconds,
spanning several tiles, with ragged segments and the degenerate cases).

Split of the parity bar:
  * score: fp32 importance within 1e-4 relative of the fp64 oracle;
  * permute: the oracle's segment order applied to the GPU's own importance
    equals the GPU kpos bit for bit; K', V' are exact gathers; the fp64 block
    sums are exact;
  * select: the oracle fed the GPU's permuted keys gives bit-identical lists;
    a decision whose oracle margin is below 1e-12 (a near-tie) is counted and
    its list checked for validity against the rule instead;
  * forward: the oracle fed the GPU's kpos and lists is within max-abs 2e-2
    and mean-abs 2e-3.
"""
import numpy as np
import pytest
import torch

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import pbs_oracle as orc
from pbs_testutil import (assert_importance_close, assert_outputs_close, compare_lists, f64,
                          i64, order_differences)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": WORKLOADS["tiny"],
    # Llama-shaped GQA, reduced length
    "gqa2k": Workload("gqa2k", 1, 8, 2, 2048, 128, 128, 512, "threshold", 0.9,
                      "per_segment", 0.02),
    # two batches, last segment shorter than S, top-k selection
    "ragged": Workload("ragged", 2, 4, 2, 1280, 128, 128, 512, "topk_frac", 0.3,
                       "per_segment", 0.02),
    "d64_b128": Workload("d64_b128", 1, 4, 1, 1024, 64, 128, 256, "threshold", 0.7,
                         "uniform", 0.05),
    "d128_b64": Workload("d128_b64", 1, 4, 4, 1024, 128, 64, 256, "topk_frac", 0.25,
                         "uniform", 0.05),
    # S = B: one block per segment
    "s_eq_b": Workload("s_eq_b", 1, 4, 2, 1024, 128, 128, 128, "threshold", 0.9,
                       "uniform", 0.05),
    # an odd number of (head, query block) items: the last CTA of the
    # two-tile forward has one tile
    "odd_items": Workload("odd_items", 1, 3, 1, 1152, 128, 128, 384, "topk_frac", 0.4,
                          "uniform", 0.05),
    # S = N: one segment, every block forced
    "s_eq_n": Workload("s_eq_n", 1, 2, 1, 1024, 64, 64, 1024, "threshold", 0.5,
                       "uniform", 0.05),
    # B = 64 with an odd number of query blocks and S = B (each query block of
    # a paired tile in its own segment), GQA with G = 3
    "b64_odd": Workload("b64_odd", 1, 3, 1, 1216, 128, 64, 64, "topk_frac", 0.3,
                        "uniform", 0.05),
}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda", 0)


def inputs(w, dev):
    q, k, v, _ = make_inputs(w)
    return (q, k, v), (q.to(dev), k.to(dev), v.to(dev))


@pytest.mark.parametrize("name", list(CASES))
def test_steps_against_oracle(name, dev):
    w = CASES[name]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    q64, k64, v64 = f64(q), f64(k), f64(v)

    imp = pbs.score(qd, kd, B)
    assert_importance_close(f64(imp), orc.score(q64, k64, B))

    perm = pbs.permute(imp, kd, vd, B, S, hq=w.hq)
    kpos = i64(perm["kpos"])
    np.testing.assert_array_equal(kpos, orc.segment_order(f64(imp), S))
    kp = perm["k_perm"]
    assert torch.equal(kp.cpu(), torch.from_numpy(np.take_along_axis(
        k.float().numpy(), kpos[..., None], axis=2)).to(torch.bfloat16))
    assert torch.equal(perm["v_perm"].cpu(), torch.from_numpy(np.take_along_axis(
        v.float().numpy(), kpos[..., None], axis=2)).to(torch.bfloat16))
    np.testing.assert_array_equal(f64(perm["kbar_sum"]), orc.block_means(f64(kp), B) * B)

    idx, cnt, mask = pbs.select_blocks(qd, kp, perm["kbar_sum"], B, S, w.mode, w.param,
                                       mask=True)
    qb, kb = orc.block_means(q64, B), orc.block_means(f64(kp), B)
    ref_idx, ref_cnt, margin = orc.select_blocks(qb, kb, S // B, w.mode, w.param, None, w.group)
    n_amb = compare_lists(idx, cnt, ref_idx, ref_cnt, margin,
                          scores=orc.block_scores(qb, kb, None, w.group), spb=S // B,
                          mode=w.mode, param=w.param)
    print(f"{name}: {n_amb} near-tie selections checked for validity")
    m = i64(mask)
    for r in np.ndindex(*ref_cnt.shape):
        assert m[r].sum() == ref_cnt[r]
        assert np.all(m[r][ref_idx[r][:ref_cnt[r]]] == 1)

    o = pbs.attn_fwd(qd, kp, perm["v_perm"], perm["kpos"], None, idx, cnt, B, S)
    ref_o = orc.attend(q64, f64(kp), f64(perm["v_perm"]), kpos, None, i64(idx), i64(cnt), B)
    assert_outputs_close(f64(o), ref_o, name)


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d128_b64"])
@pytest.mark.parametrize("permute_q", [False, True])
def test_end_to_end_against_oracle(name, permute_q, dev):
    """The whole path against the oracle's own pipeline. The permutations may
    differ only inside runs of near-equal importance; outputs must agree."""
    w = CASES[name]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    res = pbs.pbs_attention(qd, kd, vd, w.block, w.segment, w.mode, w.param,
                            permute_q=permute_q, keep=True)
    ref = orc.pbs_attention(f64(q), f64(k), f64(v), w.block, w.segment, w.mode, w.param,
                            permute_q=permute_q)
    # the orders may differ only at slots whose two keys have oracle
    # importances within the scoring tolerance of each other
    n_diff = order_differences(i64(res["kpos"]), ref["kpos"], ref["imp"])
    print(f"{name} permute_q={permute_q}: {n_diff} of {ref['kpos'].size} key slots differ "
          f"inside near-equal importance runs")
    assert_outputs_close(f64(res["o"]), ref["o"], name)


def test_permuted_query_mode_steps(dev):
    w = CASES["gqa2k"]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, q=qd)
    kpos = i64(perm["kpos"])
    qpos = np.repeat(kpos, w.group, axis=1)
    assert torch.equal(perm["q_perm"].cpu(), torch.from_numpy(np.take_along_axis(
        q.float().numpy(), qpos[..., None], axis=2)).to(torch.bfloat16))
    idx, cnt, _ = pbs.select_blocks(perm["q_perm"], perm["k_perm"], perm["kbar_sum"], B, S,
                                    w.mode, w.param)
    o_perm = pbs.attn_fwd(perm["q_perm"], perm["k_perm"], perm["v_perm"], perm["kpos"],
                          perm["kpos"], idx, cnt, B, S)
    ref = orc.attend(f64(perm["q_perm"]), f64(perm["k_perm"]), f64(perm["v_perm"]), kpos, qpos,
                     i64(idx), i64(cnt), B)
    assert_outputs_close(f64(o_perm), ref, "q-permuted forward")
    o = pbs.unpermute(o_perm, perm["kpos"], w.hkv, B, S)
    assert torch.equal(o.cpu(), torch.from_numpy(np.ascontiguousarray(
        orc.unpermute(f64(o_perm), qpos))).to(torch.bfloat16))


def test_all_blocks_equals_dense_causal(dev):
    """Theorem 3.3 on the GPU path: with every admissible block kept, the
    permuted forward equals plain causal attention (identity order, blocks
    J <= I) on the same kernel."""
    w = CASES["gqa2k"]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, hq=w.hq)
    idx, cnt, _ = pbs.select_blocks(qd, perm["k_perm"], perm["kbar_sum"], B, S, "all")
    o_all = pbs.attn_fwd(qd, perm["k_perm"], perm["v_perm"], perm["kpos"], None, idx, cnt, B, S)
    didx, dcnt, _ = pbs.select_blocks(qd, kd, None, B, S, "dense_causal")
    o_dense = pbs.attn_fwd(qd, kd, vd, None, None, didx, dcnt, B, S)
    ref = orc.dense_causal(f64(q), f64(k), f64(v))
    assert_outputs_close(f64(o_all), ref, "all blocks")
    assert_outputs_close(f64(o_dense), ref, "dense causal")
    assert_outputs_close(f64(o_all), f64(o_dense), "all vs dense")


def test_exact_importance_ties_keep_lower_index(dev):
    w = CASES["gqa2k"]
    (_, k, v), (_, kd, vd) = inputs(w, dev)
    g = torch.Generator().manual_seed(5)
    imp = torch.randint(0, 4, (1, 2, 2048), generator=g).float() / 8   # heavy ties
    perm = pbs.permute(imp.to(dev), kd, vd, 128, 512, hq=8)
    np.testing.assert_array_equal(i64(perm["kpos"]), orc.segment_order(imp.double().numpy(), 512))


def test_lse_output(dev):
    w = CASES["d128_b64"]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    idx, cnt, _ = pbs.select_blocks(qd, kd, None, w.block, w.segment, "dense_causal")
    o, lse = pbs.attn_fwd(qd, kd, vd, None, None, idx, cnt, w.block, w.segment, lse=True)
    q64, k64 = f64(q), f64(k)
    sigma = 1.0 / np.sqrt(w.d)
    for g in range(w.hq):
        logits = sigma * q64[0, g] @ k64[0, g].T
        logits = np.where(np.tril(np.ones((w.n, w.n), bool)), logits, -np.inf)
        mx = logits.max(1)
        want = mx + np.log(np.exp(logits - mx[:, None]).sum(1))
        np.testing.assert_allclose(f64(lse)[0, g], want, atol=2e-3)


def test_deterministic(dev):
    w = CASES["ragged"]
    _, (qd, kd, vd) = inputs(w, dev)
    a = pbs.pbs_attention(qd, kd, vd, w.block, w.segment, w.mode, w.param, keep=True)
    b = pbs.pbs_attention(qd, kd, vd, w.block, w.segment, w.mode, w.param, keep=True)
    for key in ("imp", "kpos", "k_perm", "kbar_sum", "cnt", "o"):
        assert torch.equal(a[key], b[key]), key


def test_empty_sequence(dev):
    q = torch.empty(1, 4, 0, 128, dtype=torch.bfloat16, device=dev)
    k = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device=dev)
    o = pbs.pbs_attention(q, k, k, 128, 512)
    assert o.shape == q.shape


def test_device_status_is_clean(dev):
    w = CASES["tiny"]
    _, (qd, kd, vd) = inputs(w, dev)
    pbs.pbs_attention(qd, kd, vd, w.block, w.segment)
    assert pbs.device_status() == 0


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d64_b128", "odd_items", "tiny", "d128_b64",
                                  "s_eq_n", "b64_odd"])
def test_tensor_core_and_warp_mma_forwards_agree(name, dev, monkeypatch):
    """The tcgen05 forward and the warp-MMA forward on the same lists, each
    against the oracle. B = 64 shapes run the kernel whose 128-row tiles pair
    two query blocks (with an odd number of query blocks in b64_odd, the last
    tile's second block lies past the end)."""
    w = CASES[name]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, hq=w.hq)
    idx, cnt, _ = pbs.select_blocks(qd, perm["k_perm"], perm["kbar_sum"], B, S, w.mode, w.param)
    args = (qd, perm["k_perm"], perm["v_perm"], perm["kpos"], None, idx, cnt, B, S)
    o_tc, lse_tc = pbs.attn_fwd(*args, lse=True)
    monkeypatch.setenv("PBS_FORWARD", "mma")
    o_mma, lse_mma = pbs.attn_fwd(*args, lse=True)
    monkeypatch.delenv("PBS_FORWARD")
    ref = orc.attend(f64(q), f64(perm["k_perm"]), f64(perm["v_perm"]), i64(perm["kpos"]), None,
                     i64(idx), i64(cnt), B)
    assert_outputs_close(f64(o_tc), ref, "tcgen05")
    assert_outputs_close(f64(o_mma), ref, "warp mma")
    np.testing.assert_allclose(f64(lse_tc), f64(lse_mma), atol=1e-3)
    assert pbs.device_status() == 0


SCORE_SHAPES = {
    # (batch, hq, hkv, n, d, B): every G*B up to 512 takes the tcgen05 kernel;
    # where G*B is not a multiple of 128 (64, 192) the last 128-row slice of
    # probe rows is half padding
    "r512_d128": (1, 8, 2, 2048, 128, 128),
    "r256_b2": (2, 4, 2, 1280, 128, 128),
    "r384": (1, 6, 2, 1536, 128, 128),
    "r512_d64": (1, 4, 1, 1024, 64, 128),
    # B = 64 probe rows, n % 128 == 64: the last key tile is half past the end
    "r128_b64_tail": (1, 4, 2, 1088, 128, 64),
    "r64_mma": (1, 4, 4, 1024, 128, 64),
    "r64_d64": (1, 1, 1, 1024, 64, 64),
    "r192_b64": (2, 6, 2, 1088, 128, 64),
}


@pytest.mark.parametrize("name", list(SCORE_SHAPES))
def test_score_kernels_against_oracle(name, dev, monkeypatch):
    """Both scoring kernels (tcgen05 and warp-MMA) against the oracle's
    importance, and against each other."""
    b, hq, hkv, n, d, B = SCORE_SHAPES[name]
    w = Workload(name, b, hq, hkv, n, d, B, n, "threshold", 0.9, "uniform", 0.05, seed=3)
    (q, k, _), (qd, kd, _) = inputs(w, dev)
    want = orc.score(f64(q), f64(k), B)
    imp_tc = pbs.score(qd, kd, B)
    monkeypatch.setenv("PBS_SCORE", "mma")
    imp_mma = pbs.score(qd, kd, B)
    monkeypatch.delenv("PBS_SCORE")
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    assert_importance_close(f64(imp_tc), want)
    assert_importance_close(f64(imp_mma), want)
    # the two kernels sum in different orders: agreement to fp32 rounding
    np.testing.assert_allclose(f64(imp_tc), f64(imp_mma), rtol=1e-4, atol=0)


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d64_b128", "odd_items", "s_eq_b"])
@pytest.mark.parametrize("permute_q", [False, True])
def test_two_tile_and_one_tile_forwards_agree(name, permute_q, dev, monkeypatch):
    """The two-tile tcgen05 forward (the default) and the one-tile one on the
    same lists: both against the oracle, and equal to bf16 rounding."""
    w = CASES[name]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, q=qd if permute_q else None, hq=w.hq)
    q_used = perm["q_perm"] if permute_q else qd
    qpos = perm["kpos"] if permute_q else None
    idx, cnt, _ = pbs.select_blocks(q_used, perm["k_perm"], perm["kbar_sum"], B, S, w.mode,
                                    w.param)
    args = (q_used, perm["k_perm"], perm["v_perm"], perm["kpos"], qpos, idx, cnt, B, S)
    o2, lse2 = pbs.attn_fwd(*args, lse=True)
    monkeypatch.setenv("PBS_FORWARD", "tc1")
    o1, lse1 = pbs.attn_fwd(*args, lse=True)
    monkeypatch.delenv("PBS_FORWARD")
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    qpos64 = None if qpos is None else np.repeat(i64(qpos), w.group, axis=1)
    ref = orc.attend(f64(q_used), f64(perm["k_perm"]), f64(perm["v_perm"]), i64(perm["kpos"]),
                     qpos64, i64(idx), i64(cnt), B)
    assert_outputs_close(f64(o2), ref, "two-tile")
    assert_outputs_close(f64(o1), ref, "one-tile")
    assert_outputs_close(f64(o2), f64(o1), "two-tile vs one-tile")
    np.testing.assert_allclose(f64(lse2), f64(lse1), atol=1e-4)


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d64_b128", "odd_items", "d128_b64", "s_eq_n"])
@pytest.mark.parametrize("forward", ["default", "tc1", "mma"])
def test_fused_unpermute_equals_two_calls(name, forward, dev, monkeypatch):
    """pbs_attn_fwd_unpermute writes each row at its query's original
    position: bit for bit the output of pbs_attn_fwd followed by
    pbs_unpermute, with the LSE moved the same way."""
    w = CASES[name]
    if forward != "default":
        monkeypatch.setenv("PBS_FORWARD", forward)
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, q=qd, hq=w.hq)
    idx, cnt, _ = pbs.select_blocks(perm["q_perm"], perm["k_perm"], perm["kbar_sum"], B, S,
                                    w.mode, w.param)
    args = (perm["q_perm"], perm["k_perm"], perm["v_perm"], perm["kpos"], perm["kpos"], idx, cnt,
            B, S)
    o_perm, lse_perm = pbs.attn_fwd(*args, lse=True)
    o_two = pbs.unpermute(o_perm, perm["kpos"], w.hkv, B, S)
    o_one, lse_one = pbs.attn_fwd(*args, lse=True, unpermute=True)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    assert torch.equal(o_one, o_two)
    qpos = np.repeat(i64(perm["kpos"]), w.group, axis=1)
    lse_two = np.empty_like(f64(lse_perm))
    np.put_along_axis(lse_two, qpos, f64(lse_perm), axis=2)
    np.testing.assert_array_equal(f64(lse_one), lse_two)
    # and the path entry point uses it
    o_path = pbs.pbs_attention(qd, kd, vd, B, S, w.mode, w.param, permute_q=True)
    assert torch.equal(o_path, o_one)


def test_fused_unpermute_rejects_output_aliasing_an_input(dev):
    w = CASES["gqa2k"]
    _, (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, q=qd, hq=w.hq)
    idx, cnt, _ = pbs.select_blocks(perm["q_perm"], perm["k_perm"], perm["kbar_sum"], B, S,
                                    w.mode, w.param)
    with pytest.raises(pbs.PbsError):
        pbs.attn_fwd(perm["q_perm"], perm["k_perm"], perm["v_perm"], perm["kpos"], perm["kpos"],
                     idx, cnt, B, S, out=perm["q_perm"], unpermute=True)


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d64_b128", "odd_items", "d128_b64"])
def test_host_buffer_path_against_oracle(name, dev):
    """pbs_attention_host on page-locked host tensors, one KV group at a time
    with the copies overlapped: against the oracle's pipeline (as the device
    path), and close to the device path on the same inputs."""
    w = CASES[name]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o_host = pbs.attention_host(qh, kh, vh, w.block, w.segment, w.mode, w.param)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    ref = orc.pbs_attention(f64(q), f64(k), f64(v), w.block, w.segment, w.mode, w.param)
    assert_outputs_close(f64(o_host), ref["o"], name)
    o_dev = pbs.pbs_attention(qd, kd, vd, w.block, w.segment, w.mode, w.param)
    assert_outputs_close(f64(o_host), f64(o_dev), "host vs device path")


def test_host_buffer_path_many_groups_reuse_both_slots(dev):
    """Eight KV groups over two batches: every slot is reused several times
    and each group's output lands at its own place."""
    w = Workload("groups8", 2, 8, 4, 1024, 128, 128, 256, "topk_frac", 0.5, "uniform", 0.05,
                 seed=11)
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    o_host = pbs.attention_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), w.block,
                                w.segment, w.mode, w.param)
    o_dev = pbs.pbs_attention(qd, kd, vd, w.block, w.segment, w.mode, w.param)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    assert_outputs_close(f64(o_host), f64(o_dev), "host vs device path")


@pytest.mark.parametrize("name", ["gqa2k", "d128_b64", "groups8"])
def test_host_buffer_path_steps_of_query_heads(name, dev, monkeypatch):
    """The host path streams each KV group's query heads in steps (selection,
    forward and copies per step). Every step size gives the same output bit
    for bit: a query head's lists and rows do not depend on which heads share
    its launch."""
    w = CASES.get(name) or Workload("groups8", 2, 8, 4, 1024, 128, 128, 256, "topk_frac", 0.5,
                                    "uniform", 0.05, seed=11)
    q, k, v, _ = make_inputs(w)
    q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    outs = {}
    for step in (w.group, 2, 1):
        if w.group % step:
            continue
        monkeypatch.setenv("PBS_HOST_STEP_HEADS", str(step))
        o = pbs.attention_host(q, k, v, w.block, w.segment, w.mode, w.param)
        torch.cuda.synchronize()  # the output is valid once the stream has synchronised
        assert pbs.device_status() == 0
        outs[step] = o.clone()
    for step, o in outs.items():
        assert torch.equal(o, outs[w.group]), f"step of {step} heads"


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d64_b128", "odd_items", "d128_b64", "tiny"])
def test_broadcast_forward_writes_every_buffer(name, dev):
    """pbs_attn_fwd_bcast writes the forward's rows into every buffer at the
    given head offset (as each rank of a head-sharded run writes its heads
    into its own and its peers' outputs) and nothing else; the rows are bit
    for bit pbs_attn_fwd's."""
    w = CASES[name]
    _, (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, hq=w.hq)
    idx, cnt, _ = pbs.select_blocks(qd, perm["k_perm"], perm["kbar_sum"], B, S, w.mode, w.param)
    args = (qd, perm["k_perm"], perm["v_perm"], perm["kpos"])
    o_ref = pbs.attn_fwd(*args, None, idx, cnt, B, S)
    b, hq, n, d = qd.shape
    sentinel = torch.tensor(-7.0, dtype=torch.bfloat16)
    for n_out, total, offset in ((1, hq, 0), (3, 3 * hq, hq), (2, 2 * hq + 1, hq + 1)):
        outs = [torch.full((b, total, n, d), -7.0, dtype=torch.bfloat16, device=dev)
                for _ in range(n_out)]
        pbs.attn_fwd_bcast(*args, idx, cnt, B, S, outs, head_offset=offset)
        torch.cuda.synchronize()
        assert pbs.device_status() == 0
        for o in outs:
            assert torch.equal(o[:, offset:offset + hq], o_ref)
            rest = torch.cat([o[:, :offset], o[:, offset + hq:]], dim=1)
            assert bool((rest.cpu() == sentinel).all())


@pytest.mark.parametrize("mode,param", [("threshold", 1.0), ("threshold", 0.01),
                                        ("topk_frac", 1.0), ("topk_frac", 0.01)])
def test_selection_extremes_against_oracle(mode, param, dev):
    """The ends of the sparsity parameter: tau = 1 keeps blocks until the
    whole mass (every admissible block unless the last ones carry no mass in
    fp64), f = 1 keeps k = I + 1 blocks, and tiny tau or f keep the own
    segment alone (it is always kept and already holds more than tau, or
    more blocks than k). Lists bit for bit against the oracle, the top-k
    counts against their closed form, outputs within the forward's
    tolerance."""
    w = CASES["gqa2k"].with_(mode=mode, param=param)
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    imp = pbs.score(qd, kd, B)
    perm = pbs.permute(imp, kd, vd, B, S, hq=w.hq)
    kp = perm["k_perm"]
    idx, cnt, _ = pbs.select_blocks(qd, kp, perm["kbar_sum"], B, S, mode, param)
    qb, kb = orc.block_means(f64(q), B), orc.block_means(f64(kp), B)
    ref_idx, ref_cnt, margin = orc.select_blocks(qb, kb, S // B, mode, param, None, w.group)
    # rows decided by a gap below 1e-12 (tau = 1 reaches the whole mass only
    # up to rounding) are checked for validity, every other row bit for bit
    n_amb = compare_lists(idx, cnt, ref_idx, ref_cnt, margin,
                          scores=orc.block_scores(qb, kb, None, w.group), spb=S // B, mode=mode,
                          param=param)
    print(f"{mode} {param}: {n_amb} of {ref_cnt.size} rows are near-ties, checked for validity")
    c = i64(cnt)
    spb, nb = S // B, w.nb
    I = np.arange(nb)
    own = np.minimum(spb, nb - (I // spb) * spb)
    if mode == "topk_frac":  # own segment, plus k - own earlier blocks
        k_i = np.maximum(1, np.floor(param * (I + 1))).astype(np.int64)
        want = own + np.minimum((I // spb) * spb, np.maximum(0, k_i - own))
        assert np.array_equal(c, np.broadcast_to(want, c.shape))
    if param == 0.01:
        assert np.array_equal(c, np.broadcast_to(own, c.shape))
    o = pbs.attn_fwd(qd, kp, perm["v_perm"], perm["kpos"], None, idx, cnt, B, S)
    ref_o = orc.attend(f64(q), f64(kp), f64(perm["v_perm"]), i64(perm["kpos"]), None, i64(idx),
                       i64(cnt), B)
    assert_outputs_close(f64(o), ref_o, f"{mode} {param}")
    assert pbs.device_status() == 0
