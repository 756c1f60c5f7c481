"""The head-sharded path on one GPU, shard by shard.

With the KV groups of one sequence split over `world` ranks (the pages'
tensor-parallel runs at 256K and 512K, sciencestack.ai Figure 3 caption),
rank r computes its KV heads [r*hkv/world, (r+1)*hkv/world) and their query
heads, and its forward writes every output row into every rank's
whole-output buffer at head offset r*hq/world (pbs_attn_fwd_bcast). Here each
pretend rank runs on the same device, in turn, into `world` local buffers.

Checked: with the unsharded importance, every buffer assembled from the
shards equals the unsharded path's output bit for bit (the permutation,
selection and forward are per KV group and per query head); each shard's own
scoring agrees with the unsharded importance within the scoring tolerance (a
launch over fewer KV heads splits the keys over more CTAs, so the last bits
may differ); and the whole sharded path, each shard on its own importance,
matches the oracle's pipeline: key orders differ only inside runs of
near-equal importance, outputs of sampled query blocks within the forward's
tolerance.
"""
import numpy as np
import pytest
import torch

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200.workloads import Workload, make_inputs
from oracle import pbs_oracle as orc
from pbs_testutil import (IMP_RTOL, assert_outputs_close, f64, i64, order_differences)

pytestmark = pytest.mark.gpu

W = Workload("shard4", 1, 16, 4, 2048, 128, 128, 512, "topk_frac", 0.3, "per_segment", 0.02,
             seed=9)


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda", 0)


def shard_steps(q, k, v, w, imp, outs, head_offset):
    B, S = w.block, w.segment
    perm = pbs.permute(imp, k, v, B, S, hq=q.shape[1])
    idx, cnt, _ = pbs.select_blocks(q, perm["k_perm"], perm["kbar_sum"], B, S, w.mode, w.param)
    pbs.attn_fwd_bcast(q, perm["k_perm"], perm["v_perm"], perm["kpos"], idx, cnt, B, S, outs,
                       head_offset=head_offset)
    return perm, idx, cnt


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_path_equals_unsharded_and_oracle(world, dev):
    w = W
    G, per = w.group, w.hkv // world
    q, k, v, _ = make_inputs(w, dev)
    full = pbs.pbs_attention(q, k, v, w.block, w.segment, w.mode, w.param, keep=True)
    torch.cuda.synchronize()
    shape = (w.batch, w.hq, w.n, w.d)

    # the unsharded importance, shard by shard: bit for bit
    outs = [torch.full(shape, -3.0, dtype=torch.bfloat16, device=dev) for _ in range(world)]
    for r in range(world):
        h0, h1 = r * per, (r + 1) * per
        shard_steps(q[:, h0 * G:h1 * G].contiguous(), k[:, h0:h1].contiguous(),
                    v[:, h0:h1].contiguous(), w, full["imp"][:, h0:h1].contiguous(), outs,
                    h0 * G)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    for o in outs:
        assert torch.equal(o, full["o"])

    # each shard on its own importance
    outs = [torch.full(shape, -3.0, dtype=torch.bfloat16, device=dev) for _ in range(world)]
    imp_s, kpos_s, idx_s, cnt_s, kp_s, vp_s = [], [], [], [], [], []
    for r in range(world):
        h0, h1 = r * per, (r + 1) * per
        qs, ks, vs = (q[:, h0 * G:h1 * G].contiguous(), k[:, h0:h1].contiguous(),
                      v[:, h0:h1].contiguous())
        imp = pbs.score(qs, ks, w.block, w.segment)
        perm, idx, cnt = shard_steps(qs, ks, vs, w, imp, outs, h0 * G)
        imp_s.append(imp), kpos_s.append(perm["kpos"]), idx_s.append(idx), cnt_s.append(cnt)
        kp_s.append(perm["k_perm"]), vp_s.append(perm["v_perm"])
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    imp_sh = torch.cat(imp_s, dim=1)
    rel = ((imp_sh.double() - full["imp"].double()).abs() / full["imp"].double().abs()).max()
    assert rel.item() <= IMP_RTOL

    ref = orc.pbs_attention(f64(q), f64(k), f64(v), w.block, w.segment, w.mode, w.param)
    n_diff = order_differences(i64(torch.cat(kpos_s, dim=1)), ref["kpos"], ref["imp"])
    print(f"world {world}: {n_diff} key slots differ from the oracle inside near-ties")
    # sampled query blocks of every head, against the oracle fed the shard's
    # own order and lists (the forward's parity), and the oracle's pipeline
    blocks = [0, 3, 4, 9, w.nb - 1]
    for g in range(w.hq):
        r, gl = divmod(g, per * G)
        hk = gl // G
        got = np.stack([f64(outs[0][0, g, I * w.block:(I + 1) * w.block]) for I in blocks])
        want = orc.attend_blocks(f64(q[:, g:g + 1]), f64(kp_s[r][:, hk:hk + 1]),
                                 f64(vp_s[r][:, hk:hk + 1]), i64(kpos_s[r][:, hk:hk + 1]), None,
                                 i64(idx_s[r][:, gl:gl + 1]), i64(cnt_s[r][:, gl:gl + 1]),
                                 w.block, [(0, 0, I) for I in blocks])
        assert_outputs_close(got, want, f"head {g}")
        pipe = np.stack([ref["o"][0, g, I * w.block:(I + 1) * w.block] for I in blocks])
        assert_outputs_close(got, pipe, f"head {g} vs the oracle's pipeline")
