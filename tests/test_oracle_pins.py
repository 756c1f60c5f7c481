"""Pins for the CPU oracle against facts fixed by the mathematics.

Each test ties one oracle step to something other than the oracle itself: a
library routine (torch's scaled_dot_product_attention), a closed form, an
invariant of attention (Lemma 3.1, Lemma 3.2, Theorem 3.3 of "Sparser
Block-Sparse Attention via Token Permutation"), brute-force enumeration on
tiny inputs, or a hand-worked example in the style of that paper's Figure 1
(B = 1, S = 4).
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import pbs_oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore")


def rand_qkv(seed, b=1, hq=2, hkv=1, n=64, d=16):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((b, hq, n, d))
    k = rng.standard_normal((b, hkv, n, d))
    v = rng.standard_normal((b, hkv, n, d))
    return q, k, v


def sdpa(q, k, v, mask=None, causal=False, scale=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    out = F.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else t(mask),
        is_causal=causal, scale=scale, enable_gqa=True)
    return out.numpy()


def within_segment_perm(rng, b, h, n, segment):
    pos = np.empty((b, h, n), dtype=np.int64)
    for bi in range(b):
        for hi in range(h):
            for s0 in range(0, n, segment):
                pos[bi, hi, s0:s0 + segment] = s0 + rng.permutation(segment)
    return pos


# ---------------------------------------------------------------- attention
def test_dense_causal_matches_library():
    q, k, v = rand_qkv(0, b=2, hq=4, hkv=2, n=48, d=8)
    np.testing.assert_allclose(orc.dense_causal(q, k, v), sdpa(q, k, v, causal=True),
                               rtol=0, atol=1e-12)


def test_all_blocks_identity_is_dense_causal():
    q, k, v = rand_qkv(1, hq=4, hkv=2, n=64, d=8)
    nb = 8
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, 4, nb, 1))
    cnt = np.full((1, 4, nb), nb, dtype=np.int32)
    o = orc.attend(q, k, v, None, None, idx, cnt, 8)
    np.testing.assert_allclose(o, sdpa(q, k, v, causal=True), atol=1e-12)


def test_theorem_3_3_permute_attend_unpermute():
    """All blocks kept: permuting Q, K, V inside segments, attending with the
    carried positions and inverting the query order gives dense causal."""
    rng = np.random.default_rng(2)
    q, k, v = rand_qkv(2, hq=4, hkv=2, n=64, d=8)
    block, segment = 4, 16
    kpos = within_segment_perm(rng, 1, 2, 64, segment)
    perm = {"kpos": kpos, "k_perm": orc.gather_rows(k, kpos),
            "v_perm": orc.gather_rows(v, kpos)}
    qpos = np.repeat(kpos, 2, axis=1)
    q_perm = orc.gather_rows(q, qpos)
    nb = 64 // block
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, 4, nb, 1))
    cnt = np.full((1, 4, nb), nb, dtype=np.int32)
    o_perm = orc.attend(q_perm, perm["k_perm"], perm["v_perm"], kpos, qpos, idx, cnt, block)
    np.testing.assert_allclose(orc.unpermute(o_perm, qpos), sdpa(q, k, v, causal=True),
                               atol=1e-12)


def test_lemma_3_2_query_equivariance():
    """Permuting the query rows permutes the output rows the same way."""
    rng = np.random.default_rng(3)
    q, k, v = rand_qkv(3, hq=2, hkv=2, n=32, d=8)
    nb = 4
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, 2, nb, 1))
    cnt = np.full((1, 2, nb), nb, dtype=np.int32)
    qpos = within_segment_perm(rng, 1, 2, 32, 32)
    o = orc.attend(q, k, v, None, None, idx, cnt, 8)
    o_p = orc.attend(orc.gather_rows(q, qpos), k, v, None, qpos, idx, cnt, 8)
    np.testing.assert_allclose(o_p, orc.gather_rows(o, qpos), atol=1e-12)


def test_lemma_3_1_key_value_invariance():
    """Reordering (key, value, position) triples inside each block leaves the
    output unchanged for any block selection."""
    rng = np.random.default_rng(4)
    q, k, v = rand_qkv(4, hq=2, hkv=1, n=64, d=8)
    block, segment = 8, 32
    imp = rng.random((1, 1, 64))
    perm = orc.permute(imp, k, v, segment)
    idx, cnt, _ = orc.select_blocks(orc.block_means(q, block),
                                    orc.block_means(perm["k_perm"], block),
                                    segment // block, "threshold", 0.5, None, 2)
    o1 = orc.attend(q, perm["k_perm"], perm["v_perm"], perm["kpos"], None, idx, cnt, block)
    inner = within_segment_perm(rng, 1, 1, 64, block)
    o2 = orc.attend(q, orc.gather_rows(perm["k_perm"], inner),
                    orc.gather_rows(perm["v_perm"], inner),
                    np.take_along_axis(perm["kpos"], inner, axis=2), None, idx, cnt, block)
    np.testing.assert_allclose(o1, o2, atol=1e-12)


def test_identity_permutation_is_plain_block_sparse():
    """kpos = identity: the output is causal attention restricted to the kept
    blocks, i.e. the library routine with that token-level mask."""
    q, k, v = rand_qkv(5, hq=2, hkv=1, n=64, d=8)
    block, segment = 8, 16
    idx, cnt, _ = orc.select_blocks(orc.block_means(q, block), orc.block_means(k, block),
                                    segment // block, "topk_frac", 0.3, None, 2)
    o = orc.attend(q, k, v, None, None, idx, cnt, block)
    for g in range(2):
        blockmask = np.zeros((8, 8), dtype=bool)
        for i in range(8):
            blockmask[i, idx[0, g, i, :cnt[0, g, i]]] = True
        mask = np.kron(blockmask, np.ones((block, block), dtype=bool)) & np.tril(
            np.ones((64, 64), dtype=bool))
        ref = sdpa(q[:, g:g + 1], k, v, mask=mask)
        np.testing.assert_allclose(o[:, g:g + 1], ref, atol=1e-12)


def test_attend_blocks_is_masked_library_attention_on_the_permuted_sequence():
    """attend_blocks on a within-segment key order and grouped heads: each
    requested query block's rows equal the library routine on the permuted
    K, V with the token mask 'key block kept and original key position <=
    query position', query head g reading KV head g // G."""
    rng = np.random.default_rng(23)
    q, k, v = rand_qkv(23, b=2, hq=4, hkv=2, n=64, d=8)
    block, segment = 8, 32
    kpos = within_segment_perm(rng, 2, 2, 64, segment)
    kp = orc.gather_rows(k, kpos)
    vp = orc.gather_rows(v, kpos)
    idx, cnt, _ = orc.select_blocks(orc.block_means(q, block), orc.block_means(kp, block),
                                    segment // block, "threshold", 0.7, None, 2)
    want_blocks = [(0, 0, 7), (0, 3, 2), (1, 1, 4), (1, 2, 0), (1, 3, 5)]
    got = orc.attend_blocks(q, kp, vp, kpos, None, idx, cnt, block, want_blocks)
    for t, (bi, g, blk) in enumerate(want_blocks):
        h = g // 2
        blockmask = np.zeros((8, 8), dtype=bool)
        for i in range(8):
            blockmask[i, idx[bi, g, i, :cnt[bi, g, i]]] = True
        mask = np.kron(blockmask, np.ones((block, block), dtype=bool)) & \
            (kpos[bi, h][None, :] <= np.arange(64)[:, None])
        ref = sdpa(q[bi:bi + 1, g:g + 1], kp[bi:bi + 1, h:h + 1], vp[bi:bi + 1, h:h + 1],
                   mask=mask)[0, 0]
        np.testing.assert_allclose(got[t], ref[blk * block:(blk + 1) * block], atol=1e-12)


def test_block_flops_counts_the_multiply_adds_of_a_block_loop():
    """block_flops is twice the multiply-adds that a block-by-block forward
    performs: a plain loop over the kept blocks that counts every product it
    forms (q.k per logit, p*v per output element), and whose output matches
    attend, so that the count is of real work."""
    q, k, v = rand_qkv(29, hq=2, hkv=1, n=32, d=4)
    block, segment = 8, 16
    idx, cnt, _ = orc.select_blocks(orc.block_means(q, block), orc.block_means(k, block),
                                    segment // block, "topk_frac", 0.5, None, 2)
    sigma = orc.resolve_scale(None, 4)
    macs = 0
    out = np.zeros((1, 2, 32, 4))
    for g in range(2):
        for I in range(4):
            rows = range(I * block, (I + 1) * block)
            kept = idx[0, g, I, :cnt[0, g, I]]
            logits = np.full((block, 32), -np.inf)
            for J in kept:
                for r in rows:
                    for c in range(J * block, (J + 1) * block):
                        acc = 0.0
                        for e in range(4):
                            acc += q[0, g, r, e] * k[0, 0, c, e]
                            macs += 1
                        if c <= r:
                            logits[r - I * block, c] = sigma * acc
            w = np.exp(logits - logits.max(axis=1, keepdims=True))
            w /= w.sum(axis=1, keepdims=True)
            for J in kept:
                for r in rows:
                    for c in range(J * block, (J + 1) * block):
                        for e in range(4):
                            out[0, g, r, e] += w[r - I * block, c] * v[0, 0, c, e]
                            macs += 1
    np.testing.assert_allclose(out, orc.attend(q, k, v, None, None, idx, cnt, block), atol=1e-12)
    assert orc.block_flops(cnt, block, 4) == 2 * macs


def test_single_segment_is_dense_causal():
    """S = N: every block is in the on-diagonal segment, so the whole path
    (with its permutation) reproduces dense causal attention."""
    q, k, v = rand_qkv(6, hq=4, hkv=2, n=64, d=8)
    for mode, param in (("threshold", 0.5), ("topk_frac", 0.1)):
        res = orc.pbs_attention(q, k, v, 8, 64, mode, param)
        np.testing.assert_allclose(res["o"], sdpa(q, k, v, causal=True), atol=1e-12)
        res = orc.pbs_attention(q, k, v, 8, 64, mode, param, permute_q=True)
        np.testing.assert_allclose(res["o"], sdpa(q, k, v, causal=True), atol=1e-12)


def test_segment_equal_block_selection_ignores_permutation():
    """S = B: a block is a segment, so its mean key (and the lists) cannot
    depend on the order inside it."""
    q, k, v = rand_qkv(7, hq=2, hkv=1, n=64, d=8)
    rng = np.random.default_rng(7)
    imp = rng.random((1, 1, 64))
    perm = orc.permute(imp, k, v, 8)
    a = orc.select_blocks(orc.block_means(q, 8), orc.block_means(perm["k_perm"], 8), 1,
                          "threshold", 0.8, None, 2)
    b = orc.select_blocks(orc.block_means(q, 8), orc.block_means(k, 8), 1,
                          "threshold", 0.8, None, 2)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("segment", [32, 64])        # 64: shorter last segment
def test_all_mode_after_permutation_is_dense_causal(segment):
    q, k, v = rand_qkv(8, hq=4, hkv=1, n=96, d=8)
    res = orc.pbs_attention(q, k, v, 8, segment, "all", 0.0)
    np.testing.assert_allclose(res["o"], sdpa(q, k, v, causal=True), atol=1e-12)
    res = orc.pbs_attention(q, k, v, 8, segment, "all", 0.0, permute_q=True)
    np.testing.assert_allclose(res["o"], sdpa(q, k, v, causal=True), atol=1e-12)


# ---------------------------------------------------------------- scoring
def test_score_equals_library_attention_probabilities():
    """Attention against V = identity returns the probability matrix itself,
    so the mean over the probe rows must equal the importance."""
    q, k, _ = rand_qkv(9, b=2, hq=4, hkv=2, n=40, d=8)
    block = 8
    imp = orc.score(q, k, block)
    n = 40
    eye = np.eye(n)[None, None]
    mask = np.arange(n)[None, :] <= np.arange(n - block, n)[:, None]
    for bi in range(2):
        for h in range(2):
            rows = q[bi:bi + 1, 2 * h:2 * h + 2, n - block:]
            p = sdpa(rows, k[bi:bi + 1, h:h + 1], eye, mask=mask)  # [1, 2, block, n]
            np.testing.assert_allclose(imp[bi, h], p.reshape(-1, n).mean(0), atol=1e-14)


def test_score_closed_forms():
    # one probe row that sees exactly one key
    q = np.ones((1, 1, 1, 4))
    k = np.ones((1, 1, 1, 4))
    assert orc.score(q, k, 1)[0, 0, 0] == 1.0
    # identical keys: row at offset r sees r+1 keys uniformly
    n = block = 6
    q, _, _ = rand_qkv(10, hq=1, hkv=1, n=n, d=4)
    k = np.ones((1, 1, n, 4))
    want = [sum(1.0 / (r + 1) for r in range(j, n)) / n for j in range(n)]
    np.testing.assert_allclose(orc.score(q, k, block)[0, 0], want, atol=1e-15)
    # rows sum to one; keys after the last position carry no weight
    q, k, _ = rand_qkv(11, hq=4, hkv=1, n=32, d=8)
    imp = orc.score(q, k, 8)
    assert abs(imp.sum() - 1.0) < 1e-12


# ------------------------------------------------------------- permutation
def test_segment_order_sorts_descending_with_stable_ties():
    rng = np.random.default_rng(12)
    imp = rng.random((2, 3, 48)).round(1)        # many exact ties
    kpos = orc.segment_order(imp, 16)
    for bi in range(2):
        for h in range(3):
            for s0 in range(0, 48, 16):
                seg = kpos[bi, h, s0:s0 + 16]
                assert sorted(seg.tolist()) == list(range(s0, s0 + 16))
                vals = imp[bi, h, seg]
                assert np.all(vals[:-1] >= vals[1:])
                for p in range(15):
                    if vals[p] == vals[p + 1]:
                        assert seg[p] < seg[p + 1]


def test_figure1_style_worked_example():
    """B = 1, S = 4, N = 8, d = 1 (the setting of Figure 1), worked by hand.

    All queries are 1, so the last row's logits are the keys themselves and
    the importance is softmax(k). Keys [0.5, 2, -1, 2 | 1, 0, 3, -2]:
    segment 0 sorts to original indices [1, 3, 0, 2] (tie 2 = 2 keeps 1
    before 3), segment 1 to [6, 4, 5, 7]. Block scores of query block 7 are
    the permuted keys [2, 2, .5, -1, 3, 1, 0, -2]; the own segment holds
    (e^3 + e + 1 + e^-2) / Z = 0.5877 of the mass, so tau = 0.9 adds slot 0
    (mass 0.7691) and slot 1 (0.9505) and stops.
    """
    k = np.array([0.5, 2, -1, 2, 1, 0, 3, -2]).reshape(1, 1, 8, 1)
    q = np.ones((1, 1, 8, 1))
    v = np.arange(8, dtype=float).reshape(1, 1, 8, 1)
    res = orc.pbs_attention(q, k, v, 1, 4, "threshold", 0.9)
    assert res["kpos"][0, 0].tolist() == [1, 3, 0, 2, 6, 4, 5, 7]
    lists = [res["idx"][0, 0, i, :res["cnt"][0, 0, i]].tolist() for i in range(8)]
    assert lists[:4] == [[0, 1, 2, 3]] * 4
    assert lists[7] == [0, 1, 4, 5, 6, 7]
    # row 7 attends to original keys 1, 3 (slots 0, 1) and 4..7
    ks = [2, 2, 1, 0, 3, -2]
    vs = [1, 3, 4, 5, 6, 7]
    z = sum(math.exp(x) for x in ks)
    o7 = sum(math.exp(x) * y for x, y in zip(ks, vs)) / z
    assert abs(res["o"][0, 0, 7, 0] - o7) < 1e-12
    # top-k with f = 0.75: k_I = floor(0.75 (I+1)) -> 3, 4, 5, 6 for I = 4..7
    res = orc.pbs_attention(q, k, v, 1, 4, "topk_frac", 0.75)
    lists = [res["idx"][0, 0, i, :res["cnt"][0, 0, i]].tolist() for i in range(8)]
    assert lists[4:] == [[4, 5, 6, 7], [4, 5, 6, 7], [0, 4, 5, 6, 7], [0, 1, 4, 5, 6, 7]]
    # segment 0 under top-k: k_I = max(1, floor(.75 (I+1))) < 4 = |own segment|
    assert lists[:4] == [[0, 1, 2, 3]] * 4


# --------------------------------------------------------------- selection
def _rows_of(q, k, block, segment, seed):
    idx = orc.block_means(q, block)
    kb = orc.block_means(k, block)
    return idx, kb


def test_block_score_is_mean_of_token_logits():
    """sigma * mean(Q_I) . mean(K_J) = mean over the B x B token logits."""
    q, k, _ = rand_qkv(13, hq=1, hkv=1, n=32, d=8)
    B = 8
    qb, kb = orc.block_means(q, B), orc.block_means(k, B)
    sigma = orc.resolve_scale(None, 8)
    tok = sigma * q[0, 0] @ k[0, 0].T
    for i in range(4):
        for j in range(4):
            want = tok[i * B:(i + 1) * B, j * B:(j + 1) * B].mean()
            assert abs(sigma * qb[0, 0, i] @ kb[0, 0, j] - want) < 1e-13


def test_block_scores_map_query_heads_to_their_kv_heads():
    """block_scores[b, g, I, J] is the mean of the B x B token logits of
    query head g against KV head g // G (grouped-query attention: G
    consecutive query heads share one KV head), for every pair, batch and
    head."""
    q, k, _ = rand_qkv(17, hq=6, hkv=3, n=32, d=8, b=2)
    B, G = 8, 2
    sigma = orc.resolve_scale(None, 8)
    a = orc.block_scores(orc.block_means(q, B), orc.block_means(k, B), None, G)
    assert a.shape == (2, 6, 4, 4)
    for bi in range(2):
        for g in range(6):
            tok = sigma * q[bi, g] @ k[bi, g // G].T
            want = tok.reshape(4, B, 4, B).mean(axis=(1, 3))
            np.testing.assert_allclose(a[bi, g], want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("tau", [0.3, 0.6, 0.9, 0.97])
def test_threshold_selection_brute_force(tau):
    """Among all subsets T of earlier-segment blocks whose mass with the own
    segment reaches tau, the kept set is the one of least size and, at that
    size, of largest mass."""
    rng = np.random.default_rng(int(tau * 100))
    spb, nseg = 2, 4
    nb = spb * nseg
    for trial in range(6):
        a_all = rng.standard_normal(nb) * 1.5
        for i in range(nb):
            seg = i // spb
            adm = (seg + 1) * spb
            a = a_all[:adm]
            kept, _ = orc.select_row(a, i, spb, "threshold", tau)
            pi = np.exp(a - a.max())
            pi /= pi.sum()
            forced = set(range(seg * spb, adm))
            earlier = range(seg * spb)
            best = None
            for r in range(len(earlier) + 1):
                for t in itertools.combinations(earlier, r):
                    m = pi[list(forced | set(t))].sum()
                    if m >= np.float32(tau) and (best is None or m > best[1]):
                        best = (set(t), m)
                if best is not None:
                    break
            if best is None:          # tau unreachable: everything admissible
                best = (set(earlier), 1.0)
            assert set(kept.tolist()) == forced | best[0]


@pytest.mark.parametrize("frac", [0.1, 0.25, 0.5, 0.9])
def test_topk_selection_brute_force(frac):
    rng = np.random.default_rng(int(frac * 100))
    spb, nseg = 2, 4
    nb = spb * nseg
    for trial in range(4):
        a_all = rng.standard_normal(nb)
        for i in range(nb):
            seg = i // spb
            a = a_all[:(seg + 1) * spb]
            kept, _ = orc.select_row(a, i, spb, "topk_frac", frac)
            k_i = max(1, math.floor(float(np.float32(frac)) * (i + 1)))
            extra = min(seg * spb, max(0, k_i - spb))
            best = max(itertools.combinations(range(seg * spb), extra),
                       key=lambda t: sum(a[list(t)]))
            assert set(kept.tolist()) == set(range(seg * spb, (seg + 1) * spb)) | set(best)


def _kept(a, i, spb, mode, tau):
    return tuple(orc.select_row(a, i, spb, mode, tau)[0].tolist())


def _perturbations(a, tau, mode, delta):
    """Every single move of size delta of what the decision reads: tau up or
    down (THRESHOLD), and each admissible block score up or down."""
    if mode == "threshold":
        for s in (1.0, -1.0):
            yield a, tau + s * delta
    for j in range(len(a)):
        for s in (1.0, -1.0):
            b = a.copy()
            b[j] += s * delta
            yield b, tau


@pytest.mark.parametrize("mode,param", [("threshold", 0.3), ("threshold", 0.6),
                                        ("threshold", 0.9), ("threshold", 0.999),
                                        ("threshold", 1.0), ("topk_frac", 0.25),
                                        ("topk_frac", 0.5), ("topk_frac", 0.75)])
def test_selection_margin_is_the_distance_to_the_next_decision(mode, param):
    """The margin select_row reports is what the GPU comparison trusts to
    tell decided rows from near-ties. Pinned by brute force: moving tau or any
    one block score by 0.99 x the margin keeps the kept set, and some such
    move by 1.01 x the margin changes it (so the margin is neither too small
    nor too large). An infinite margin means no move changes the set. Scores
    are spread so that every finite margin is far above the float32 rounding
    of tau."""
    rng = np.random.default_rng(int(param * 1000) + len(mode))
    spb, nseg = 2, 10
    nb = spb * nseg
    tested = {"finite": 0, "inf": 0}
    for trial in range(12):
        a_all = rng.standard_normal(nb) * 1.5
        if param == 1.0:     # blocks whose mass is below fp64 resolution at 1
            a_all[rng.integers(0, nb, 3)] -= 45.0
        for i in range(nb):
            a = a_all[:(i // spb + 1) * spb]
            kept, margin = orc.select_row(a, i, spb, mode, param)
            kept = tuple(kept.tolist())
            tau = float(np.float32(param))
            if not math.isfinite(margin):
                tested["inf"] += 1
                for delta in (0.5, 5.0):
                    for b, t in _perturbations(a, tau, mode, delta):
                        assert _kept(b, i, spb, mode, t) == kept, (i, delta)
                continue
            if margin < 1e-5:
                continue       # a near-tie: reported, not compared, on the GPU
            tested["finite"] += 1
            for b, t in _perturbations(a, tau, mode, 0.99 * margin):
                assert _kept(b, i, spb, mode, t) == kept, (i, margin)
            assert any(_kept(b, i, spb, mode, t) != kept
                       for b, t in _perturbations(a, tau, mode, 1.01 * margin)), (i, margin)
    assert tested["finite"] >= 15 and tested["inf"] >= 12, tested


def test_selection_margin_of_an_exhausted_threshold_walk():
    """tau = 1 and a row whose masses, added in the walk's order, stay just
    below 1 in fp64: every earlier block is taken without reaching tau, and
    the decision flips once tau drops to the mass before the last block, so
    that distance is the margin (not +inf)."""
    rng = np.random.default_rng(21)
    for _ in range(1000):
        a = rng.standard_normal(6)                     # query block 4, spb 2
        pi = np.exp(a - a.max())
        pi /= pi.sum()
        order = np.argsort(-a[:4], kind="stable")
        walk = pi[4:].sum() + np.cumsum(pi[order])
        if walk[-1] < 1.0 and walk[-2] < 1.0:
            break
    else:
        pytest.fail("no row whose fp64 walk stays below 1")
    kept, margin = orc.select_row(a, 4, 2, "threshold", 1.0)
    assert kept.tolist() == [0, 1, 2, 3, 4, 5]
    assert margin == 1.0 - walk[-2]
    assert _kept(a, 4, 2, "threshold", 1.0 - 1.01 * margin) != tuple(kept.tolist())


def test_shorter_last_segment_forces_its_own_blocks():
    q, k, v = rand_qkv(16, hq=2, hkv=1, n=96, d=8)
    res = orc.pbs_attention(q, k, v, 8, 64, "topk_frac", 0.05)
    for i in range(8, 12):          # query blocks of the 4-block last segment
        assert res["idx"][0, 0, i, :res["cnt"][0, 0, i]].tolist() == [8, 9, 10, 11]
    assert res["kpos"][0, 0, 64:].min() == 64


def test_select_lists_are_ascending_and_admissible():
    q, k, v = rand_qkv(14, hq=4, hkv=2, n=128, d=8)
    res = orc.pbs_attention(q, k, v, 8, 32, "threshold", 0.9)
    idx, cnt = res["idx"], res["cnt"]
    for g in range(4):
        for i in range(16):
            lst = idx[0, g, i, :cnt[0, g, i]]
            assert np.all(np.diff(lst) > 0)
            seg = i // 4
            assert set(range(seg * 4, seg * 4 + 4)) <= set(lst.tolist())
            assert lst.max() < (seg + 1) * 4
            assert np.all(idx[0, g, i, cnt[0, g, i]:] == -1)


def test_bf16_block_sums_are_exact():
    """fp64 block sums of bf16 inputs are exact for the synthetic workloads,
    so any summation order gives the same bits."""
    from long_context_sparse_segment_b200.workloads import WORKLOADS, make_inputs
    q, k, v, _ = make_inputs(WORKLOADS["tiny"])
    x = k.double().numpy()[0, 0]
    B = 64
    for j in range(0, 1024, B):
        for t in range(0, 64, 7):
            exact = sum(Fraction(float(val)) for val in x[j:j + B, t])
            assert Fraction(float(x[j:j + B, t].sum())) == exact


def test_unpermute_inverts_gather():
    rng = np.random.default_rng(15)
    x = rng.standard_normal((2, 3, 32, 4))
    pos = within_segment_perm(rng, 2, 3, 32, 8)
    np.testing.assert_array_equal(orc.unpermute(orc.gather_rows(x, pos), pos), x)


# ---------------------------------------------------------------- diagnostics
def _diag_inputs(seed=4, n=256, block=16, segment=64, hq=2, hkv=1, d=16):
    g = np.random.default_rng(seed)
    q = g.standard_normal((1, hq, n, d))
    k = g.standard_normal((1, hkv, n, d))
    v = g.standard_normal((1, hkv, n, d))
    return q, k, v, block, segment


def test_block_mass_rows_sum_to_one_and_respect_causality():
    q, k, _, B, S = _diag_inputs()
    m = orc.block_mass(q, k, None, B)
    np.testing.assert_allclose(m.sum(-1), 1.0, atol=1e-12)
    nb = m.shape[-1]
    assert np.all(m[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] == 0)


def test_block_mass_is_attention_probability_mass():
    # brute force from torch's attention probabilities (V = identity)
    q, k, _, B, S = _diag_inputs(n=64, block=8, hq=1, d=8)
    n = q.shape[2]
    eye = torch.eye(n, dtype=torch.float64)[None, None]
    probs = sdpa(q, k, eye, causal=True)[0, 0]               # [n, n] = P
    want = probs.reshape(n // 8, 8, n // 8, 8).sum(axis=(1, 3)) / 8
    np.testing.assert_allclose(orc.block_mass(q, k, None, 8)[0, 0], want, atol=1e-12)


def test_block_mass_permutation_moves_mass_only_inside_segments():
    # Lemma 3.1: the probabilities do not change, only the blocks they fall in;
    # a segment's total mass is the same with and without permutation
    q, k, v, B, S = _diag_inputs()
    imp = orc.score(q, k, B)
    perm = orc.permute(imp, k, v, S)
    m0 = orc.block_mass(q, k, None, B)
    m1 = orc.block_mass(q, perm["k_perm"], perm["kpos"], B)
    spb = S // B
    seg = lambda m: m.reshape(*m.shape[:3], -1, spb).sum(-1)
    np.testing.assert_allclose(seg(m0), seg(m1), atol=1e-12)
    assert not np.allclose(m0, m1)


def test_coverage_of_all_blocks_is_one_and_of_own_block_is_its_mass():
    q, k, _, B, S = _diag_inputs()
    m = orc.block_mass(q, k, None, B)
    nb = m.shape[-1]
    idx = np.tile(np.arange(nb), (1, 2, nb, 1)).astype(np.int32)
    cnt = np.broadcast_to(np.arange(1, nb + 1), (1, 2, nb)).astype(np.int32)
    np.testing.assert_allclose(orc.coverage(m, idx, cnt), 1.0, atol=1e-12)
    own = np.broadcast_to(np.arange(nb)[:, None], (1, 2, nb, 1)).astype(np.int32)
    one = np.ones((1, 2, nb), dtype=np.int32)
    np.testing.assert_allclose(orc.coverage(m, own, one),
                               np.diagonal(m, axis1=2, axis2=3), atol=1e-15)


def test_blocks_for_coverage_brute_force():
    q, k, _, B, S = _diag_inputs(n=128, block=16)
    m = orc.block_mass(q, k, None, B)
    for target in (0.5, 0.9, 0.975, 1.0 - 1e-9):
        got = orc.blocks_for_coverage(m, target)
        for bi, g, i in np.ndindex(*got.shape):
            row = m[bi, g, i]
            # fewest blocks of any subset reaching the target, by enumeration
            nb = len(row)
            best = min(r for r in range(1, nb + 1)
                       for c in itertools.combinations(range(nb), r)
                       if row[list(c)].sum() >= target - 1e-15)
            assert got[bi, g, i] == best


def test_blocks_for_coverage_planted_key():
    # one key with an overwhelming logit for every query after it: its block
    # alone holds almost all the mass of every later query block
    q, k, _, B, S = _diag_inputs(n=128, block=16, hq=1)
    k[0, 0, 40] = 50.0 * q[0, 0].mean(axis=0) / np.linalg.norm(q[0, 0].mean(axis=0))
    q[0, 0] += q[0, 0].mean(axis=0)
    m = orc.block_mass(q, k, None, B)
    got = orc.blocks_for_coverage(m, 0.5)
    assert np.all(got[0, 0, 3:] == 1)
    assert np.all(m[0, 0, 3:, 2] > 0.5)
