"""CPU oracle for the permuted block-sparse attention (PBS-Attn) prefill path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The CUDA library
never calls it, and it shares no code with the CUDA library.

Everything here is plain numpy in fp64: bf16 inputs are converted exactly
to fp64 and every step is evaluated in fp64. A matrix product, a sort, an
exponential and a sum are the only library primitives used. There is no
blocking, fusion or reordering beyond what each step's definition states.
Query rows are independent under the definition, so ``attend`` may be asked
for a subset of rows.

Sources (page title, then section):

* "Sparser Block-Sparse Attention via Token Permutation", gist.science
  technical summary, "Methodik", subsections 2 (segmented permutation),
  3 (global-importance key permutation) and 4 (implementation: block
  selection by mean pooling).
* "Sparser Block-Sparse Attention via Token Permutation", sciencestack.ai,
  Figure 1 caption (on-diagonal segments always computed) and Lemma 3.1,
  Lemma 3.2, Theorem 3.3 (permutation invariance / equivariance).
* "Sparser Block Attention", skillmd.com, "Implementation Steps"
  (inverse permutation by argsort; number of active blocks as a fraction of
  the block count, at least one).

Readings where the pages are silent (each also listed in the design notes):

* Importance: softmax probabilities of the last B query rows of every query
  head in the KV head's group, over all N keys with the causal mask, averaged
  over those G*B rows.
* Block score: a_IJ = sigma * mean(Q block I) . mean(K' block J), softmax over
  the admissible blocks J (segment of J <= segment of I).
* THRESHOLD(tau): keep the blocks of the query's own segment, then add the
  earlier-segment blocks in descending score (ties: lower J) until the kept
  softmax mass reaches tau (stop at mass >= tau).
* TOPK_FRAC(f): k = max(1, floor(f * (I + 1))); keep the own-segment blocks
  plus the best max(0, k - |own|) earlier-segment blocks (ties: lower J).
* Softmax scale sigma = 1/sqrt(d) unless a positive scale is given.
"""
from __future__ import annotations

import math

import numpy as np

MODES = {"threshold": 0, "topk_frac": 1, "all": 2, "dense_causal": 3}


def resolve_scale(scale, d):
    """sigma = scale if scale > 0 else 1/sqrt(d), as a float64."""
    if scale is not None and scale > 0:
        return float(np.float64(scale))
    return 1.0 / math.sqrt(d)


def _softmax_rows(x):
    m = np.max(x, axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# Step 1: key importance from the last query block
# (gist.science summary, "Methodik" 3, "Proxy-Bewertung")
# --------------------------------------------------------------------------
def score(q, k, block, scale=None):
    """Global key importance per (batch, KV head).

    q: [b, hq, n, d], k: [b, hkv, n, d] (fp64). The probe queries are the
    last ``block`` rows of each of the G = hq/hkv query heads that share KV
    head h. Each probe row attends causally over all n keys; the importance
    of key j is the mean of its softmax probability over the G*block rows.
    Returns imp [b, hkv, n] (fp64); each row of imp sums to 1.
    """
    b, hq, n, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    sigma = resolve_scale(scale, d)
    pos = np.arange(n - block, n)
    visible = np.arange(n)[None, :] <= pos[:, None]          # [block, n]
    visible = np.tile(visible, (g, 1))                         # [g*block, n]
    imp = np.zeros((b, hkv, n))
    for bi in range(b):
        for h in range(hkv):
            rows = q[bi, h * g:(h + 1) * g, n - block:, :].reshape(g * block, d)
            logits = sigma * (rows @ k[bi, h].T)
            logits = np.where(visible, logits, -np.inf)
            p = _softmax_rows(logits)
            imp[bi, h] = p.mean(axis=0)
    return imp


# --------------------------------------------------------------------------
# Step 2: segment-local key permutation
# (gist.science summary, "Methodik" 2 and 3, "Sortierung")
# --------------------------------------------------------------------------
def segment_order(imp, segment):
    """kpos [b, hkv, n] (int64): original key index at each permuted slot.

    Inside each contiguous segment of ``segment`` keys the keys are sorted by
    importance, largest first; equal importances keep the lower index first.
    Segments keep their place, so inter-segment causality is unchanged.
    """
    b, h, n = imp.shape
    kpos = np.empty((b, h, n), dtype=np.int64)
    for bi in range(b):
        for hi in range(h):
            for s0 in range(0, n, segment):
                seg = imp[bi, hi, s0:s0 + segment]
                kpos[bi, hi, s0:s0 + segment] = s0 + np.argsort(-seg, kind="stable")
    return kpos


def gather_rows(x, pos):
    """x[b, h, pos[b, h, p], :] for every permuted slot p."""
    return np.take_along_axis(x, pos[..., None], axis=2)


def permute(imp, k, v, segment, q=None):
    """Apply the segment-local order to K and V (and optionally Q).

    Returns dict with kpos, k_perm, v_perm and, when q is given (permuted-
    query mode), q_perm and qpos [b, hq, n] where query head g uses the
    order of its KV head g // G.
    """
    kpos = segment_order(imp, segment)
    out = {"kpos": kpos, "k_perm": gather_rows(k, kpos), "v_perm": gather_rows(v, kpos)}
    if q is not None:
        g = q.shape[1] // k.shape[1]
        qpos = np.repeat(kpos, g, axis=1)
        out["qpos"] = qpos
        out["q_perm"] = gather_rows(q, qpos)
    return out


# --------------------------------------------------------------------------
# Step 3: block selection from mean-pooled scores
# (gist.science summary, "Methodik" 4 "Block-Auswahl"; sciencestack.ai
#  Figure 1 caption; skillmd.com "Implementation Steps")
# --------------------------------------------------------------------------
def block_means(x, block):
    """Mean of each run of ``block`` consecutive rows: [b, h, n/block, d]."""
    b, h, n, d = x.shape
    return x.reshape(b, h, n // block, block, d).sum(axis=3) / block


def select_row(a, i_blk, spb, mode, param):
    """Kept key blocks of query block ``i_blk`` (ascending) and a margin.

    a: block scores of the admissible key blocks 0 .. (seg(I)+1)*spb - 1,
    cut at the last block (a shorter last segment has fewer blocks).
    The margin is the smallest gap that decides the result: for THRESHOLD
    the distance of the kept mass to tau on either side of the cut (the mass
    before the last block taken, also when the walk ran out of blocks before
    reaching tau, and the mass after it) and the score gap at the cut; for
    TOPK_FRAC the score gap at the cut. Moving tau, or any one block score,
    by less than the margin leaves the kept set as it is. It is +inf where
    nothing is decided.
    """
    seg = i_blk // spb
    forced = np.arange(seg * spb, len(a))
    if mode == "all":
        return np.arange(len(a)), math.inf
    if mode == "dense_causal":
        return np.arange(i_blk + 1), math.inf
    n_earlier = seg * spb
    # earlier-segment blocks by descending score, ties to the lower index
    order = np.argsort(-a[:n_earlier], kind="stable")
    margin = math.inf
    if mode == "threshold":
        tau = float(np.float64(np.float32(param)))
        pi = np.exp(a - a.max())
        pi = pi / pi.sum()
        mass = pi[forced].sum()
        taken = 0
        if mass < tau:
            while taken < n_earlier and mass < tau:
                before = mass
                mass = mass + pi[order[taken]]
                taken += 1
            if taken > 0:
                # tau at or below the mass before the last block ends the
                # walk one block earlier, whether or not tau was reached
                margin = min(margin, tau - before)
        if taken < n_earlier:
            margin = min(margin, mass - tau)
        if 0 < taken < n_earlier:
            margin = min(margin, a[order[taken - 1]] - a[order[taken]])
    elif mode == "topk_frac":
        frac = float(np.float64(np.float32(param)))
        k_i = max(1, math.floor(frac * (i_blk + 1)))
        taken = min(n_earlier, max(0, k_i - len(forced)))
        if 0 < taken < n_earlier:
            margin = a[order[taken - 1]] - a[order[taken]]
    else:
        raise ValueError(mode)
    kept = np.sort(np.concatenate([order[:taken], forced]))
    return kept, margin


def block_scores(q_pooled, k_pooled, scale, group):
    """a[b, g, I, J] = sigma * qbar_{g,I} . kbar_{h,J} with h = g // group,
    for every pair (admissibility is applied by the caller): [b, hq, nb, nb]."""
    b, hq, nb, d = q_pooled.shape
    sigma = resolve_scale(scale, d)
    a = np.empty((b, hq, nb, nb))
    for bi in range(b):
        for g in range(hq):
            a[bi, g] = sigma * (q_pooled[bi, g] @ k_pooled[bi, g // group].T)
    return a


def select_blocks(q_pooled, k_pooled, spb, mode, param, scale, group):
    """Block lists for every (batch, query head, query block).

    q_pooled: [b, hq, nb, d] block means of Q (or of the permuted Q);
    k_pooled: [b, hkv, nb, d] block means of the permuted K.
    Returns (idx [b, hq, nb, nb] int32 padded with -1, cnt [b, hq, nb] int32,
    margin [b, hq, nb] float64).
    """
    b, hq, nb, d = q_pooled.shape
    idx = np.full((b, hq, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((b, hq, nb), dtype=np.int32)
    margin = np.full((b, hq, nb), math.inf)
    a = block_scores(q_pooled, k_pooled, scale, group)
    for bi in range(b):
        for g in range(hq):
            scores = a[bi, g]                                   # [nb, nb]
            for i in range(nb):
                adm = min(nb, ((i // spb) + 1) * spb)
                kept, mg = select_row(scores[i, :adm], i, spb, mode, param)
                idx[bi, g, i, :len(kept)] = kept
                cnt[bi, g, i] = len(kept)
                margin[bi, g, i] = mg
    return idx, cnt, margin


# --------------------------------------------------------------------------
# Step 4: block-sparse causal attention on the permuted sequence
# (sciencestack.ai Figure 1 caption; gist.science "Methodik" 2 and 4)
# --------------------------------------------------------------------------
def attend_blocks(q, k_perm, v_perm, kpos, qpos, idx, cnt, block, blocks, scale=None):
    """``attend`` for whole query blocks only: blocks is an iterable of
    (batch, head, query block); returns [len(blocks), block, d]."""
    hkv = k_perm.shape[1]
    g_sz = q.shape[1] // hkv
    sigma = resolve_scale(scale, q.shape[3])
    blocks = list(blocks)
    out = np.zeros((len(blocks), block, q.shape[3]))
    for t, (bi, g, blk) in enumerate(blocks):
        r = np.arange(blk * block, (blk + 1) * block)
        out[t] = _attend_rows(q, k_perm, v_perm, kpos, qpos, idx, cnt, block, sigma, bi, g,
                              g // g_sz, blk, r)
    return out


def attend(q, k_perm, v_perm, kpos, qpos, idx, cnt, block, scale=None, rows=None):
    """Output rows of the permuted block-sparse attention.

    For query row i (in the order of q) of head g in query block I = i//B,
    the keys are the permuted slots p of the kept blocks of (g, I) whose
    original position kpos[p] is <= the query's original position qpos[i]
    (qpos None: the natural position i). Softmax over those keys of
    sigma * q_i . k'_p, output the probability-weighted sum of v'_p.

    q: [b, hq, n, d]; k_perm, v_perm: [b, hkv, n, d]; kpos: [b, hkv, n] or
    None (identity); qpos: [b, hq, n] or None; idx/cnt from select_blocks.
    rows: optional iterable of (batch, head, row) triples; returns then an
    array [len(rows), d]. Otherwise returns o [b, hq, n, d].
    """
    b, hq, n, d = q.shape
    hkv = k_perm.shape[1]
    g_sz = hq // hkv
    sigma = resolve_scale(scale, d)
    if rows is None:
        out = np.zeros((b, hq, n, d))
        todo = [(bi, g, blk) for bi in range(b) for g in range(hq)
                for blk in range(n // block)]
        for bi, g, blk in todo:
            r = np.arange(blk * block, (blk + 1) * block)
            out[bi, g, r] = _attend_rows(q, k_perm, v_perm, kpos, qpos, idx, cnt,
                                         block, sigma, bi, g, g // g_sz, blk, r)
        return out
    rows = list(rows)
    out = np.zeros((len(rows), d))
    for t, (bi, g, i) in enumerate(rows):
        out[t] = _attend_rows(q, k_perm, v_perm, kpos, qpos, idx, cnt, block, sigma,
                              bi, g, g // g_sz, i // block, np.array([i]))[0]
    return out


def _attend_rows(q, k_perm, v_perm, kpos, qpos, idx, cnt, block, sigma, bi, g, h,
                 blk, r):
    kept = idx[bi, g, blk, :cnt[bi, g, blk]]
    slots = (kept[:, None] * block + np.arange(block)[None, :]).reshape(-1)
    orig_k = slots if kpos is None else kpos[bi, h, slots]
    orig_q = r if qpos is None else qpos[bi, g, r]
    visible = orig_k[None, :] <= orig_q[:, None]
    logits = sigma * (q[bi, g, r] @ k_perm[bi, h, slots].T)
    logits = np.where(visible, logits, -np.inf)
    p = _softmax_rows(logits)
    return p @ v_perm[bi, h, slots]


# --------------------------------------------------------------------------
# Step 5: inverse permutation of the output rows
# (skillmd.com "Implementation Steps"; sciencestack.ai Theorem 3.3)
# --------------------------------------------------------------------------
def unpermute(o_perm, qpos):
    """o[b, g, qpos[b, g, p]] = o_perm[b, g, p]; qpos None returns o_perm."""
    if qpos is None:
        return o_perm.copy()
    out = np.empty_like(o_perm)
    np.put_along_axis(out, qpos[..., None], o_perm, axis=2)
    return out


# --------------------------------------------------------------------------
# The whole path, and the dense causal attention it approximates
# --------------------------------------------------------------------------
def pbs_attention(q, k, v, block, segment, mode, param, scale=None, permute_q=False):
    """All five steps; returns a dict with every intermediate and o."""
    group = q.shape[1] // k.shape[1]
    spb = segment // block
    imp = score(q, k, block, scale)
    perm = permute(imp, k, v, segment, q if permute_q else None)
    q_used = perm["q_perm"] if permute_q else q
    qpos = perm.get("qpos")
    idx, cnt, margin = select_blocks(block_means(q_used, block),
                                     block_means(perm["k_perm"], block),
                                     spb, mode, param, scale, group)
    o_perm = attend(q_used, perm["k_perm"], perm["v_perm"], perm["kpos"], qpos,
                    idx, cnt, block, scale)
    out = dict(perm, imp=imp, idx=idx, cnt=cnt, margin=margin, o_perm=o_perm)
    out["o"] = unpermute(o_perm, qpos)
    return out


def dense_causal(q, k, v, scale=None):
    """Plain causal softmax attention with GQA, fp64: [b, hq, n, d]."""
    b, hq, n, d = q.shape
    g = hq // k.shape[1]
    sigma = resolve_scale(scale, d)
    mask = np.tril(np.ones((n, n), dtype=bool))
    out = np.empty((b, hq, n, d))
    for bi in range(b):
        for h in range(hq):
            logits = sigma * (q[bi, h] @ k[bi, h // g].T)
            p = _softmax_rows(np.where(mask, logits, -np.inf))
            out[bi, h] = p @ v[bi, h // g]
    return out


def block_flops(cnt, block, d):
    """Tensor-core work of the forward: 4*B*B*d per kept (head, block) pair."""
    return 4.0 * block * block * d * float(np.asarray(cnt, dtype=np.int64).sum())


# --------------------------------------------------------------------------
# Diagnostics: attention coverage and block-level density
# (sciencestack.ai Figure 2 caption: the coverage of a selection is the total
#  attention score its blocks hold; Figure 4: block-level density with and
#  without permutation; gist.science "Experimentelle Ergebnisse", Sparsity)
# --------------------------------------------------------------------------
def block_mass(q, k_perm, kpos, block, scale=None):
    """Exact attention mass of every (query block, key block) pair.

    Query row i (natural order) attends causally over all n keys: the key in
    permuted slot p is visible when its original position kpos[p] <= i
    (kpos None: identity). With the dense softmax probabilities P_ip,
    mass[b, g, I, J] = (1/B) * sum over rows i of block I and slots p of
    block J of P_ip. Every (b, g, I) row of mass sums to 1.
    q: [b, hq, n, d]; k_perm: [b, hkv, n, d]; kpos: [b, hkv, n] or None.
    Returns [b, hq, nb, nb] fp64.
    """
    b, hq, n, d = q.shape
    hkv = k_perm.shape[1]
    g_sz = hq // hkv
    nb = n // block
    sigma = resolve_scale(scale, d)
    mass = np.zeros((b, hq, nb, nb))
    for bi in range(b):
        for g in range(hq):
            h = g // g_sz
            orig = np.arange(n) if kpos is None else kpos[bi, h]
            logits = sigma * (q[bi, g] @ k_perm[bi, h].T)              # [n, n]
            visible = orig[None, :] <= np.arange(n)[:, None]
            p = _softmax_rows(np.where(visible, logits, -np.inf))
            mass[bi, g] = p.reshape(nb, block, nb, block).sum(axis=(1, 3)) / block
    return mass


def coverage(mass, idx, cnt):
    """Mass held by each (b, g, I) selection: sum of mass[b, g, I, J] over the
    first cnt entries J of idx[b, g, I]. Returns [b, hq, nb] fp64."""
    b, hq, nb, _ = mass.shape
    out = np.zeros((b, hq, nb))
    for bi, g, i in np.ndindex(b, hq, nb):
        out[bi, g, i] = mass[bi, g, i, idx[bi, g, i, :cnt[bi, g, i]]].sum()
    return out


def blocks_for_coverage(mass, target):
    """Fewest key blocks that hold at least `target` of each row's mass:
    the blocks in descending mass, counted until their sum reaches target.
    Returns [b, hq, nb] int64."""
    b, hq, nb, _ = mass.shape
    out = np.zeros((b, hq, nb), dtype=np.int64)
    for bi, g, i in np.ndindex(b, hq, nb):
        run = np.cumsum(np.sort(mass[bi, g, i])[::-1])
        out[bi, g, i] = min(nb, int(np.searchsorted(run, target)) + 1)
    return out
