"""Comparison helpers shared by the GPU parity tests."""
import numpy as np
import torch

# Output tolerance: bf16 inputs and output, fp32 accumulation.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# Relative tolerance of the fp32 importance against the fp64 oracle.
IMP_RTOL = 1e-4
# A selection decision whose deciding gap is below this is reported, not
# compared: both sides evaluate it in fp64 but in different summation orders.
AMBIGUOUS = 1e-12


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def i64(t):
    return t.detach().cpu().numpy().astype(np.int64)


def assert_outputs_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def assert_importance_close(got, want):
    got, want = np.asarray(got), np.asarray(want)
    rel = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
    assert rel.max() <= IMP_RTOL, f"importance rel err {rel.max():.3e}"
    return float(rel.max())


def valid_selection(kept, a, i_blk, spb, mode, param, eps=AMBIGUOUS):
    """Whether ``kept`` is a correct answer for a near-tie row: one that the
    selection rule gives once tau or the block scores move by at most eps.

    a: the fp64 block scores of the admissible blocks of query block i_blk.
    The own segment is kept; the earlier blocks kept are the best ones up to
    score ties within eps; THRESHOLD: the kept mass reaches tau - eps unless
    every earlier block is kept, and without its lowest-scoring earlier block
    the mass stays below tau + eps; TOP-K: their number is the rule's."""
    kept = np.asarray(kept, dtype=np.int64)
    adm = len(a)
    seg0 = (i_blk // spb) * spb
    if np.any(np.diff(kept) <= 0) or kept.min() < 0 or kept.max() >= adm:
        return False
    if not set(range(seg0, adm)) <= set(kept.tolist()):
        return False
    taken = kept[kept < seg0]
    rest = np.setdiff1d(np.arange(seg0), taken)
    if len(taken) and len(rest) and a[taken].min() < a[rest].max() - eps:
        return False
    if mode == "threshold":
        tau = float(np.float32(param))
        pi = np.exp(a - a.max())
        pi = pi / pi.sum()
        mass = pi[kept].sum()
        if len(rest) and mass < tau - eps:
            return False
        if len(taken) and mass - pi[taken[np.argmin(a[taken])]] >= tau + eps:
            return False
        return True
    if mode == "topk_frac":
        k_i = max(1, int(np.floor(float(np.float32(param)) * (i_blk + 1))))
        return len(taken) == min(seg0, max(0, k_i - (adm - seg0)))
    return False


def compare_lists(idx, cnt, ref_idx, ref_cnt, margin, rows=None, scores=None, spb=None,
                  mode=None, param=None):
    """Bit-exact comparison of block lists on every decided row. A row whose
    oracle margin is below AMBIGUOUS (a near-tie that both sides decide in
    fp64 but sum in different orders) is checked for validity instead: the
    GPU's list must be one the rule gives within that margin (needs the
    oracle's block scores, scores[b, g, I, :]). Returns the number of such
    rows."""
    idx, cnt = i64(idx), i64(cnt)
    amb = margin < AMBIGUOUS
    it = np.ndindex(*ref_cnt.shape) if rows is None else rows
    n_amb = 0
    for r in it:
        c = int(cnt[r])
        if amb[r]:
            n_amb += 1
            assert scores is not None, f"row {r}: near-tie without the scores to check it"
            i_blk = r[-1]
            adm = min(scores.shape[-1], (i_blk // spb + 1) * spb)
            assert valid_selection(idx[r][:c], scores[r][:adm], i_blk, spb, mode, param), \
                f"row {r}: near-tie answered with an invalid list {idx[r][:c].tolist()}"
            continue
        want = int(ref_cnt[r])
        assert c == want, f"row {r}: count {c} != {want}"
        np.testing.assert_array_equal(idx[r][:c], ref_idx[r][:c], err_msg=f"row {r}")
    return n_amb


def order_differences(kpos, ref_kpos, ref_imp, rtol=2 * IMP_RTOL):
    """Slots where the GPU's key order differs from the oracle's. Both orders
    sort importances that agree within IMP_RTOL, so at a differing slot the
    two keys' oracle importances must agree within twice that (a swap inside
    a run of near-equal importance); anything else fails. Returns the number
    of differing slots."""
    kpos, ref_kpos = np.asarray(kpos), np.asarray(ref_kpos)
    diff = np.nonzero(kpos != ref_kpos)
    a = np.take_along_axis(ref_imp, kpos, axis=-1)[diff]
    b = np.take_along_axis(ref_imp, ref_kpos, axis=-1)[diff]
    rel = np.abs(a - b) / np.maximum(np.maximum(np.abs(a), np.abs(b)), 1e-300)
    assert rel.size == 0 or rel.max() <= rtol, \
        f"{rel.size} slots differ, one by {rel.max():.2e} relative importance"
    return int(rel.size)
