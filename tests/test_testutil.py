"""The parity helpers themselves, on the CPU: the validity check of a
near-tie selection accepts what the oracle's rule gives and rejects a list
with a block too many, too few or swapped; the key-order check accepts swaps
of near-equal importances only."""
import numpy as np
import pytest

from oracle import pbs_oracle as orc
from pbs_testutil import order_differences, valid_selection


@pytest.mark.parametrize("mode,param", [("threshold", 0.5), ("threshold", 0.9),
                                        ("threshold", 1.0), ("topk_frac", 0.3),
                                        ("topk_frac", 0.6)])
def test_valid_selection_accepts_the_rule_and_rejects_its_neighbours(mode, param):
    rng = np.random.default_rng(7)
    spb, nb = 2, 16
    rejected = 0
    for _ in range(10):
        a_all = rng.standard_normal(nb) * 2.0
        for i in range(nb):
            a = a_all[:(i // spb + 1) * spb]
            kept, margin = orc.select_row(a, i, spb, mode, param)
            assert valid_selection(kept, a, i, spb, mode, param)
            if margin < 1e-6:
                continue
            seg0 = (i // spb) * spb
            others = [j for j in range(seg0) if j not in kept]
            earlier = [j for j in kept if j < seg0]
            wrong = []
            if others:
                wrong.append(np.sort(np.append(kept, others[0])))
            if earlier:
                wrong.append(np.array([j for j in kept if j != earlier[0]]))
            if earlier and others:     # the worst block kept instead of the best
                worst = min(others, key=lambda j: a[j])
                best = max(earlier, key=lambda j: a[j])
                wrong.append(np.sort(np.append([j for j in kept if j != best], worst)))
            wrong.append(np.array([j for j in kept if j != kept[-1]]))    # own block dropped
            for w in wrong:
                assert not valid_selection(w, a, i, spb, mode, param), (i, w)
                rejected += 1
    assert rejected > 50


def test_order_differences_accepts_near_ties_only():
    imp = np.array([[[0.5, 0.3, 0.3 * (1 + 1e-5), 0.1]]])
    ref = np.array([[[0, 2, 1, 3]]])
    assert order_differences(np.array([[[0, 1, 2, 3]]]), ref, imp) == 2
    assert order_differences(ref, ref, imp) == 0
    with pytest.raises(AssertionError):
        order_differences(np.array([[[1, 2, 0, 3]]]), ref, imp)
