"""GPU parity of the attention-coverage and block-density diagnostics
(pbs_block_mass, pbs_coverage) against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200 import diagnostics as diag
from oracle import pbs_oracle as orc
from pbs_testutil import f64, i64
from test_gpu_parity import CASES, inputs

pytestmark = pytest.mark.gpu

MASS_RTOL, MASS_ATOL = 1e-4, 1e-6


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda", 0)


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "d64_b128", "odd_items", "s_eq_b"])
@pytest.mark.parametrize("permuted", [False, True])
def test_block_mass_against_oracle(name, permuted, dev):
    w = CASES[name]
    (q, k, v), (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    if permuted:
        imp = pbs.score(qd, kd, B)
        perm = pbs.permute(imp, kd, vd, B, S, hq=w.hq)
        kp, kpos = perm["k_perm"], perm["kpos"]
    else:
        kp, kpos = kd, None
    mass = diag.block_mass(qd, kp, kpos, B, S)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    want = orc.block_mass(f64(q), f64(kp), None if kpos is None else i64(kpos), B)
    np.testing.assert_allclose(f64(mass), want, rtol=MASS_RTOL, atol=MASS_ATOL)
    np.testing.assert_allclose(f64(mass).sum(-1), 1.0, atol=1e-4)


@pytest.mark.parametrize("name", ["gqa2k", "ragged", "odd_items"])
@pytest.mark.parametrize("target", [0.5, 0.9, 0.975])
def test_coverage_and_blocks_needed_against_oracle(name, target, dev):
    w = CASES[name]
    _, (qd, kd, vd) = inputs(w, dev)
    B, S = w.block, w.segment
    res = pbs.pbs_attention(qd, kd, vd, B, S, w.mode, w.param, keep=True)
    mass = diag.block_mass(qd, res["k_perm"], res["kpos"], B, S)
    shp = pbs.shape_of(qd, kd, B, S)
    cov, need = diag.coverage(mass, shp, res["idx"], res["cnt"], target)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    m = f64(mass)  # the oracle applied to the GPU's own masses
    np.testing.assert_allclose(f64(cov), orc.coverage(m, i64(res["idx"]), i64(res["cnt"])),
                               rtol=1e-6, atol=1e-7)
    want = orc.blocks_for_coverage(m, target)
    got = i64(need)
    # a row whose running sum meets the target within rounding is not compared
    run = np.cumsum(-np.sort(-m, axis=-1), axis=-1)
    near = np.abs(run - target).min(axis=-1) < 1e-9
    assert np.array_equal(got[~near], want[~near])
    assert near.mean() < 0.01


def test_report_runs_and_is_consistent(dev):
    w = CASES["gqa2k"]
    _, (qd, kd, vd) = inputs(w, dev)
    r = diag.report(qd, kd, vd, w.block, w.segment, w.mode, w.param, target=0.9)
    torch.cuda.synchronize()
    assert pbs.device_status() == 0
    assert 0.0 < r["coverage_perm"] <= 1.0 + 1e-6 and 0.0 < r["coverage_noperm"] <= 1.0 + 1e-6
    assert 0.0 < r["ideal_density_perm"] <= 1.0 and 0.0 < r["ideal_density_noperm"] <= 1.0
    # kept blocks over dense-causal blocks: the forced own segment includes
    # blocks J > I, so the bound is the admissible-block count
    nb, spb = w.n // w.block, w.segment // w.block
    adm = sum(min(nb, (i // spb + 1) * spb) for i in range(nb)) / (nb * (nb + 1) / 2)
    assert 0.0 < r["density_perm"] <= adm + 1e-9
    assert 0.0 < r["density_noperm"] <= adm + 1e-9
