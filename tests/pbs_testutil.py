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


def compare_lists(idx, cnt, ref_idx, ref_cnt, margin, rows=None):
    """Bit-exact comparison of block lists on every decided row; returns the
    number of rows whose decision margin was too small to compare."""
    idx, cnt = i64(idx), i64(cnt)
    amb = margin < AMBIGUOUS * np.maximum(1.0, 1.0)
    it = np.ndindex(*ref_cnt.shape) if rows is None else rows
    n_amb = 0
    for r in it:
        if amb[r]:
            n_amb += 1
            continue
        c = int(ref_cnt[r])
        assert int(cnt[r]) == c, f"row {r}: count {int(cnt[r])} != {c}"
        np.testing.assert_array_equal(idx[r][:c], ref_idx[r][:c], err_msg=f"row {r}")
    return n_amb
