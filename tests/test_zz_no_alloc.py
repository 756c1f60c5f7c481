"""pbs_score_static: importance scoring with no workspace from the caller.

Some callers cannot allocate device memory when they call the library (for
example a plugin of an inference engine that owns every device allocation
and forbids cudaMalloc). pbs_score_static serves them from a fixed scratch
array inside libpbs. These tests call it through the C ABI and check it
against pbs_score on two calls in a row, with different shapes, so that the
second call runs on the scratch contents the first one left behind: bit for
bit, since both run the same deterministic kernels.

This file is named to be collected last: a run that stops at its first
failure has run every other test before reaching it.
"""
import ctypes

import pytest
import torch

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200.workloads import Workload, make_inputs

SCRATCH_BYTES = 4 << 20   # PBS_SCORE_STATIC_SCRATCH_BYTES in include/pbs.h


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def test_oversized_shape_is_rejected_without_a_gpu():
    s = pbs.Shape(64, 256, 64, 1 << 20, 128, 128, 4096)
    assert pbs.workspace_bytes(s, 0) > SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    assert pbs.lib().pbs_score_static(fake, fake, fake, s, 0.0, None) == 6  # PBS_ERR_WORKSPACE


def test_arguments_are_checked_before_any_cuda_call():
    """Like pbs_score: an empty shape is a no-op and a bad shape or pointer
    returns its error, with no device lookup (this runs without a GPU)."""
    fake = ctypes.c_void_p(1 << 20)
    lib = pbs.lib()
    assert lib.pbs_score_static(fake, fake, fake, pbs.Shape(1, 4, 2, 0, 128, 128, 512), 0.0,
                                None) == 0                          # PBS_OK: empty
    assert lib.pbs_score_static(fake, fake, fake, pbs.Shape(1, 3, 2, 1024, 128, 128, 512), 0.0,
                                None) == 1                          # hq % hkv != 0
    assert lib.pbs_score_static(None, fake, fake, pbs.Shape(1, 4, 2, 1024, 128, 128, 512), 0.0,
                                None) == 1                          # no q
    assert lib.pbs_score_static(ctypes.c_void_p((1 << 20) + 8), fake, fake,
                                pbs.Shape(1, 4, 2, 1024, 128, 128, 512), 0.0, None) == 1


@pytest.mark.gpu
def test_static_scratch_matches_workspace_path():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dev = torch.device("cuda", 0)
    lib = pbs.lib()
    cases = [Workload("a", 1, 32, 8, 8192, 128, 128, 1024, "threshold", 0.9, "per_segment", 0.02),
             Workload("b", 2, 4, 2, 2048, 64, 64, 256, "threshold", 0.9, "uniform", 0.05)]
    for w in cases:
        q, k, _, _ = make_inputs(w, dev)
        s = pbs.Shape(w.batch, w.hq, w.hkv, w.n, w.d, w.block, w.segment)
        assert pbs.workspace_bytes(s, 0) <= SCRATCH_BYTES
        want = pbs.score(q, k, w.block, w.segment)
        got = torch.full_like(want, float("nan"))
        stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        assert lib.pbs_score_static(_ptr(q), _ptr(k), _ptr(got), s, 0.0, stream) == 0
        torch.cuda.synchronize()
        assert pbs.device_status() == 0
        # the same kernels with the same split of the keys over the CTAs and
        # fixed summation orders: bit for bit, so that a read of scratch left
        # by the previous (larger) call would show
        assert torch.equal(got, want)
