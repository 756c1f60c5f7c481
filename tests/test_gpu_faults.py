"""Failure detection without a GPU fault.

The tcgen05 kernels bound every wait. PBS_FAULT_INJECT=timeout makes the
forward's K' loader skip the first tile load (a wait that nothing will
satisfy), and PBS_FAULT_INJECT=score_pass1 / score_pass2 do the same to the
first K tile of a scoring pass: the kernel must give up after its limit
(about a second), record PBS_ERR_TIMEOUT in the device error word, free its
tensor memory and return, leaving the context usable. The problems are
small, so each test takes about a second.
"""
import pytest
import torch

import long_context_sparse_segment_b200 as pbs

pytestmark = pytest.mark.gpu
TIMEOUT = 4


@pytest.mark.parametrize("block", [128, 64])
def test_bounded_wait_reports_timeout_and_context_survives(block, monkeypatch):
    """The forward for B = 128 and the one for B = 64 (query tiles of two
    64-row blocks)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    q, k, v = (torch.randn(1, 1, 128, 128, generator=g, device=dev).bfloat16() for _ in range(3))
    idx, cnt, _ = pbs.select_blocks(q, k, None, block, 128, "all")
    good = pbs.attn_fwd(q, k, v, None, None, idx, cnt, block, 128)
    assert pbs.device_status() == 0
    monkeypatch.setenv("PBS_FAULT_INJECT", "timeout")
    pbs.attn_fwd(q, k, v, None, None, idx, cnt, block, 128)
    code, where = pbs.device_status(detail=True)
    monkeypatch.delenv("PBS_FAULT_INJECT")
    assert code == TIMEOUT
    assert where in (32, 41), where      # MMA issuer on K', or softmax on S
    again = pbs.attn_fwd(q, k, v, None, None, idx, cnt, block, 128)
    assert pbs.device_status() == 0
    assert torch.equal(again, good)


@pytest.mark.parametrize("which,sites", [("score_pass1", (51, 53, 55)),
                                         ("score_pass2", (51, 53, 55))])
def test_scoring_wait_reports_timeout_and_context_survives(which, sites, monkeypatch):
    """The same for each pass of the tcgen05 scoring: PBS_FAULT_INJECT skips
    the pass's first K tile in every CTA; the pass gives up after its limit,
    reports PBS_ERR_TIMEOUT and the wait that ran out, and the next call
    gives the importance of a clean run bit for bit."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(1)
    q = torch.randn(1, 4, 1024, 128, generator=g, device=dev).bfloat16()
    k = torch.randn(1, 1, 1024, 128, generator=g, device=dev).bfloat16()
    good = pbs.score(q, k, 128, 512)
    assert pbs.device_status() == 0
    monkeypatch.setenv("PBS_FAULT_INJECT", which)
    pbs.score(q, k, 128, 512)
    code, where = pbs.device_status(detail=True)
    monkeypatch.delenv("PBS_FAULT_INJECT")
    assert code == TIMEOUT
    assert where in sites, where   # K loader, MMA issuer on the K tile, or a row group
    again = pbs.score(q, k, 128, 512)
    assert pbs.device_status() == 0
    assert torch.equal(again, good)
