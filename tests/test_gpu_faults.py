"""Failure detection without a GPU fault.

The tcgen05 forward bounds every wait. PBS_FAULT_INJECT=timeout makes its K'
loader skip the first tile load (a wait that nothing will satisfy): the
kernel must give up after its limit (about a second), record
PBS_ERR_TIMEOUT in the device error word, free its tensor memory and return,
leaving the context usable. The problem is one CTA so the test takes ~1 s.
"""
import pytest
import torch

import long_context_sparse_segment_b200 as pbs

pytestmark = pytest.mark.gpu
TIMEOUT = 4


def test_bounded_wait_reports_timeout_and_context_survives(monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    q, k, v = (torch.randn(1, 1, 128, 128, generator=g, device=dev).bfloat16() for _ in range(3))
    idx, cnt, _ = pbs.select_blocks(q, k, None, 128, 128, "all")
    good = pbs.attn_fwd(q, k, v, None, None, idx, cnt, 128, 128)
    assert pbs.device_status() == 0
    monkeypatch.setenv("PBS_FAULT_INJECT", "timeout")
    pbs.attn_fwd(q, k, v, None, None, idx, cnt, 128, 128)
    code, where = pbs.device_status(detail=True)
    monkeypatch.delenv("PBS_FAULT_INJECT")
    assert code == TIMEOUT
    assert where in (32, 41), where      # MMA issuer on K', or softmax on S
    again = pbs.attn_fwd(q, k, v, None, None, idx, cnt, 128, 128)
    assert pbs.device_status() == 0
    assert torch.equal(again, good)
