"""Host-side checks of the C ABI: the library loads, exports every entry
point of include/pbs.h, and rejects bad arguments before launching anything
(none of these calls reaches a kernel, so no GPU is needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import long_context_sparse_segment_b200 as pbs
from long_context_sparse_segment_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from long_context_sparse_segment_b200 import build
        build.build()
    return pbs.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "pbs.h")).read()
    return set(re.findall(r"^\S[^;(]*?\b(pbs_\w+)\s*\(", text, flags=re.M))


def test_every_declared_symbol_is_exported(lib):
    declared = header_functions()
    assert declared == set(_lib.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (pbs_\w+)", out))
    assert declared <= exported


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.pbs_version()
    assert pbs.status_string(0) == "PBS_OK"
    assert pbs.status_string(4) == "PBS_ERR_TIMEOUT"
    assert pbs.status_string(99) == "PBS_ERR_UNKNOWN"


GOOD = dict(batch=1, hq=8, hkv=2, n=1024, d=128, block=128, segment=256)


def shape(**kw):
    f = dict(GOOD, **kw)
    return pbs.Shape(*(f[k] for k in ("batch", "hq", "hkv", "n", "d", "block", "segment")))


@pytest.mark.parametrize("kw,code", [
    (dict(hq=6, hkv=4), _lib.ERR_INVALID_ARG),         # hq not a multiple of hkv
    (dict(d=96), _lib.ERR_UNSUPPORTED),
    (dict(block=32), _lib.ERR_UNSUPPORTED),
    (dict(segment=200), _lib.ERR_INVALID_ARG),         # S not a multiple of B
    (dict(n=1000), _lib.ERR_INVALID_ARG),              # N not a multiple of B
    (dict(n=-128), _lib.ERR_INVALID_ARG),
    (dict(segment=16384), _lib.ERR_UNSUPPORTED),
])
def test_bad_shapes_are_rejected(lib, kw, code):
    fake = ctypes.c_void_p(1 << 20)
    s = shape(**kw)
    assert lib.pbs_score(fake, fake, fake, s, 0.0, fake, 1 << 30, None) == code
    assert lib.pbs_attn_fwd(fake, fake, fake, None, None, fake, fake, fake, None, s, 0.0,
                            None) == code
    assert lib.pbs_workspace_bytes(s, 0) == 0


def test_null_and_misaligned_pointers(lib):
    s = shape()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    ws = pbs.workspace_bytes(s, _lib.OP_SCORE)
    assert lib.pbs_score(None, fake, fake, s, 0.0, fake, ws, None) == _lib.ERR_INVALID_ARG
    assert lib.pbs_score(odd, fake, fake, s, 0.0, fake, ws, None) == _lib.ERR_INVALID_ARG
    assert lib.pbs_score(fake, fake, fake, s, 0.0, fake, ws - 1, None) == _lib.ERR_WORKSPACE
    # q without q_perm, and in-place gathers
    assert lib.pbs_permute(fake, fake, fake, fake, odd, odd, None, fake, None, s,
                           None) == _lib.ERR_INVALID_ARG
    assert lib.pbs_permute(fake, fake, fake, None, fake, fake, None, fake, None, s,
                           None) == _lib.ERR_INVALID_ARG
    assert lib.pbs_unpermute(fake, fake, fake, s, None) == _lib.ERR_INVALID_ARG


def test_selection_arguments(lib):
    s = shape()
    fake = ctypes.c_void_p(1 << 20)
    ws = pbs.workspace_bytes(s, _lib.OP_SELECT)
    for mode, param in ((0, 0.0), (0, 1.5), (1, -0.1), (7, 0.5)):
        assert lib.pbs_select_blocks(fake, fake, fake, s, mode, param, 0.0, fake, fake, None,
                                     fake, ws, None) == _lib.ERR_INVALID_ARG
    assert lib.pbs_select_blocks(fake, fake, None, s, 0, 0.9, 0.0, fake, fake, None, fake,
                                 ws // 2, None) == _lib.ERR_WORKSPACE


def test_empty_calls_launch_nothing(lib):
    s = shape(n=0)
    assert lib.pbs_score(None, None, None, s, 0.0, None, 0, None) == 0
    assert lib.pbs_attn_fwd(None, None, None, None, None, None, None, None, None, s, 0.0,
                            None) == 0
    s = shape(batch=0)
    assert lib.pbs_permute(None, None, None, None, None, None, None, None, None, s, None) == 0


def test_workspace_sizes_grow_with_the_problem(lib):
    # selection: pooled query and key sums (fp64, per block), then the score
    # keys and softmax weights of every (query head, query block, key block)
    for n in (1024, 2048):
        nb = n // GOOD["block"]
        want = 8 * nb * GOOD["d"] * (GOOD["hq"] + GOOD["hkv"]) + 2 * 8 * GOOD["hq"] * nb * nb
        assert pbs.workspace_bytes(shape(n=n), _lib.OP_SELECT) == want
    assert pbs.workspace_bytes(shape(), _lib.OP_ATTN) == 0


def test_host_path_workspace_follows_the_step_size(lib, monkeypatch):
    """The host path keeps three slots of one KV group's buffers; only the
    selection scratch depends on how many query heads a step covers (one
    step's worth is reused by the group's steps)."""
    s = shape(hq=8, hkv=2, n=2048)  # G = 4
    sizes = {}
    for step in (1, 2, 4):
        monkeypatch.setenv("PBS_HOST_STEP_HEADS", str(step))
        sizes[step] = pbs.workspace_bytes(s, _lib.OP_HOST_PATH)
    assert sizes[1] < sizes[2] < sizes[4]
    nb = 2048 // GOOD["block"]
    per_head = 8 * nb * GOOD["d"] + 2 * 8 * nb * nb  # pooled sums + scores and weights
    assert sizes[2] - sizes[1] == 3 * per_head
    assert sizes[4] - sizes[2] == 3 * 2 * per_head
    monkeypatch.setenv("PBS_HOST_STEP_HEADS", "3")  # not a divisor of G: ignored
    assert pbs.workspace_bytes(s, _lib.OP_HOST_PATH) in sizes.values()


def test_gathering_forward_and_order_only_permute_arguments(lib):
    s = shape()
    fake = ctypes.c_void_p(1 << 20)
    other = ctypes.c_void_p(1 << 24)
    odd = ctypes.c_void_p((1 << 20) + 8)
    # the carried key positions are required
    assert lib.pbs_attn_fwd_gather(fake, fake, fake, None, None, fake, fake, other, None, s,
                                   0.0, 0, None) == _lib.ERR_INVALID_ARG
    assert lib.pbs_attn_fwd_gather(fake, odd, fake, fake, None, fake, fake, other, None, s,
                                   0.0, 0, None) == _lib.ERR_INVALID_ARG
    # rows written at qpos must not land on an input still being read
    assert lib.pbs_attn_fwd_gather(fake, other, other, other, other, other, other, fake, None, s,
                                   0.0, 1, None) == _lib.ERR_INVALID_ARG
    # K' and V' are written together or not at all
    assert lib.pbs_permute(fake, fake, fake, None, other, None, None, fake, None, s,
                           None) == _lib.ERR_INVALID_ARG
    assert lib.pbs_permute(fake, fake, fake, None, None, other, None, fake, None, s,
                           None) == _lib.ERR_INVALID_ARG


def test_broadcast_forward_arguments(lib):
    s = shape()
    fake = ctypes.c_void_p(1 << 20)
    other = ctypes.c_void_p(1 << 24)
    outs = (ctypes.c_void_p * 9)(*([1 << 26] * 9))
    hq = s.hq
    call = lib.pbs_attn_fwd_bcast
    # 1..8 outputs
    assert call(fake, fake, fake, None, fake, fake, outs, 0, hq, 0, s, 0.0, None) == \
        _lib.ERR_INVALID_ARG
    assert call(fake, fake, fake, None, fake, fake, outs, 9, hq, 0, s, 0.0, None) == \
        _lib.ERR_INVALID_ARG
    # the call's heads must fit inside the buffers' heads
    assert call(fake, fake, fake, None, fake, fake, outs, 2, hq, 1, s, 0.0, None) == \
        _lib.ERR_INVALID_ARG
    assert call(fake, fake, fake, None, fake, fake, outs, 2, 2 * hq, -1, s, 0.0, None) == \
        _lib.ERR_INVALID_ARG
    # an output that is an input, a misaligned output
    alias = (ctypes.c_void_p * 2)(1 << 26, 1 << 20)
    assert call(fake, other, other, None, other, other, alias, 2, hq, 0, s, 0.0, None) == \
        _lib.ERR_INVALID_ARG
    odd = (ctypes.c_void_p * 1)((1 << 26) + 8)
    assert call(fake, fake, fake, None, fake, fake, odd, 1, hq, 0, s, 0.0, None) == \
        _lib.ERR_INVALID_ARG


def test_fused_forward_rejects_output_aliasing_an_input(lib):
    s = shape()
    fake = ctypes.c_void_p(1 << 20)
    other = ctypes.c_void_p(1 << 24)
    for out in (fake,):
        assert lib.pbs_attn_fwd_unpermute(fake, other, other, None, other, other, other, out,
                                          None, s, 0.0, None) == _lib.ERR_INVALID_ARG


def test_host_path_arguments(lib):
    s = shape()
    fake = ctypes.c_void_p(1 << 20)
    ws = pbs.workspace_bytes(s, _lib.OP_HOST_PATH)
    assert ws > 0
    call = lambda *a: lib.pbs_attention_host(*a)
    for mode, param in ((0, 0.0), (1, 1.5), (9, 0.5)):
        assert call(fake, fake, fake, fake, s, mode, param, 0.0, fake, ws, None, None,
                    None) == _lib.ERR_INVALID_ARG
    assert call(None, fake, fake, fake, s, 0, 0.9, 0.0, fake, ws, None, None,
                None) == _lib.ERR_INVALID_ARG
    assert call(fake, fake, fake, fake, s, 0, 0.9, 0.0, fake, ws - 1, None, None,
                None) == _lib.ERR_WORKSPACE
    # a KV group of 16 query heads x B = 128 probe rows exceeds the scoring kernels
    big = shape(hq=16, hkv=1)
    assert call(fake, fake, fake, fake, big, 0, 0.9, 0.0, fake, 1 << 40, None, None,
                None) == _lib.ERR_UNSUPPORTED
    assert call(None, None, None, None, shape(n=0), 0, 0.9, 0.0, None, 0, None, None, None) == 0
    # two slots of one KV group's buffers: the size grows with n, not with the group count
    assert pbs.workspace_bytes(shape(n=2048), _lib.OP_HOST_PATH) > ws
    assert pbs.workspace_bytes(shape(batch=4), _lib.OP_HOST_PATH) == ws


def test_diagnostics_arguments(lib):
    s = shape()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert lib.pbs_block_mass(fake, fake, None, fake, shape(block=64), 0.0,
                              None) == _lib.ERR_UNSUPPORTED
    assert lib.pbs_block_mass(fake, fake, None, fake, shape(hq=16, hkv=2), 0.0,
                              None) == _lib.ERR_UNSUPPORTED
    assert lib.pbs_block_mass(None, fake, None, fake, s, 0.0, None) == _lib.ERR_INVALID_ARG
    assert lib.pbs_block_mass(fake, fake, None, odd, s, 0.0, None) == _lib.ERR_INVALID_ARG
    # coverage needs the lists; the target must lie in (0, 1]
    assert lib.pbs_coverage(fake, None, None, ctypes.c_double(0.9), fake, None, s,
                            None) == _lib.ERR_INVALID_ARG
    for t in (0.0, 1.5):
        assert lib.pbs_coverage(fake, None, None, ctypes.c_double(t), None, fake, s,
                                None) == _lib.ERR_INVALID_ARG
