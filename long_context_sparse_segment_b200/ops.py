"""PyTorch-facing calls of libpbs: argument marshalling only.

Every step runs in the library's CUDA kernels; these functions only check
tensor dtypes and devices, allocate outputs with torch, and pass raw device
pointers plus the current CUDA stream through the C ABI (include/pbs.h).
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import Shape, check, lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _call(name, *args):
    """One C-ABI call, inside an NVTX range of its name (seen by Nsight
    Systems beside the kernels it launches); raises on a non-OK status."""
    torch.cuda.nvtx.range_push(name)
    try:
        return check(getattr(lib(), name)(*args), name)
    finally:
        torch.cuda.nvtx.range_pop()


def _need(t, name, dtype, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def shape_of(q, k, block, segment) -> Shape:
    b, hq, n, d = q.shape
    return Shape(b, hq, k.shape[1], n, d, block, segment)


def workspace_bytes(shape: Shape, op: int) -> int:
    return int(lib().pbs_workspace_bytes(shape, op))


def _workspace(shape, op, device, ws=None):
    need = workspace_bytes(shape, op)
    if ws is not None and ws.numel() * ws.element_size() >= need:
        return ws, need
    return torch.empty(max(need, 16), dtype=torch.uint8, device=device), need


def score(q, k, block, segment=None, scale=0.0, ws=None, out=None):
    """Key importance imp [b, hkv, n] fp32 from the last query block."""
    _need(q, "q", torch.bfloat16)
    _need(k, "k", torch.bfloat16, q.device)
    shp = shape_of(q, k, block, segment or block)
    b, hkv, n, _ = k.shape
    imp = out if out is not None else torch.empty(b, hkv, n, dtype=torch.float32, device=q.device)
    ws, need = _workspace(shp, _lib.OP_SCORE, q.device, ws)
    _call("pbs_score", _ptr(q), _ptr(k), _ptr(imp), shp, scale, _ptr(ws), need,
          _stream(q.device))
    return imp


def permute(imp, k, v, block, segment, q=None, kbar=True, hq=None, materialize=True):
    """Segment-local order and gathers. Returns dict(kpos, k_perm, v_perm,
    kbar_sum[, q_perm]); without ``materialize`` only the order and the key
    block sums are produced (k_perm, v_perm None) for attn_fwd_gather."""
    _need(imp, "imp", torch.float32)
    _need(k, "k", torch.bfloat16, imp.device)
    _need(v, "v", torch.bfloat16, imp.device)
    b, hkv, n, d = k.shape
    if q is not None:
        _need(q, "q", torch.bfloat16, imp.device)
        hq = q.shape[1]
    shp = Shape(b, hq or hkv, hkv, n, d, block, segment)
    out = {
        "kpos": torch.empty(b, hkv, n, dtype=torch.int32, device=k.device),
        "k_perm": torch.empty_like(k) if materialize else None,
        "v_perm": torch.empty_like(v) if materialize else None,
        "kbar_sum": (torch.empty(b, hkv, n // block, d, dtype=torch.float64, device=k.device)
                     if kbar else None),
        "q_perm": torch.empty_like(q) if q is not None else None,
    }
    _call("pbs_permute", _ptr(imp), _ptr(k), _ptr(v), _ptr(q), _ptr(out["k_perm"]),
          _ptr(out["v_perm"]), _ptr(out["q_perm"]), _ptr(out["kpos"]),
          _ptr(out["kbar_sum"]), shp, _stream(k.device))
    return out


def select_blocks(q, k_perm, kbar_sum, block, segment, mode, param=0.0, scale=0.0, mask=False,
                  ws=None, idx=None, cnt=None):
    """Kept block lists: (blk_idx [b,hq,nb,nb] int32, blk_cnt [b,hq,nb] int32,
    blk_mask [b,hq,nb,nb] uint8 or None)."""
    _need(q, "q", torch.bfloat16)
    if kbar_sum is not None:
        _need(kbar_sum, "kbar_sum", torch.float64, q.device)
    if k_perm is not None:
        _need(k_perm, "k_perm", torch.bfloat16, q.device)
    hkv = (k_perm if k_perm is not None else kbar_sum).shape[1]
    b, hq, n, d = q.shape
    shp = Shape(b, hq, hkv, n, d, block, segment)
    nb = n // block
    mode_id = _lib.SEL[mode] if isinstance(mode, str) else int(mode)
    idx = idx if idx is not None else torch.empty(b, hq, nb, nb, dtype=torch.int32, device=q.device)
    cnt = cnt if cnt is not None else torch.empty(b, hq, nb, dtype=torch.int32, device=q.device)
    msk = torch.empty(b, hq, nb, nb, dtype=torch.uint8, device=q.device) if mask else None
    ws, need = _workspace(shp, _lib.OP_SELECT, q.device, ws)
    _call("pbs_select_blocks", _ptr(q), _ptr(k_perm), _ptr(kbar_sum), shp, mode_id, param,
          scale, _ptr(idx), _ptr(cnt), _ptr(msk), _ptr(ws), need,
          _stream(q.device))
    return idx, cnt, msk


def attn_fwd(q, k_perm, v_perm, kpos, qpos, blk_idx, blk_cnt, block, segment, scale=0.0,
             lse=False, out=None, unpermute=False):
    """Block-sparse causal attention over the permuted keys: o [b,hq,n,d] bf16
    (and lse [b,hq,n] fp32 when asked). With ``unpermute`` (permuted queries)
    each row is written at its query's original position in the same call
    (pbs_attn_fwd_unpermute) instead of in the order of ``q``."""
    _need(q, "q", torch.bfloat16)
    _need(k_perm, "k_perm", torch.bfloat16, q.device)
    _need(v_perm, "v_perm", torch.bfloat16, q.device)
    for t, nm in ((kpos, "kpos"), (qpos, "qpos")):
        if t is not None:
            _need(t, nm, torch.int32, q.device)
    _need(blk_idx, "blk_idx", torch.int32, q.device)
    _need(blk_cnt, "blk_cnt", torch.int32, q.device)
    shp = shape_of(q, k_perm, block, segment)
    o = out if out is not None else torch.empty_like(q)
    l = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if lse else None
    _call("pbs_attn_fwd_unpermute" if unpermute else "pbs_attn_fwd", _ptr(q), _ptr(k_perm),
          _ptr(v_perm), _ptr(kpos), _ptr(qpos), _ptr(blk_idx), _ptr(blk_cnt), _ptr(o), _ptr(l),
          shp, scale, _stream(q.device))
    return (o, l) if lse else o


def attn_fwd_gather(q, k, v, kpos, qpos, blk_idx, blk_cnt, block, segment, scale=0.0,
                    lse=False, out=None, unpermute=False):
    """attn_fwd on the natural k, v: key slot p is read from row kpos[p]
    (pbs_attn_fwd_gather), so no permuted copies are needed. Same result,
    bit for bit, as attn_fwd on k[kpos], v[kpos]."""
    _need(q, "q", torch.bfloat16)
    _need(k, "k", torch.bfloat16, q.device)
    _need(v, "v", torch.bfloat16, q.device)
    _need(kpos, "kpos", torch.int32, q.device)
    if qpos is not None:
        _need(qpos, "qpos", torch.int32, q.device)
    _need(blk_idx, "blk_idx", torch.int32, q.device)
    _need(blk_cnt, "blk_cnt", torch.int32, q.device)
    shp = shape_of(q, k, block, segment)
    o = out if out is not None else torch.empty_like(q)
    l = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if lse else None
    _call("pbs_attn_fwd_gather", _ptr(q), _ptr(k), _ptr(v), _ptr(kpos), _ptr(qpos),
          _ptr(blk_idx), _ptr(blk_cnt), _ptr(o), _ptr(l), shp, scale,
          1 if unpermute else 0, _stream(q.device))
    return (o, l) if lse else o


def attn_fwd_bcast(q, k_perm, v_perm, kpos, blk_idx, blk_cnt, block, segment, outs,
                   head_offset=0, scale=0.0):
    """attn_fwd writing every output row into each tensor of ``outs``
    ([b, hq_total, n, d] bf16, on this device or mapped into its address
    space), query head g at head ``head_offset + g`` (pbs_attn_fwd_bcast)."""
    _need(q, "q", torch.bfloat16)
    _need(k_perm, "k_perm", torch.bfloat16, q.device)
    _need(v_perm, "v_perm", torch.bfloat16, q.device)
    if kpos is not None:
        _need(kpos, "kpos", torch.int32, q.device)
    _need(blk_idx, "blk_idx", torch.int32, q.device)
    _need(blk_cnt, "blk_cnt", torch.int32, q.device)
    if not outs:
        raise ValueError("outs: at least one output tensor")
    b, _, n, d = q.shape
    hq_total = outs[0].shape[1]
    for i, o in enumerate(outs):
        if (o.dtype != torch.bfloat16 or not o.is_contiguous() or o.dim() != 4
                or (o.shape[0], o.shape[2], o.shape[3]) != (b, n, d) or o.shape[1] != hq_total):
            raise ValueError(f"outs[{i}]: contiguous bf16 [b, hq_total, n, d] expected")
    ptrs = (ctypes.c_void_p * len(outs))(*[o.data_ptr() for o in outs])
    shp = shape_of(q, k_perm, block, segment)
    _call("pbs_attn_fwd_bcast", _ptr(q), _ptr(k_perm), _ptr(v_perm), _ptr(kpos),
          _ptr(blk_idx), _ptr(blk_cnt), ptrs, len(outs), hq_total,
          head_offset, shp, scale, _stream(q.device))
    return outs


def unpermute(o_perm, qpos, hkv, block, segment, out=None):
    """o[b, g, qpos[b, g/G, p]] = o_perm[b, g, p]."""
    _need(o_perm, "o_perm", torch.bfloat16)
    if qpos is not None:
        _need(qpos, "qpos", torch.int32, o_perm.device)
    b, hq, n, d = o_perm.shape
    shp = Shape(b, hq, hkv, n, d, block, segment)
    o = out if out is not None else torch.empty_like(o_perm)
    _call("pbs_unpermute", _ptr(o_perm), _ptr(qpos), _ptr(o), shp, _stream(o_perm.device))
    return o


def device_status(device=None, detail=False):
    """Synchronise, read and clear the device error word: the pbs status code
    (0 = no kernel reported a problem), plus the diagnostic detail if asked."""
    code, where = ctypes.c_int(0), ctypes.c_int(0)
    _call("pbs_get_device_status", _stream(device), ctypes.byref(code), ctypes.byref(where))
    return (code.value, where.value) if detail else code.value


def pbs_attention(q, k, v, block, segment, mode="threshold", param=0.9, scale=0.0,
                  permute_q=False, keep=False, fused_unpermute=True, gather_kv=False):
    """The whole prefill path: score -> permute -> select -> attend ->
    unpermute. Returns o [b, hq, n, d] bf16 in the natural query order, or a
    dict with every intermediate when ``keep`` is true. In permuted-query
    mode the last two steps are one call unless ``fused_unpermute`` is
    false (then ``o_perm`` holds the rows in permuted order). With
    ``gather_kv`` the permutation writes only the key order and block sums
    and the forward reads K, V through it (no K', V' copies)."""
    imp = score(q, k, block, segment, scale)
    perm = permute(imp, k, v, block, segment, q=q if permute_q else None, hq=q.shape[1],
                   materialize=not gather_kv)
    q_used = perm["q_perm"] if permute_q else q
    qpos = perm["kpos"] if permute_q else None
    idx, cnt, _ = select_blocks(q_used, perm["k_perm"], perm["kbar_sum"], block, segment, mode,
                                param, scale)
    if gather_kv:
        o = attn_fwd_gather(q_used, k, v, perm["kpos"], qpos, idx, cnt, block, segment, scale,
                            unpermute=permute_q)
        o_perm = None
    elif permute_q and fused_unpermute:
        o = attn_fwd(q_used, perm["k_perm"], perm["v_perm"], perm["kpos"], qpos, idx, cnt,
                     block, segment, scale, unpermute=True)
        o_perm = None
    else:
        o_perm = attn_fwd(q_used, perm["k_perm"], perm["v_perm"], perm["kpos"], qpos, idx, cnt,
                          block, segment, scale)
        o = unpermute(o_perm, qpos, k.shape[1], block, segment) if permute_q else o_perm
    if keep:
        return dict(perm, imp=imp, idx=idx, cnt=cnt, o_perm=o_perm, o=o, qpos=qpos)
    return o


class PathGraph:
    """One step of the whole path (``pbs_attention`` on these q, k, v, with
    the same options) captured once as a CUDA graph. ``replay()`` launches
    every kernel of the step again as one graph launch on the current
    stream, on whatever q, k, v hold at that time (copy new inputs into
    them), and returns the same output tensor (or dict with ``keep``).
    Buffers, tensor maps and launch shapes are fixed at capture, so nothing
    is allocated or encoded per replay; inputs must keep their shapes and
    storage. A first call outside the capture sets the kernels' attributes."""

    def __init__(self, q, k, v, block, segment, mode="threshold", param=0.9, scale=0.0, **kw):
        dev = q.device
        call = lambda: pbs_attention(q, k, v, block, segment, mode, param, scale, **kw)
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            call()
        torch.cuda.current_stream(dev).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.out = call()

    def replay(self):
        self.graph.replay()
        return self.out


_COPY_STREAMS = {}


def _copy_streams(device):
    """Two copy streams per device (host to device, device to host), kept
    for the life of the process."""
    key = device.index
    if key not in _COPY_STREAMS:
        _COPY_STREAMS[key] = (torch.cuda.Stream(device), torch.cuda.Stream(device))
    return _COPY_STREAMS[key]


def attention_host(q, k, v, block, segment, mode="threshold", param=0.9, scale=0.0, out=None,
                   device=None, ws=None):
    """The whole path on host tensors (pbs_attention_host): q [b, hq, n, d],
    k, v [b, hkv, n, d] bf16 on the CPU (page-locked for overlapped copies);
    returns o [b, hq, n, d] bf16 on the CPU, valid once the device's current
    stream is synchronised. The copies run on two library-owned streams and
    overlap the compute, one KV group at a time."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        if t.device.type != "cpu" or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{nm}: contiguous bf16 CPU tensor expected")
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    b, hq, n, d = q.shape
    shp = Shape(b, hq, k.shape[1], n, d, block, segment)
    o = out if out is not None else torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    need = workspace_bytes(shp, _lib.OP_HOST_PATH)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    h2d, d2h = _copy_streams(device)
    mode_id = _lib.SEL[mode] if isinstance(mode, str) else int(mode)
    _call("pbs_attention_host", _ptr(q), _ptr(k), _ptr(v), _ptr(o), shp, mode_id, param, scale,
          _ptr(ws), need, _stream(device),
          ctypes.c_void_p(h2d.cuda_stream),
          ctypes.c_void_p(d2h.cuda_stream))
    return o
