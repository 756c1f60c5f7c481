"""ctypes view of libpbs.so (include/pbs.h). Loading fails loudly when the
library has not been built: there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpbs.so")

# pbs_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_ASSERT, ERR_WORKSPACE = range(7)
# pbs_sel_mode
SEL = {"threshold": 0, "topk_frac": 1, "all": 2, "dense_causal": 3}
# pbs_op
OP_SCORE, OP_PERMUTE, OP_SELECT, OP_ATTN, OP_UNPERMUTE, OP_HOST_PATH = range(6)

# every entry point declared in include/pbs.h
EXPORTS = ("pbs_workspace_bytes", "pbs_score", "pbs_score_static", "pbs_permute",
           "pbs_select_blocks", "pbs_attn_fwd", "pbs_unpermute", "pbs_attn_fwd_unpermute",
           "pbs_attn_fwd_gather", "pbs_attn_fwd_bcast", "pbs_attention_host", "pbs_block_mass", "pbs_coverage", "pbs_get_device_status",
           "pbs_status_string", "pbs_version")


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("hq", ctypes.c_int), ("hkv", ctypes.c_int),
                ("n", ctypes.c_int), ("d", ctypes.c_int), ("block", ctypes.c_int),
                ("segment", ctypes.c_int)]


class PbsError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "pbs_workspace_bytes": (_sz, [Shape, _i]),
    "pbs_score": (_i, [_vp, _vp, _vp, Shape, _f, _vp, _sz, _vp]),
    "pbs_score_static": (_i, [_vp, _vp, _vp, Shape, _f, _vp]),
    "pbs_permute": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, Shape, _vp]),
    "pbs_select_blocks": (_i, [_vp, _vp, _vp, Shape, _i, _f, _f, _vp, _vp, _vp, _vp, _sz, _vp]),
    "pbs_attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, Shape, _f, _vp]),
    "pbs_unpermute": (_i, [_vp, _vp, _vp, Shape, _vp]),
    "pbs_attn_fwd_unpermute": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, Shape, _f, _vp]),
    "pbs_attn_fwd_gather": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, Shape, _f, _i,
                                 _vp]),
    "pbs_attn_fwd_bcast": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(_vp), _i, _i, _i,
                                Shape, _f, _vp]),
    "pbs_block_mass": (_i, [_vp, _vp, _vp, _vp, Shape, _f, _vp]),
    "pbs_coverage": (_i, [_vp, _vp, _vp, ctypes.c_double, _vp, _vp, Shape, _vp]),
    "pbs_attention_host": (_i, [_vp, _vp, _vp, _vp, Shape, _i, _f, _f, _vp, _sz,
                                _vp, _vp, _vp]),
    "pbs_get_device_status": (_i, [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "pbs_status_string": (ctypes.c_char_p, [_i]),
    "pbs_version": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m long_context_sparse_segment_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().pbs_status_string(status).decode()


def check(status: int, what: str) -> None:
    if status != OK:
        raise PbsError(status, what)
