"""B200 (sm_100a) implementation of the prefill path of Permuted Block-Sparse
Attention: importance scoring, segment-local key permutation, block
selection, the block-sparse causal forward and the inverse permutation.

The compute lives in libpbs.so (C ABI in include/pbs.h); this package only
marshals torch tensors into it.
"""
from .ops import (PathGraph, attention_host, attn_fwd, attn_fwd_bcast, attn_fwd_gather,
                  device_status, pbs_attention, permute, score, select_blocks, shape_of,
                  unpermute, workspace_bytes)
from ._lib import EXPORTS, LIB_PATH, SEL, PbsError, Shape, lib, status_string

__all__ = ["PathGraph", "attention_host", "attn_fwd", "attn_fwd_bcast", "attn_fwd_gather",
           "device_status", "pbs_attention", "permute", "score", "select_blocks", "shape_of",
           "unpermute", "workspace_bytes", "EXPORTS", "LIB_PATH", "SEL", "PbsError", "Shape",
           "lib", "status_string"]
