"""Sparse spatiotemporal attention for video latents on B200 (sm_100a).

The compute lives in libsta.so (C ABI in include/sta.h); this package is its
Python binding plus host-side buffer plumbing.  Importing the package loads
the library and fails if it has not been built.
"""
from . import _lib
from ._lib import (AttnParams, BlockLists, Problem, SelectorParams, StaError, STA_ATTN_LISTS,
                   STA_ATTN_ROUTED, STA_BF16, STA_F32, STA_SEL_ENTROPY, STA_SEL_IBCS_SIP,
                   STA_SEL_DYNRAD, STA_SEL_RADIAL, STA_SEL_ROUTED, STA_SEL_TRA_TOKEN,
                   STA_DEV_BAD_INDEX, STA_DEV_CAPACITY, STA_DEV_DEBUG, STA_DEV_EMPTY_ROW,
                   STA_DEV_TIMEOUT)
from .api import (sta_attn_workspace, sta_build_blocks, sta_build_blocks_rows,
                  sta_build_blocks_workspace, sta_debug_build, sta_dense_attn_entropy_fwd,
                  sta_dense_attn_fwd, sta_dev_status_string, sta_permute_tokens,
                  sta_selftest_index_check, sta_sparse_attn_fwd, sta_sparse_attn_fwd_noalloc,
                  sta_status_string, sta_version)

_lib.load()
