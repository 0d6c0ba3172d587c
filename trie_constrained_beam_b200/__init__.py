"""Catalog-constrained wide-beam semantic-ID expansion for NVIDIA B200 (sm_100a).

The compute lives in ``libsidbeam.so`` (CUDA, C ABI in include/sidbeam.h);
``native`` is its ctypes binding and ``search`` a buffer/loop helper.
"""
from . import native  # noqa: F401
from .native import (  # noqa: F401
    SidbeamError,
    Trie,
    beam_finalize,
    beam_step,
    beam_step_gumbel,
    beam_step_gumbel_workspace_size,
    beam_step_skipped_rows,
    beam_step_noalloc,
    beam_step_workspace_size,
    catalog_score_topk,
    catalog_score_topk_sim,
    catalog_score_workspace_size,
    fused_lmhead_step,
    fused_lmhead_workspace_size,
    lmhead_logits,
    sid_trie_build,
    sid_trie_info,
    sid_trie_leaf_codes,
    sid_trie_leaf_rows,
    sidbeam_get_device_status,
    sidbeam_last_error,
    sidbeam_version,
)
from .search import BeamSearch  # noqa: F401

__version__ = "0.1.0"
