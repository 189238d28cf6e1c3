"""PBSA (Persistent Block-Sparse Attention) for B200: C-ABI CUDA library + thin binding.

``_lib`` mirrors the C entry points of ``include/pbsa.h`` (marshalling only); ``cache``
sequences them for one attention layer's KV cache; ``inputs`` draws seeded synthetic
workloads.  The CUDA library is loaded on first use and its absence is an error.
"""
from ._lib import (PBSAError, Geom, make_geom, load, pbsa_attend, pbsa_attend_bwd, pbsa_blockify,
                   pbsa_blockify_hsa_select, pbsa_blockify_kv, pbsa_blockify_score_select, pbsa_blockify_select_ex,
                   pbsa_blockify_train_select,
                   pbsa_bwd_workspace_bytes, pbsa_get_device_error, pbsa_memory_update,
                   pbsa_memory_update_apply, pbsa_memory_update_noalloc, pbsa_memory_update_noalloc_error,
                   pbsa_memory_update_plan,
                   pbsa_score_select, pbsa_selftest_wait_timeout, pbsa_status_string, pbsa_workspace_bytes)
from .cache import ChunkDecodeStep, LayerConfig, PBSALayerCache

__all__ = ["PBSAError", "Geom", "make_geom", "load", "pbsa_attend", "pbsa_attend_bwd", "pbsa_blockify",
           "pbsa_blockify_hsa_select", "pbsa_blockify_kv", "pbsa_blockify_score_select", "pbsa_blockify_select_ex",
           "pbsa_blockify_train_select",
           "pbsa_bwd_workspace_bytes", "pbsa_get_device_error", "pbsa_memory_update", "pbsa_memory_update_apply",
           "pbsa_memory_update_noalloc", "pbsa_memory_update_noalloc_error", "pbsa_memory_update_plan", "pbsa_score_select",
           "pbsa_selftest_wait_timeout", "pbsa_status_string", "pbsa_workspace_bytes", "ChunkDecodeStep", "LayerConfig", "PBSALayerCache"]
