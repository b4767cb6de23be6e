"""CSA2 hierarchical sparse-attention decode on B200 (sm_100a).

The compute path is libcsa2.so (hand-written CUDA kernels behind a C ABI,
include/csa2.h); ``csa2`` is its thin Python binding.
"""
from .csa2 import (EXPORTS, FULL, REINDEX, REUSE, Csa2Error, Layer, LayerPlan, Rows, check_status,
                   csa2_fp4_quantize, csa2_index_full, csa2_layer_plan, csa2_reindex, csa2_sparse_attn_fp4,
                   csa2_topk_pool, lib, new_status)

__all__ = ["EXPORTS", "FULL", "REINDEX", "REUSE", "Csa2Error", "Layer", "LayerPlan", "Rows", "check_status",
           "csa2_fp4_quantize", "csa2_index_full", "csa2_layer_plan", "csa2_reindex", "csa2_sparse_attn_fp4",
           "csa2_topk_pool", "lib", "new_status"]
