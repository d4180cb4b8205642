"""B200-native token-sparse layer library (Jenga contextual token sparsity).

The compute path is libjenga.so (hand-written sm_100a CUDA behind the C ABI in
include/jenga.h); this package is its Python binding.  Importing it does not
need a GPU; calling an op without the built library or without a CUDA device
raises -- there is no CPU fallback.
"""
from . import _lib  # noqa: F401
from .api import (LayerHandle, jenga_check_device_status, jenga_gather, jenga_layer_score_qk,  # noqa: F401
                  jenga_compose_block_indices, jenga_lm_loss_segmented, jenga_mlp_block_scores, jenga_predict_blocks, jenga_predict_blocks_qk, jenga_profile_enable, jenga_profile_report, jenga_scale_rows,
                  jenga_scatter_add, jenga_score_blocks, jenga_select, jenga_set_wait_budget_ns,
                  jenga_sparse_layer_bwd, jenga_sparse_layer_fwd, jenga_sparse_layer_fwd_mlp, jenga_test_gemm, jenga_version, new_lora_grads)

__all__ = [n for n in dir() if n.startswith("jenga_")] + ["LayerHandle", "new_lora_grads"]
