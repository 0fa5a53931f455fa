"""B200 (sm_100a) head-aware tile-sparse attention (Veda).

The C ABI lives in ``include/veda.h`` and ``libveda.so`` (built in-tree by
``build.py``); ``binding`` is its ctypes wrapper and ``pipeline`` chains the
calls into the per-layer inference path.  Importing this package loads the
library and fails loudly if it is not built.
"""
from .binding import (  # noqa: F401
    LIB, LIB_PATH, Problem, VedaError, make_mlp, make_mlp_grad, veda_attn_backward_workspace, veda_attn_config, veda_bounds_checked, veda_distill_loss_grad,
    veda_distill_workspace, veda_head_error, veda_score_topk_workspace, veda_selftest_bounds, veda_selftest_wait_timeout,
    veda_set_wait_timeout_ns, veda_sync_status, veda_tile_map_maxpool, veda_tile_map_maxpool_grid, veda_tile_map_workspace, veda_tile_permute, veda_tile_permute_tripool,
    veda_tile_score_topk, veda_tile_sparse_attn, veda_tile_sparse_attn_backward_grid, veda_tile_sparse_attn_grid, veda_tile_unpermute, veda_tripool,
    veda_tripool_grid, veda_version)
from .pipeline import VedaAttention, VedaAttentionHost, tile_sparse_attention  # noqa: F401
from .tiling_search import tiling_search  # noqa: F401
