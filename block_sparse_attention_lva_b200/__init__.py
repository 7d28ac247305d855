"""Block-sparse softmax attention for video diffusion transformers on B200 (sm_100a).

The compute lives in ``liblva.so`` (C ABI, ``include/lva.h``): a spatiotemporal-tile token
reorder, a GPU block-mask -> CSR builder, and a TMA + tcgen05 block-sparse attention
kernel.  This package is the thin Python binding over it; importing it loads the library
and fails if the library has not been built.
"""
from ._binding import (LVA_MASK_ALL, LVA_MASK_LVSA_FRAMES, LVA_MASK_STATIC, LVA_MASK_TWO_STAGE,
                       LVA_MASK_WINDOW_ANCHOR,
                       LIB_PATH, LvaError, MaskParams, lva_block_mask_max_nnz, lva_block_sparse_attn,
                       lva_aggregate_masks, lva_block_energy, lva_block_sparse_attn_raster, lva_block_sparse_lse,
                       lva_broadcast_blocks, lva_window_transposed_attn,
                       lva_build_block_mask, lva_build_block_mask_ws, lva_block_mask_workspace_bytes,
                       lva_build_block_mask_noalloc,
                       lva_device_error, lva_reorder_tokens, lva_select_blocks,
                       lva_selftest_wait, lva_version, lva_layer_step_host)
from .pipeline import SquadTwoPass, StaticMaskCalibrator, VideoBlockSparseAttention, mask_params_for
from .sharding import HeadShard, head_range, shard_rows

__all__ = ["LVA_MASK_ALL", "LVA_MASK_LVSA_FRAMES", "LVA_MASK_STATIC", "LVA_MASK_TWO_STAGE", "LVA_MASK_WINDOW_ANCHOR", "LIB_PATH",
           "LvaError", "MaskParams", "lva_block_mask_max_nnz", "lva_block_sparse_attn", "lva_broadcast_blocks",
           "lva_build_block_mask", "lva_build_block_mask_ws", "lva_block_mask_workspace_bytes",
           "lva_build_block_mask_noalloc",
           "lva_device_error", "lva_reorder_tokens", "lva_version",
           "lva_block_energy", "lva_select_blocks", "lva_aggregate_masks", "lva_block_sparse_attn_raster", "lva_block_sparse_lse",
           "lva_window_transposed_attn", "lva_selftest_wait", "lva_layer_step_host",
           "SquadTwoPass", "StaticMaskCalibrator", "VideoBlockSparseAttention", "mask_params_for",
           "HeadShard", "head_range", "shard_rows"]
