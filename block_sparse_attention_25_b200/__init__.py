"""Retained-mass block-sparse attention for long 3D video token sequences on B200.

The compute path is libbsattn.so (hand-written sm_100a CUDA behind a C ABI, declared in
include/bsattn.h); this package is its thin binding plus the seeded input generator.
"""
from .bsattn import (  # noqa: F401
    BsaError, Shape, bsattn_fwd, block_mass, dense_fwd_mass, pooled_mass, OP_POOLED_MASS, clear_status, default_scale, device_status,
    device_status_words, lib, new_workspace, tile_permute, tile_permute_quant_e4m3, topp_select,
    workspace_bytes, OP_BLOCK_MASS, OP_FWD, OP_TOPP_SELECT, OP_PATTERN, pattern_csr,
    topp_select_noalloc, PAT_DIAGONAL, PAT_MULTI_DIAGONAL, PAT_VERTICAL_STRIPE, PAT_SURROUNDING,
    PAT_CRISS_CROSS, ClusterShape, kmeans, cluster_layout, cluster_permute, cluster_mass,
    topp_select_rows, cluster_fwd, new_cluster_workspace, new_cluster_fwd_workspace,
    bsattn_fwd_raster, save_lists, load_lists,
)

__all__ = [
    "BsaError", "Shape", "bsattn_fwd", "block_mass", "dense_fwd_mass", "pooled_mass", "clear_status", "default_scale",
    "device_status", "device_status_words", "lib", "new_workspace", "tile_permute",
    "tile_permute_quant_e4m3", "topp_select", "workspace_bytes", "pattern_csr",
    "topp_select_noalloc", "ClusterShape", "kmeans", "cluster_layout", "cluster_permute",
    "cluster_mass", "topp_select_rows", "cluster_fwd", "bsattn_fwd_raster", "save_lists",
    "load_lists",
]
