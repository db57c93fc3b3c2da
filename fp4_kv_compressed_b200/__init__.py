"""B200-native CSA2 global-attention decode path over an FP4-compressed KV cache.

The compute lives in libcsa2.so (hand-written CUDA for sm_100a behind the C ABI
of include/csa2.h).  This package is the thin Python side: a ctypes binding with
the C names (argument marshalling only) and the layer-stack driver that owns the
device buffers.  Importing it loads the library and raises if it is missing.
"""
from ._binding import (CSA2_OP_INDEX_FULL, CSA2_OP_INDEX_REINDEX, CSA2_OP_SPARSE_ATTN,
                       CSA2GlobalKV, CSA2PagedKV, CSA2Rope, CSA2SWA, Csa2Error, DEFAULT_WAIT_LIMIT_NS,
                       DEVERR_INDEX, DEVERR_NMAX, DEVERR_PAGE, DEVERR_RANGE, DEVERR_ROPE, DEVERR_SLOT,
                       DEVERR_TIMEOUT, EXPORTS, LIB_PATH, Rope, csa2_debug_set_waits,
                       csa2_attn_combine, csa2_index_full, csa2_index_full_slice, csa2_index_full_tc,
                       csa2_index_merge, csa2_index_reindex, csa2_quantize_append_paged,
                       csa2_index_full_paged, csa2_index_reindex_paged,
                       csa2_sparse_attn_decode_paged, csa2_sparse_attn_decode_reuse,
                       csa2_index_reindex_settled, csa2_index_reindex_paged_settled,
                       csa2_sparse_attn_decode_paged_reuse,
                       csa2_quantize_append, csa2_quantize_append_rope, csa2_read_device_error,
                       csa2_sparse_attn_decode, csa2_sparse_attn_decode_append,
                       csa2_sparse_attn_decode_append_rope, csa2_workspace_size, load_library)
from .stack import DecodeStack, GlobalKV, GroupSpec, LayerPlan, PagedKV, SwaRing, plan_layers

load_library()

__all__ = [
    "CSA2_OP_INDEX_FULL", "CSA2_OP_INDEX_REINDEX", "CSA2_OP_SPARSE_ATTN", "CSA2GlobalKV",
    "CSA2Rope", "CSA2SWA", "Csa2Error", "DEFAULT_WAIT_LIMIT_NS", "DEVERR_TIMEOUT",
    "csa2_debug_set_waits", "DEVERR_PAGE", "DEVERR_INDEX", "DEVERR_NMAX", "DEVERR_RANGE",
    "DEVERR_ROPE", "DEVERR_SLOT", "EXPORTS", "LIB_PATH", "Rope", "csa2_index_full",
    "csa2_index_full_tc", "csa2_index_reindex", "csa2_attn_combine", "csa2_index_full_slice",
    "csa2_index_merge", "CSA2PagedKV", "csa2_quantize_append_paged", "csa2_index_full_paged",
    "csa2_index_reindex_paged", "csa2_sparse_attn_decode_paged", "csa2_sparse_attn_decode_reuse",
    "csa2_index_reindex_settled", "csa2_index_reindex_paged_settled", "csa2_sparse_attn_decode_paged_reuse",
    "PagedKV", "csa2_quantize_append",
    "csa2_quantize_append_rope", "csa2_read_device_error", "csa2_sparse_attn_decode",
    "csa2_sparse_attn_decode_append", "csa2_sparse_attn_decode_append_rope",
    "csa2_workspace_size",
    "load_library", "DecodeStack", "GlobalKV", "GroupSpec", "LayerPlan", "SwaRing",
    "plan_layers",
]
