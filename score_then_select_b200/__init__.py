"""Score-then-select sparse decode attention for B200 (sm_100a).

The decode path runs in libqs.so (hand-written CUDA behind the C ABI in include/qs.h);
this package is its ctypes binding plus torch helpers that allocate the caches. There is
no CPU fallback: importing the binding's entry points requires the built library.
"""
from .binding import (QsError, LIB_PATH, EXPORTS, lib, make_config, make_cache, qs_version,
                      qs_workspace_size, qs_workspace_init, qs_append_kv, qs_score,
                      qs_select_topk, qs_sparse_attn, qs_decode, qs_device_status,
                      qs_sparse_attn_noalloc, qs_attention_launches, qs_selftest_wait_timeout,
                      qs_dense_workspace_size, qs_dense_attn, qs_gather_kv,
                      qs_calib_workspace_size, qs_calibrate_basis, qs_rabitq_score,
                      qs_select_top_p, qs_decode_top_p, qs_gather_kv_nvfp4k, qs_select_topk_radix,
                      qs_semantic_index_workspace_size,
                      qs_semantic_index, qs_semantic_select, status_string)

__all__ = ["QsError", "LIB_PATH", "EXPORTS", "lib", "make_config", "make_cache", "qs_version",
           "qs_workspace_size", "qs_workspace_init", "qs_append_kv", "qs_score",
           "qs_select_topk", "qs_sparse_attn", "qs_decode", "qs_device_status", "status_string",
           "qs_sparse_attn_noalloc", "qs_attention_launches", "qs_selftest_wait_timeout",
           "qs_dense_workspace_size", "qs_dense_attn", "qs_gather_kv",
           "qs_calib_workspace_size", "qs_calibrate_basis", "qs_rabitq_score",
           "qs_select_top_p", "qs_decode_top_p", "qs_gather_kv_nvfp4k", "qs_select_topk_radix",
           "qs_semantic_index_workspace_size",
           "qs_semantic_index", "qs_semantic_select"]
