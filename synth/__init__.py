"""Seeded synthetic inputs for the score-then-select decode step (no method arithmetic)."""
from .workloads import (Workload, TINY, TINY_NEEDLE, TOKEN32K, BLOCK128K, NVFP4_128K, RAGGED,
                        FP8_128K, FP8_TOKEN32K, CENTROID_128K, CENTROID_S32, TOKEN128K,
                        TINY_FP8, TINY_CENTROID, RABITQ_TOKEN128K, SEMANTIC_128K, NVFP4_STORE_128K,
                        FULL, ORDER, VARIANTS, small)
from .gen import (Inputs, lengths, proj_matrix, page_table, row_kv, row_queries, calibration,
                  rotations, rounding_draws)

__all__ = ["Workload", "TINY", "TINY_NEEDLE", "TOKEN32K", "BLOCK128K", "NVFP4_128K", "RAGGED",
           "FP8_128K", "FP8_TOKEN32K", "CENTROID_128K", "CENTROID_S32", "TOKEN128K",
           "TINY_FP8", "TINY_CENTROID", "RABITQ_TOKEN128K", "SEMANTIC_128K", "NVFP4_STORE_128K",
           "FULL", "ORDER",
           "VARIANTS", "small", "Inputs",
           "lengths", "proj_matrix", "page_table", "row_kv", "row_queries", "calibration",
           "rotations", "rounding_draws"]
