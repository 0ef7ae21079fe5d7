"""Workload definitions: shapes and input recipes of the five synthetic decode steps.

These are plain data. They hold no arithmetic of the method (scoring, selection,
attention); they only say what shapes the synthetic inputs have and how they are drawn.

The shapes follow the pages' workloads:
  * "Jet-QSparse" (Full text): 128K context, batch 16, 128-token blocks, 64 / 128
    blocks per KV head, NVFP4 keys, FP16 value aggregation with FP32 accumulation.
  * "Joint Subspace Sparse Attention" (Fig. 1, Fig. 3, Fig. 4, Table 12): token-level
    budget B = 2,048, projection rank r = 32 / 64, group-mean query scoring.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    context: int                 # L for fixed-length workloads (tokens incl. the current one)
    block_size: int              # S
    budget: int                  # k, in blocks
    proxy_rank: int              # r > 0: projected-key proxy; 0: NVFP4, centroid or binary
    proxy_dtype: str             # 'f32' | 'bf16' | 'e4m3' | 'nvfp4' | 'centroid' | 'rabitq'
    v_dtype: str                 # stored V: 'bf16' | 'f16'
    v_agg_dtype: str             # PV operand precision: 'bf16' | 'f16'
    out_dtype: str               # 'f32' | 'bf16'
    force_sink: bool
    force_last: bool
    n_keep_hp: int               # NVFP4: blocks kept at full precision (always selected)
    softmax_scale: float         # 0 => 1/sqrt(d)
    key_recipe: str              # 'outliers' | 'offset' | 'mixture'
    query_recipe: str            # 'needle' | 'normal' | 'planted'
    seed: int
    page_size: int = 128
    ragged: bool = False         # lengths drawn per sequence (mixture workload)
    n_outlier_ch: int = 0
    outlier_scale: float = 1.0
    needle_block: int = -1
    needle_boost: float = 0.0    # >0: the needle block's keys get +boost*w before rounding
    n_planted: int = 0
    calib_tokens: int = 4096     # NVFP4 centring / tensor-scale calibration prefix
    ragged_overrides: tuple = ()  # ((seq, L), ...) applied after the uniform draw
    ragged_min: int = 4096
    ragged_max: int = 131072
    top_p: float = 0.0           # > 0: top-p selection of this share of the estimated mass,
                                 # at most `budget` blocks (binary proxy)
    key_storage: str = "bf16"    # 'nvfp4': the attention reads the NVFP4 keys (kept blocks BF16)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale > 0 else self.head_dim ** -0.5

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# Tiny decode step with a planted needle block (block 37 of 128). Its output is FP32, so
# the P.V operands are FP16 (P rounded at 2^-11 relative; BF16 values convert exactly):
# BF16 P (2^-8) cannot hold the FP32 output's relative-L2 bound of 1e-3.
TINY = Workload(
    name="tiny_needle_b1_h4_d64_L2048", batch=1, n_q_heads=4, n_kv_heads=1, head_dim=64,
    context=2048, block_size=16, budget=8, proxy_rank=16, proxy_dtype="f32",
    v_dtype="bf16", v_agg_dtype="f16", out_dtype="f32", force_sink=False, force_last=False,
    n_keep_hp=0, softmax_scale=1.0 / 8.0, key_recipe="outliers", query_recipe="needle",
    seed=1001, n_outlier_ch=2, outlier_scale=8.0, needle_block=37)

# Same as TINY, but the needle block's keys are pushed along a drawn unit direction so
# that the needle is guaranteed to beat the block-max noise (used for the invariant).
TINY_NEEDLE = TINY.replace(name="tiny_needle_boosted", needle_boost=12.0)

# Token-level selection (S = 1), B = 2,048 tokens per KV head, FP16 value aggregation.
TOKEN32K = Workload(
    name="token_b16_h32kv8_d128_L32768_r32_B2048", batch=16, n_q_heads=32, n_kv_heads=8,
    head_dim=128, context=32768, block_size=1, budget=2048, proxy_rank=32, proxy_dtype="bf16",
    v_dtype="bf16", v_agg_dtype="f16", out_dtype="bf16", force_sink=False, force_last=False,
    n_keep_hp=0, softmax_scale=0.0, key_recipe="outliers", query_recipe="normal", seed=1002,
    n_outlier_ch=4, outlier_scale=10.0)

# Block-level long-context decode: the headline 128K, batch-16 step.
BLOCK128K = Workload(
    name="block_b16_h40kv8_d128_L131072_S128_k64_r32", batch=16, n_q_heads=40, n_kv_heads=8,
    head_dim=128, context=131072, block_size=128, budget=64, proxy_rank=32, proxy_dtype="bf16",
    v_dtype="bf16", v_agg_dtype="bf16", out_dtype="bf16", force_sink=True, force_last=True,
    n_keep_hp=0, softmax_scale=0.0, key_recipe="offset", query_recipe="planted", seed=1003,
    n_planted=8)

# NVFP4 centred-key scan with the 128K shapes; V stored FP16; 2 blocks kept in BF16.
NVFP4_128K = BLOCK128K.replace(
    name="nvfp4_b16_h40kv8_d128_L131072_S128_k128", budget=128, proxy_rank=0,
    proxy_dtype="nvfp4", v_dtype="f16", v_agg_dtype="f16", n_keep_hp=2, seed=1004)

# The NVFP4 storage variant ("Jet-QSparse ...", Full text): the same step, with the
# attention reading every key from the NVFP4 cache (dequantised, un-centred, rounded to
# BF16) except the two kept blocks, whose BF16 keys are read.
NVFP4_STORE_128K = NVFP4_128K.replace(name="nvfp4store_b16_h40kv8_d128_L131072_S128_k128",
                                      key_storage="nvfp4", seed=1015)

# The 128K block-level step with the projected-key cache stored as FP8 E4M3 ("Joint Subspace
# Sparse Attention for Efficient Long-Context Decoding", Figure 10: FP8 or BF16 scoring
# cache; the full KV cache and the attention stay BF16).
FP8_128K = BLOCK128K.replace(name="fp8_b16_h40kv8_d128_L131072_S128_k64_r32", proxy_dtype="e4m3",
                             seed=1006)

# Token-level selection over an FP8 E4M3 projected-key cache of rank 64 (B = 2,048 tokens).
FP8_TOKEN32K = TOKEN32K.replace(name="fp8_token_b16_h32kv8_d128_L32768_r64_B2048",
                                proxy_rank=64, proxy_dtype="e4m3", seed=1007)

# Token-level selection at 128K context, B = 2,048 tokens per KV head: the setting of the
# component-level latency ("Joint Subspace Sparse Attention ...", Figure 9) and of the
# gather-free comparison (Figure 6); selection over 131,072 candidates per row.
TOKEN128K = TOKEN32K.replace(name="token_b16_h32kv8_d128_L131072_r32_B2048", context=131072,
                             seed=1010)

# Centroid scoring ("Coarse Semantic Blocks ...", Abstract): each block scored by the mean
# of its keys against the group-mean query, from per-block FP32 key sums (no projection).
CENTROID_128K = BLOCK128K.replace(name="centroid_b16_h40kv8_d128_L131072_S128_k64",
                                  proxy_rank=0, proxy_dtype="centroid", seed=1008)
# The same with 32-token blocks (four centroids per page), k = 256 blocks.
CENTROID_S32 = BLOCK128K.replace(name="centroid_b16_h40kv8_d128_L131072_S32_k256", block_size=32,
                                 budget=256, proxy_rank=0, proxy_dtype="centroid", seed=1009)

# Binary (RaBitQ) proxy with a top-p budget ("RaBitQCache", Abstract): 1-bit codes of the
# rotated centred keys against a 4-bit query code; the fewest tokens whose estimated
# attention mass reaches p = 0.9, at most 2,048 per KV head. The 128K token-level shape,
# so it compares with the rank-32 top-k step on the same keys and queries' recipe.
RABITQ_TOKEN128K = TOKEN128K.replace(name="rabitq_b16_h32kv8_d128_L131072_p0.9_B2048",
                                     proxy_rank=0, proxy_dtype="rabitq", top_p=0.9, seed=1013)

# Semantic blocks ("Coarse Semantic Blocks ...", Abstract): a k-means index over each
# sequence's prompt (all but the newest token), clusters of about 128 tokens, the 64
# best-scoring clusters attended, together with every token after the prompt. Keys from
# the mixture recipe, so that clusters of non-contiguous tokens exist.
SEMANTIC_128K = BLOCK128K.replace(name="semantic_b16_h40kv8_d128_L131072_S128_k64",
                                  proxy_rank=0, proxy_dtype="semantic", key_recipe="mixture",
                                  query_recipe="normal", force_sink=False, force_last=False,
                                  seed=1014)

# Ragged batch: 32 sequences, lengths uniform in [4096, 131072], G = 8, r = 64, S = 64.
RAGGED = Workload(
    name="ragged_b32_h64kv8_d128_S64_k32_r64", batch=32, n_q_heads=64, n_kv_heads=8,
    head_dim=128, context=131072, block_size=64, budget=32, proxy_rank=64, proxy_dtype="bf16",
    v_dtype="bf16", v_agg_dtype="bf16", out_dtype="bf16", force_sink=True, force_last=True,
    n_keep_hp=0, softmax_scale=0.0, key_recipe="mixture", query_recipe="normal", seed=1005,
    ragged=True, ragged_overrides=((29, 100), (30, 1000), (31, 2047)))

# d = 64 variants of the tiny step: FP8 projected keys (rank 32) and centroid scoring
TINY_FP8 = TINY.replace(name="tiny_fp8_b1_h4_d64_L2048_r32", proxy_rank=32, proxy_dtype="e4m3",
                        seed=1011)
TINY_CENTROID = TINY.replace(name="tiny_centroid_b1_h4_d64_L2048", proxy_rank=0,
                             proxy_dtype="centroid", seed=1012)

FULL = {w.name: w for w in (TINY, TOKEN32K, BLOCK128K, NVFP4_128K, RAGGED)}
ORDER = [TINY, TOKEN32K, BLOCK128K, NVFP4_128K, RAGGED]
# variants of the configurations above (FP8 projected keys, centroid scoring, 128K token
# level, the binary proxy with a top-p budget)
VARIANTS = [FP8_128K, FP8_TOKEN32K, CENTROID_128K, CENTROID_S32, TOKEN128K, RABITQ_TOKEN128K,
            NVFP4_STORE_128K]
# SEMANTIC_128K is not among them: its oracle step also needs the prompt length.


def small(w: Workload) -> Workload:
    """A reduced-size copy of a workload that the CPU oracle finishes in seconds.

    Sizes still span several tiles, several pages and a ragged tail (a context that is not
    a multiple of the block or page size), and keep every structural feature.
    """
    if w.name.startswith("tiny"):
        return w
    if w.proxy_dtype == "nvfp4":
        return w.replace(name=w.name + "_small", batch=2, context=5000 + 77, budget=12,
                         calib_tokens=1024)
    if w.ragged:
        return w.replace(name=w.name + "_small", batch=5, context=3000, budget=10,
                         ragged_min=700, ragged_max=3000,
                         ragged_overrides=((3, 100), (4, 641)))
    if w.block_size == 1:
        return w.replace(name=w.name + "_small", batch=2, context=3000 + 13, budget=200)
    return w.replace(name=w.name + "_small", batch=2, context=6000 + 45, budget=12,
                     n_planted=4)
