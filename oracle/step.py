"""One decode step of one row (sequence b, KV head g), composed from the oracle's parts.

TEST INFRASTRUCTURE: only tests, the smoke check and the bench's CPU-baseline leg use this.

Order of the step, following "Joint Subspace Sparse Attention for Efficient Long-Context
Decoding" (Figure 1) and "Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse
Attention" (Full text):
  1. the row's scoring cache: projected keys k . P (stored f32 / bf16), or the centred
     keys packed to NVFP4;
  2. proxy block scores beta (max over each block's valid tokens);
  3. forced blocks plus the best-scoring rest, ascending;
  4. exact softmax attention of every query head of the group over the selected tokens.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import formats as F
from . import method as M


@dataclass
class RowParams:
    S: int                     # block size
    budget: int                # k, blocks
    scale: float               # softmax scale
    proxy: str                 # 'f32' | 'bf16' | 'e4m3' | 'nvfp4' | 'centroid'
    v_dtype: str               # 'bf16' | 'f16'
    force_sink: bool = False
    force_last: bool = False
    n_keep: int = 0            # NVFP4: blocks kept at full precision
    key_storage: str = "bf16"  # 'nvfp4': attention over the NVFP4 storage variant's keys


def row_params_of(w) -> RowParams:
    """The row parameters of a workload description (its block size, budget, softmax scale,
    proxy kind, value format and forced blocks)."""
    return RowParams(S=w.block_size, budget=w.budget, scale=w.scale, proxy=w.proxy_dtype,
                     v_dtype=w.v_dtype, force_sink=w.force_sink, force_last=w.force_last,
                     n_keep=w.n_keep_hp, key_storage=getattr(w, "key_storage", "bf16"))


def decode_v(v_bits: np.ndarray, v_dtype: str) -> np.ndarray:
    return F.f16_to_f64(v_bits) if v_dtype == "f16" else F.bf16_to_f64(v_bits)


def row_scoring_cache(p: RowParams, k_bits, P=None, mu=None, g_k=None):
    """The row's stored scoring cache: proxy entries, (codes, scales, x32) for NVFP4, or the
    per-block key sums for centroid scoring."""
    if p.proxy == "centroid":
        return M.centroid_sums(k_bits, p.S, len(k_bits))
    if p.proxy == "nvfp4":
        x32 = M.centre(k_bits, mu)
        codes, scales = M.nvfp4_pack(x32, g_k)
        return codes, scales, x32
    return M.proxy_store(k_bits, P, p.proxy)


def row_block_scores(p: RowParams, cache, q_bits, L: int, P=None, g_q=None, g_k=None,
                     q_all_bits=None):
    """beta [nb] for one row from its scoring cache."""
    if p.proxy == "centroid":
        return M.centroid_block_scores(q_bits, cache[:-(-L // p.S)], p.S, L)
    if p.proxy == "nvfp4":
        codes, scales, _ = cache
        qx = F.bf16_to_f64(q_bits).astype(np.float32)
        q_codes, q_scales = M.nvfp4_pack(qx, g_q)
        hs = M.nvfp4_head_scores(q_codes, q_scales, g_q, codes[:L], scales[:L], g_k)
        return M.nvfp4_block_scores(hs, p.S)
    qt = M.proxy_query(q_bits, P)
    s = M.token_scores(M.proxy_decode(cache, p.proxy)[:L], qt)
    return M.block_max(s, p.S)


def row_forced(p: RowParams, nb: int, cache=None, L: int = 0, g_k=None):
    keep = ()
    if p.proxy == "nvfp4" and p.n_keep > 0:
        codes, scales, x32 = cache
        err = M.block_quant_error(x32[:L], codes[:L], scales[:L], g_k, p.S, L)
        keep = M.kept_blocks(err, p.n_keep)
    return M.forced_blocks(nb, p.force_sink, p.force_last, keep), keep


def decode_row(p: RowParams, k_bits, v_bits, q_bits, L: int, P=None, mu=None, g_k=None,
               g_q=None, sel_override=None, keep_override=None):
    """Full oracle step for one row. Returns a dict of every intermediate.

    ``sel_override``: attend over this selection instead of the oracle's own (used once a
    GPU selection has been accepted as a valid top-k under the near-tie rule).
    ``keep_override``: with NVFP4 key storage, the kept (BF16) blocks whose stored keys are
    attended (used once the GPU's kept pair has been accepted under the near-tie rule).

    With ``p.key_storage == 'nvfp4'`` ("Jet-QSparse ...", Full text: the persistent cache
    keeps the attended keys in NVFP4, at most two blocks per sequence at BF16, and attention
    is computed on them), the keys attended are nvfp4_attended_keys: the kept blocks'
    stored BF16 keys, elsewhere the NVFP4 value dequantised and un-centred, exactly
    (returned as ``K_att``).
    """
    cache = row_scoring_cache(p, k_bits[:L], P, mu, g_k)
    beta = row_block_scores(p, cache, q_bits, L, P=P, g_q=g_q, g_k=g_k)
    nb = beta.shape[0]
    forced, keep = row_forced(p, nb, cache, L, g_k)
    sel = M.select_blocks(beta, p.budget, forced)
    use = sel if sel_override is None else np.asarray(sel_override, dtype=np.int64)
    tokens = M.block_tokens(use, p.S, L)
    q = F.bf16_to_f64(q_bits)
    if p.key_storage == "nvfp4":
        codes, scales, _ = cache
        kept = keep if keep_override is None else np.asarray(keep_override, dtype=np.int64)
        K = M.nvfp4_attended_keys(k_bits[:L], codes, scales, g_k, mu, kept, p.S, L)
    else:
        K = F.bf16_to_f64(k_bits[:L])
    V = decode_v(v_bits[:L], p.v_dtype)
    out = M.sparse_attention(q, K, V, tokens, p.scale)
    return dict(cache=cache, beta=beta, forced=forced, keep=keep, sel=sel, tokens=tokens,
                out=out, K_att=K)


# ---- the binary proxy with a top-p budget ("RaBitQCache", Abstract) ------------------------

@dataclass
class TopPParams:
    S: int                     # block size (1: token level)
    p: float                   # fraction of the estimated attention mass to cover
    budget: int                # most blocks a row may attend
    scale: float               # softmax scale (estimated weights and attention)
    v_dtype: str               # 'bf16' | 'f16'
    force_sink: bool = False
    force_last: bool = False


def top_p_params_of(w) -> TopPParams:
    """The binary proxy's row parameters of a workload description; p as the float32 that
    the library takes."""
    return TopPParams(S=w.block_size, p=float(np.float32(w.top_p)), budget=w.budget,
                      scale=w.scale, v_dtype=w.v_dtype, force_sink=w.force_sink,
                      force_last=w.force_last)


def decode_row_top_p(p: TopPParams, k_bits, v_bits, q_bits, L: int, R, c, u,
                     sel_override=None):
    """One row's step with the binary proxy: codes of the keys, the query's 4-bit code,
    estimated scores and weights, block masses, the top-p selection, then exact attention
    over the selected tokens. R: rotation [d][d]; c: the row's centre [d]; u: the query's
    rounding draws [d]."""
    bits, g = M.rabitq_encode(k_bits[:L], R, c)
    n, delta, vl, qbar = M.rabitq_query(q_bits, R, u)
    s = M.rabitq_scores(bits, g, n, delta, vl, c, qbar)
    w = M.estimated_weights(s, p.scale)
    mass = M.block_mass(w, p.S)
    forced = M.forced_blocks(mass.shape[0], p.force_sink, p.force_last)
    sel = M.select_top_p(mass, p.p, p.budget, forced)
    use = sel if sel_override is None else np.asarray(sel_override, dtype=np.int64)
    tokens = M.block_tokens(use, p.S, L)
    out = M.sparse_attention(F.bf16_to_f64(q_bits), F.bf16_to_f64(k_bits[:L]),
                             decode_v(v_bits[:L], p.v_dtype), tokens, p.scale)
    return dict(bits=bits, g=g, codes=n, delta=delta, vl=vl, qbar=qbar, scores=s, weights=w,
                mass=mass, forced=forced, sel=sel, tokens=tokens, out=out)


# ---- semantic blocks ("Coarse Semantic Blocks ...", Abstract) -------------------------------

@dataclass
class SemanticParams:
    S: int                     # target tokens per cluster: C = ceil(L0 / S)
    budget: int                # clusters selected
    iters: int                 # Lloyd iterations of the index
    scale: float               # softmax scale
    v_dtype: str               # 'bf16' | 'f16'


def decode_row_semantic(p: SemanticParams, k_bits, v_bits, q_bits, L0: int, L: int,
                        sel_override=None):
    """One row's step with a semantic-block index over its first L0 tokens: cluster the
    prompt's keys, score the clusters by their centroids, select the top clusters, then
    exact attention over their members and every token after the prompt."""
    C = -(-L0 // p.S)
    assign, cent = M.kmeans_keys(k_bits[:L0], C, p.iters)
    beta = M.semantic_block_scores(q_bits, cent)
    sel = M.select_blocks(beta, p.budget, np.zeros(0, dtype=np.int64))
    use = sel if sel_override is None else np.asarray(sel_override, dtype=np.int64)
    tokens = M.semantic_tokens(assign, use, L0, L)
    out = M.sparse_attention(F.bf16_to_f64(q_bits), F.bf16_to_f64(k_bits[:L]),
                             decode_v(v_bits[:L], p.v_dtype), tokens, p.scale)
    return dict(assign=assign, centroids=cent, beta=beta, sel=sel, tokens=tokens, out=out)
