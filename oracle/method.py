"""Plain CPU oracle of the score-then-select decode step.

TEST INFRASTRUCTURE: only tests, the smoke check and the bench's CPU-baseline leg may
import this. It shares no code with the CUDA path and never calls it.

Everything is float64 except where the method fixes a rounding decision (the proxy
cache's stored precision, the NVFP4 codes), which is taken in float32 exactly as the
method states it, so that integer-valued results (codes, selected indices) can be
compared bit for bit.

Sources (page title, then the part of the page):
  [JSSA]  "Joint Subspace Sparse Attention for Efficient Long-Context Decoding"
          - Figure 1: for one KV head, the mean of its query heads scores a projected-key
            cache in a shared low-dimensional subspace; the top-B positions are selected;
            all query heads of the group share that index set; attention then reads the
            original full-dimensional keys and values at those positions.
          - Abstract: distinct per-KV-head selections under the standard GQA layout.
          - Table 15: per-KV-head selection (the variant built here).
          - Figure 10: the projected scoring cache may be stored at reduced precision
            while the full KV cache and the final attention stay BF16.
  [JQS]   "Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention"
          - Full text: NVFP4 cache; a dense FP4 scan scores the whole key history; 128-token
            blocks are selected; FP16 value aggregation with FP32 accumulation; calibrated
            key centring; at most two BF16 pages kept; cache packed from BF16 activations.
  [RQC]   "RaBitQCache" (the abstract page)
          - Abstract: keys scored through randomised rotated binary quantisation with
            binary-INT4 arithmetic, an unbiased estimator with an error bound, and a top-p
            budget that follows the estimated attention mass.
  [CSB]   "Coarse Semantic Blocks for Efficient Training-Free Sparse Attention"
          - Abstract: a prompt-specific key index clusters the keys into large blocks of
            non-contiguous tokens; a query scores blocks by their centroids and attends to
            the original keys and values of the blocks it selects.
  [RBQ]   The estimator's published form: J. Gao and C. Long, "RaBitQ: Quantizing
          High-Dimensional Vectors with a Theoretical Error Bound for Approximate Nearest
          Neighbor Search", SIGMOD 2024 (section 3: the codebook, the estimator and its
          unbiasedness; the randomised uniform scalar quantisation of the query).

Readings where the pages are silent (each listed in the design notes):
  * block score = max over the block's valid tokens (and, on the NVFP4 path, over the
    group's query heads); the proxy scores are unscaled (scaling does not change order);
  * forced blocks (sink, last, kept) count against the budget; ties go to the lower index;
  * attention is exact softmax over the selected tokens only;
  * the binary proxy's readings are listed above its section.

Parity pins live in tests/test_oracle_*.py. The aggregation of per-head NVFP4 scores into
one score per block (max over heads) is a reading the pages do not fix: its *definition*
is parity unpinned; its implementation is checked by brute force on tiny inputs. The same
holds for the semantic blocks' clustering algorithm.
"""
from __future__ import annotations

import numpy as np

from . import formats as F

# ============================================================================================
# Writer: projected-key cache  [JSSA, Figure 1; Figure 10]
# ============================================================================================


def proxy_keys_f32(k_bits: np.ndarray, P: np.ndarray) -> np.ndarray:
    """Projected keys k~ = k . P, evaluated in float32.

    k_bits: stored BF16 keys [n][d]; P: float32 [d][r].
    Fixed evaluation: for each output j, acc = 0; for i = 0..d-1 in order,
    acc = fp32(acc + fp32(k_i * P_ij)) (two roundings per term, no fused multiply-add).
    """
    k32 = F.bf16_to_f64(k_bits).astype(np.float32)
    P32 = np.asarray(P, dtype=np.float32)
    acc = np.zeros((k32.shape[0], P32.shape[1]), dtype=np.float32)
    for i in range(k32.shape[1]):
        prod = k32[:, i:i + 1] * P32[i:i + 1, :]       # float32 x float32 -> rounded float32
        acc = acc + prod                                # rounded float32
    return acc


def proxy_store(k_bits: np.ndarray, P: np.ndarray, dtype: str):
    """Stored proxy cache entries: float32 values ('f32'), BF16 bit patterns ('bf16') or
    FP8 E4M3 codes ('e4m3', the reduced-precision scoring cache of [JSSA, Figure 10]), each
    a rounding of the float32 projected key."""
    acc = proxy_keys_f32(k_bits, P)
    if dtype == "f32":
        return acc
    if dtype == "bf16":
        return F.f32_to_bf16_rne(acc)
    if dtype == "e4m3":
        return F.e4m3_encode(acc)
    raise ValueError(dtype)


def proxy_decode(stored, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.asarray(stored, dtype=np.float32).astype(np.float64)
    if dtype == "e4m3":
        return F.e4m3_value(stored)
    return F.bf16_to_f64(stored)


# ============================================================================================
# Score: group-mean projected query against the projected keys  [JSSA, Figure 1]
# ============================================================================================


def proxy_query(q_bits: np.ndarray, P: np.ndarray) -> np.ndarray:
    """q~ = (mean of the group's query heads) . P, float64. q_bits: BF16 [G][d]."""
    qbar = F.bf16_to_f64(q_bits).mean(axis=0)
    return qbar @ np.asarray(P, dtype=np.float64)


def token_scores(proxy: np.ndarray, qt: np.ndarray) -> np.ndarray:
    """s_t = q~ . k~_t for every token (float64). proxy: decoded [L][r]."""
    return proxy @ qt


def block_max(s: np.ndarray, S: int) -> np.ndarray:
    """beta_j = max of s over the valid tokens of block j (tokens j*S .. j*S+S-1, < L)."""
    L = s.shape[-1]
    nb = (L + S - 1) // S
    pad = nb * S - L
    if pad:
        s = np.concatenate([s, np.full(s.shape[:-1] + (pad,), -np.inf)], axis=-1)
    return s.reshape(s.shape[:-1] + (nb, S)).max(axis=-1)


# ============================================================================================
# Select: forced blocks, then the best-scoring rest  [JSSA, Figure 1; JQS, Full text]
# ============================================================================================


def forced_blocks(nb: int, force_sink: bool, force_last: bool, keep=()) -> np.ndarray:
    f = set()
    if force_sink:
        f.add(0)
    if force_last:
        f.add(nb - 1)
    for j in keep:
        if 0 <= j < nb:
            f.add(int(j))
    return np.array(sorted(f), dtype=np.int64)


def select_blocks(beta: np.ndarray, budget: int, forced: np.ndarray) -> np.ndarray:
    """Indices of the selected blocks, ascending.

    If the budget covers every block, every block is selected. Otherwise the forced blocks
    are taken first and the remaining budget - |forced| slots go to the other blocks in
    order of decreasing score, ties to the lower index.
    """
    nb = beta.shape[0]
    if nb <= budget:
        return np.arange(nb, dtype=np.int64)
    forced = np.asarray(forced, dtype=np.int64)
    is_forced = np.zeros(nb, dtype=bool)
    is_forced[forced] = True
    rest = np.nonzero(~is_forced)[0]
    order = np.lexsort((rest, -beta[rest]))             # primary: -beta, secondary: index
    take = rest[order[: budget - len(forced)]]
    return np.sort(np.concatenate([forced, take]))


def kth_threshold(beta: np.ndarray, budget: int, forced: np.ndarray):
    """(s*, tau): the last score taken from the non-forced blocks, and its tie tolerance.

    tau = 1e-4 * max(|s*|, 1e-30): the relative near-tie band within which two selections
    are both valid top-k sets.
    """
    nb = beta.shape[0]
    is_forced = np.zeros(nb, dtype=bool)
    is_forced[np.asarray(forced, dtype=np.int64)] = True
    rest = beta[~is_forced]
    need = budget - int(is_forced.sum())
    if nb <= budget or need <= 0 or rest.size == 0:
        return None, None
    s_star = np.sort(rest)[::-1][need - 1]
    return s_star, 1e-4 * max(abs(s_star), 1e-30)


def selection_valid(beta: np.ndarray, budget: int, forced: np.ndarray, got: np.ndarray,
                    rel_tol: float = 1e-4) -> tuple[bool, str]:
    """Is ``got`` a valid selection, up to near-ties at the k-th score?

    Valid iff: it has the right size; it holds every forced block; every chosen non-forced
    block scores at least s* - tau; every unchosen block scores at most s* + tau; and it
    is strictly ascending.
    """
    nb = beta.shape[0]
    got = np.asarray(got, dtype=np.int64)
    want = select_blocks(beta, budget, forced)
    if len(got) != len(want):
        return False, f"size {len(got)} != {len(want)}"
    if np.any(np.diff(got) <= 0):
        return False, "not strictly ascending"
    if np.any(got < 0) or np.any(got >= nb):
        return False, "index out of range"
    if nb <= budget:
        return bool(np.array_equal(got, want)), "dense"
    if not set(np.asarray(forced).tolist()) <= set(got.tolist()):
        return False, "forced block missing"
    if np.array_equal(got, want):
        return True, "exact"
    s_star, _ = kth_threshold(beta, budget, forced)
    tau = rel_tol * max(abs(s_star), 1e-30)
    extra = np.setdiff1d(got, want)
    missing = np.setdiff1d(want, got)
    if np.all(beta[extra] >= s_star - tau) and np.all(beta[missing] <= s_star + tau):
        return True, f"near-tie ({len(extra)} swapped)"
    return False, f"{len(extra)} swapped outside the tie band"


def block_tokens(sel: np.ndarray, S: int, L: int) -> np.ndarray:
    """Token positions covered by the selected blocks (valid tokens only), ascending."""
    if len(sel) == 0:
        return np.zeros(0, dtype=np.int64)
    t = (np.asarray(sel, dtype=np.int64)[:, None] * S + np.arange(S)[None, :]).reshape(-1)
    return t[t < L]


# ============================================================================================
# Sparse attention and the log-sum-exp combine  [JSSA, Figure 1; JQS, Full text]
# ============================================================================================


def sparse_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, tokens: np.ndarray,
                     scale: float) -> np.ndarray:
    """o_h = sum_t softmax_t(scale * q_h . k_t) v_t over the given tokens only (float64).

    q: [G][d], K/V: [L][d] (decoded), tokens: positions. Softmax is normalised over the
    selected tokens only.
    """
    Kt = K[tokens]
    Vt = V[tokens]
    logits = scale * (q @ Kt.T)                               # [G][T]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    return (p @ Vt) / p.sum(axis=1, keepdims=True)


def attention_partial(q: np.ndarray, K: np.ndarray, V: np.ndarray, tokens: np.ndarray,
                      scale: float):
    """One split's partial state (m, l, o) with o unnormalised: o = sum_t e^(x_t - m) v_t."""
    if len(tokens) == 0:
        G, d = q.shape[0], V.shape[1]
        return np.full(G, -np.inf), np.zeros(G), np.zeros((G, d))
    logits = scale * (q @ K[tokens].T)
    m = logits.max(axis=1)
    p = np.exp(logits - m[:, None])
    return m, p.sum(axis=1), p @ V[tokens]


def lse_combine(ms, ls, os_) -> np.ndarray:
    """o = sum_s e^(m_s - M) o_s / sum_s e^(m_s - M) l_s, M = max_s m_s."""
    ms = np.asarray(ms)
    M = ms.max(axis=0)
    w = np.exp(ms - M[None, :])
    w = np.where(np.isfinite(ms), w, 0.0)
    num = np.einsum("sg,sgd->gd", w, np.asarray(os_))
    den = np.einsum("sg,sg->g", w, np.asarray(ls))
    return num / den[:, None]


# ============================================================================================
# Attending over the NVFP4 keys  [JQS, Full text]
# The storage variant of the page keeps the attended keys in NVFP4 too, with at most two
# blocks per sequence kept in BF16 to bound the quantisation error, and computes attention
# on them. Reading: the key of a token in a kept block is its stored BF16 key; every other
# key is its NVFP4 scoring copy decoded and un-centred (dequantised value + the row's
# calibrated mean), exactly (nvfp4_attended_keys: what the fused attention computes with).
# nvfp4_attended_keys_bf16 is the same key rounded to BF16: what a gather into a BF16
# buffer for dense attention holds.
# ============================================================================================


def nvfp4_attended_keys(k_bits: np.ndarray, codes: np.ndarray, scales: np.ndarray, g_k,
                        mu: np.ndarray, keep, S: int, L: int) -> np.ndarray:
    """Keys [L][d] (float64) the storage variant attends over: BF16 keys in kept blocks,
    dequant(codes, scales, g_k) + mu elsewhere."""
    K = nvfp4_dequant(codes[:L], scales[:L], g_k) + np.asarray(mu, dtype=np.float32).astype(np.float64)
    bf = F.bf16_to_f64(k_bits[:L])
    for j in keep:
        t0, t1 = int(j) * S, min(L, (int(j) + 1) * S)
        K[t0:t1] = bf[t0:t1]
    return K


def nvfp4_attended_keys_bf16(k_bits: np.ndarray, codes: np.ndarray, scales: np.ndarray, g_k,
                             mu: np.ndarray, keep, S: int, L: int) -> np.ndarray:
    """The same keys as BF16 bit patterns [L][d], as an attention with BF16 operands takes
    them: kept blocks keep their stored BF16 keys; elsewhere, per element,
    bf16_rne(fp32(fp32(fp32(e * sigma) * g_k) + mu)) (e * sigma is exact in float32; the
    product with g_k and the sum with mu are each rounded to float32)."""
    n, d = codes[:L].shape
    e = F.e2m1_value(codes[:L]).astype(np.float32)
    sig = F.ue4m3_value(scales[:L]).astype(np.float32).repeat(16, axis=1)
    v = (e * sig).astype(np.float32)                                        # exact
    v = (v * np.float32(g_k)).astype(np.float32)
    v = (v + np.asarray(mu, dtype=np.float32)[None, :]).astype(np.float32)
    out = F.f32_to_bf16_rne(v)
    bits = np.asarray(k_bits[:L], dtype=np.uint16)
    for j in keep:
        t0, t1 = int(j) * S, min(L, (int(j) + 1) * S)
        out[t0:t1] = bits[t0:t1]
    return out


# ============================================================================================
# Centroid scoring of contiguous blocks  ["Coarse Semantic Blocks ...", Abstract]
# The page scores each block by its centroid against the query. Reading: the centroid of a
# block is the mean of its valid stored keys, kept as a float32 running sum in token order
# (the cache entry) and divided by the block's valid count when scoring; the block score is
# the group-mean query dotted with it, which equals the mean of the block's exact
# group-mean scores. Blocks stay contiguous (the semantic, non-contiguous clustering of
# the page is not built).
# ============================================================================================


def centroid_sums(k_bits: np.ndarray, S: int, L: int) -> np.ndarray:
    """float32 sums of the valid keys of each block, added in token order -> [nb][d]."""
    k32 = F.bf16_to_f64(k_bits[:L]).astype(np.float32)
    nb = -(-L // S)
    out = np.zeros((nb, k32.shape[1]), dtype=np.float32)
    for t in range(L):
        j = t // S
        out[j] = k32[t] if t % S == 0 else (out[j] + k32[t])   # one float32 rounding per add
    return out


def centroid_block_scores(q_bits: np.ndarray, sums: np.ndarray, S: int, L: int) -> np.ndarray:
    """beta_j = qbar . (sum_j / count_j) in float64, count_j = valid tokens of block j."""
    qbar = F.bf16_to_f64(q_bits).mean(axis=0)
    nb = sums.shape[0]
    cnt = np.minimum(S, L - np.arange(nb) * S).astype(np.float64)
    return (sums.astype(np.float64) @ qbar) / cnt


# ============================================================================================
# JSSA-style basis from calibration moments  [JSSA, Abstract; Table 9]
# The pages learn the shared subspace by minimising a tractable (marginal) bound on the
# token-score preservation error, with a closed-form spectral solution, and compare raw
# with unit-trace-normalised group-mean moments (Table 9). The bound itself is not on the
# pages. Reading: P = the top-r eigenvectors of M = C_q / tr(C_q) + C_k / tr(C_k), with
# C_q the second moment of the calibration group-mean queries and C_k that of the keys
# (each normalised to unit trace, so neither side dominates by scale). PARITY UNPINNED as
# a reading of the pages; the spectral solution of this definition is pinned.
# ============================================================================================


def calibration_moment(q_bits: np.ndarray, k_bits: np.ndarray) -> np.ndarray:
    """M = C_q / tr(C_q) + C_k / tr(C_k) for one KV head (float64).

    q_bits: BF16 calibration queries [n][G][d] (the group's heads), k_bits: BF16 keys [m][d].
    C_q = mean over positions of qbar qbar^T, qbar = mean of the group's heads; C_k likewise.
    """
    qbar = F.bf16_to_f64(q_bits).mean(axis=1)
    k = F.bf16_to_f64(k_bits)
    cq = qbar.T @ qbar / qbar.shape[0]
    ck = k.T @ k / k.shape[0]
    return cq / np.trace(cq) + ck / np.trace(ck)


def spectral_basis(Mx: np.ndarray, r: int):
    """Top-r eigenvectors of the symmetric Mx as columns of P [d][r] (eigenvalue descending),
    each signed so that its largest-magnitude entry (lowest index on ties) is positive;
    returns (P, eigenvalues[:r])."""
    w, V = np.linalg.eigh(Mx)
    order = np.argsort(-w, kind="stable")[:r]
    P = V[:, order].copy()
    for c in range(r):
        i = int(np.argmax(np.abs(P[:, c])))
        if P[i, c] < 0:
            P[:, c] = -P[:, c]
    return P, w[order]


def jssa_basis(q_bits: np.ndarray, k_bits: np.ndarray, r: int):
    """The basis of one KV head: spectral_basis(calibration_moment(q, k), r)."""
    return spectral_basis(calibration_moment(q_bits, k_bits), r)


# ============================================================================================
# Full-KV attention and gather-then-attend  [JSSA, Figure 2 (b); Figure 6 (a)]
# The pages compare the sparse attention stage with attention over the whole cache
# (full-KV) and with a variant that first copies the selected tokens into a contiguous
# buffer and then runs dense attention over it (gather-then-attend).
# ============================================================================================


def dense_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, L: int,
                    scale: float) -> np.ndarray:
    """Full-KV attention: o_h = sum_{t < L} softmax_t(scale * q_h . k_t) v_t (float64).

    q: [G][d]; K/V: [>= L][d] decoded. L = 0 gives zeros (no token to attend to).
    """
    if L == 0:
        return np.zeros((q.shape[0], V.shape[1]))
    logits = scale * (q @ K[:L].T)
    w = np.exp(logits - logits.max(axis=1, keepdims=True))
    return (w @ V[:L]) / w.sum(axis=1, keepdims=True)


def gather_blocks(sel: np.ndarray, S: int, L: int):
    """Gathered layout of one row: the source token of every gathered slot, and the count.

    Gathered slot i * S + u holds token sel[i] * S + u (u < S), for the selected blocks in
    their ascending order; a slot whose token is at or past L holds nothing (-1). Only the
    row's last block can be cut by L and it is the last selected block when selected, so
    the filled slots form a prefix. Returns (src [len(sel) * S] int64, n_valid).
    """
    sel = np.asarray(sel, dtype=np.int64)
    src = np.full(len(sel) * S, -1, dtype=np.int64)
    for i, blk in enumerate(sel):
        for u in range(S):
            t = blk * S + u
            if t < L:
                src[i * S + u] = t
    n_valid = int((src >= 0).sum())
    return src, n_valid


# ============================================================================================
# NVFP4 path  [JQS, Full text]
# ============================================================================================

E2M1_MAX = 6.0
UE4M3_MAX = 448.0


def nvfp4_pack(x32: np.ndarray, g: np.float32):
    """Pack float32 values [n][d] into NVFP4: E2M1 codes [n][d] and UE4M3 scales [n][d/16].

    Per group of 16 consecutive elements:
      a = max |x|; sf = fp32(a / fp32(6 g)); sigma = UE4M3(sf) (nearest even, satfinite);
      if sigma decodes to 0 every code is 0; else e_i = E2M1(fp32(x_i / fp32(sigma g)))
      (nearest even, satfinite). All divisions and products are rounded float32 ops.
    """
    x32 = np.asarray(x32, dtype=np.float32)
    n, d = x32.shape
    g = np.float32(g)
    grp = x32.reshape(n, d // 16, 16)
    a = np.abs(grp).max(axis=2)                                   # exact
    den = np.float32(np.float32(E2M1_MAX) * g)
    sf = (a / den).astype(np.float32)
    sig = F.ue4m3_encode(sf)
    sigv = F.ue4m3_value(sig).astype(np.float32)                  # exact in float32
    den2 = (sigv * g).astype(np.float32)
    safe = np.where(sigv > 0, den2, np.float32(1.0))
    t = (grp / safe[:, :, None]).astype(np.float32)
    codes = F.e2m1_encode(t)
    codes = np.where((sigv > 0)[:, :, None], codes, 0).astype(np.uint8)
    return codes.reshape(n, d), sig.astype(np.uint8)


def nvfp4_dequant(codes: np.ndarray, scales: np.ndarray, g) -> np.ndarray:
    """float64 values e * sigma * g for codes [n][d], scales [n][d/16]."""
    n, d = codes.shape
    e = F.e2m1_value(codes).reshape(n, d // 16, 16)
    s = F.ue4m3_value(scales)[:, :, None]
    return (e * s * np.float64(np.float32(g))).reshape(n, d)


def centre(k_bits: np.ndarray, mu: np.ndarray) -> np.ndarray:
    """x = fp32(k) - mu, a rounded float32 subtraction."""
    return (F.bf16_to_f64(k_bits).astype(np.float32) - np.asarray(mu, dtype=np.float32)
            ).astype(np.float32)


def query_scale(q_bits_all: np.ndarray) -> np.float32:
    """Per-step query tensor scale g_q = fp32(max |q| / fp32(6 * 448)) over the whole q."""
    a = np.float32(np.abs(F.bf16_to_f64(q_bits_all)).max())
    return np.float32(a / np.float32(E2M1_MAX * UE4M3_MAX))


def nvfp4_head_scores(q_codes, q_scales, g_q, k_codes, k_scales, g_k) -> np.ndarray:
    """s[h, t] = sum over d of dequant(q_h) * dequant(k_t), float64. -> [G][L]."""
    qd = nvfp4_dequant(q_codes, q_scales, g_q)
    kd = nvfp4_dequant(k_codes, k_scales, g_k)
    return qd @ kd.T


def nvfp4_block_scores(head_scores: np.ndarray, S: int) -> np.ndarray:
    """beta_j = max over the group's heads and the block's valid tokens."""
    return block_max(head_scores.max(axis=0), S)


def block_quant_error(x32: np.ndarray, codes: np.ndarray, scales: np.ndarray, g_k, S: int,
                      L: int) -> np.ndarray:
    """Squared NVFP4 error of each complete block: sum over tokens and dims of (x - deq x)^2.

    Only complete blocks ((j + 1) * S <= L) have an error; incomplete ones get -inf.
    """
    err_tok = ((x32.astype(np.float64) - nvfp4_dequant(codes, scales, g_k)) ** 2).sum(axis=1)
    nb = (L + S - 1) // S
    out = np.full(nb, -np.inf)
    nfull = L // S
    out[:nfull] = err_tok[: nfull * S].reshape(nfull, S).sum(axis=1)
    return out


def kept_blocks(err: np.ndarray, n_keep: int) -> np.ndarray:
    """The n_keep complete blocks with the largest quantisation error (ties: lower index)."""
    valid = np.nonzero(np.isfinite(err))[0]
    order = np.lexsort((valid, -err[valid]))
    return np.sort(valid[order[:n_keep]])


# ============================================================================================
# Binary proxy with an adaptive top-p budget  [RQC, Abstract; RBQ]
# The page scores every cached key with a 1-bit code of its randomly rotated direction and
# an INT4 code of the rotated query, and lets the attended set grow until the estimated
# attention mass reaches p. The estimator is the published RaBitQ one [RBQ]:
#   o = k - c (the row's centre c), y = o R (R a random d x d rotation, its columns the
#   rotated axes), code bits b_i = [y_i > 0], x_i = (2 b_i - 1) / sqrt(d);
#   <o, q> ~= |o| <x, q R> / <x, y / |o|> = (|o|^2 / |y|_1) sum_i (2 b_i - 1) (q R)_i.
# Over a uniformly random rotation the ratio is an unbiased estimate of <o, q>, and
# rounding each rotated query entry to the 4-bit grid at random (floor(t + u), u uniform)
# keeps it unbiased. Readings (the pages give no more than the abstract):
#   * the query is the mean of the group's query heads, the centre one vector per row;
#   * the estimated score of token t is g_t sum_i (2 b_i - 1)(Delta n_i + v_l) + <c, qbar>;
#   * the estimated attention weights are softmax(scale * score) over the row's valid
#     tokens; a block's mass is the sum of its tokens' weights (S = 1: token level);
#   * forced blocks are taken first and count toward the mass; the rest follow in order of
#     decreasing mass (ties: lower index) until the taken mass reaches p, or the budget
#     (the largest number of blocks a row may attend) is full.
# The stored code bits, g_t and the query's codes are decided in float32 in a fixed order
# (as the CUDA writer and scan compute them), so they compare bit for bit; scores, weights
# and masses are float64.
# ============================================================================================

RQ_QUERY_BITS = 4
RQ_QUERY_LEVELS = (1 << RQ_QUERY_BITS) - 1           # codes 0 .. 15


def _rotate_f32(x32: np.ndarray, R: np.ndarray) -> np.ndarray:
    """y = x R in float32: y_i = sum over j ascending of fp32(x_j * R_ji), each product and
    each partial sum rounded (no fused multiply-add). x32: [n][d]; R: float32 [d][d]."""
    x32 = np.asarray(x32, dtype=np.float32)
    R32 = np.asarray(R, dtype=np.float32)
    acc = np.zeros((x32.shape[0], R32.shape[1]), dtype=np.float32)
    for j in range(x32.shape[1]):
        acc = acc + x32[:, j:j + 1] * R32[j:j + 1, :]
    return acc


def _f32_sum_seq(x32: np.ndarray) -> np.ndarray:
    """Row sums of a float32 [n][m] array, added left to right with a rounding per step."""
    acc = np.zeros(x32.shape[0], dtype=np.float32)
    for j in range(x32.shape[1]):
        acc = acc + x32[:, j]
    return acc


def rabitq_encode(k_bits: np.ndarray, R: np.ndarray, c: np.ndarray):
    """Binary codes of keys [n][d] (BF16): bits [n][d] (0/1, uint8) and g [n] (float32).

    o = fp32(k) - c (rounded float32); y = o R (_rotate_f32); b_i = [y_i > 0];
    g = fp32(fp32 sum_j o_j^2 / fp32 sum_i |y_i|) with both sums taken left to right in
    float32, and g = 0 where sum |y_i| = 0 (a key equal to the centre).
    """
    o = centre(k_bits, c)
    y = _rotate_f32(o, R)
    bits = (y > 0).astype(np.uint8)
    n2 = _f32_sum_seq((o * o).astype(np.float32))
    l1 = _f32_sum_seq(np.abs(y))
    safe = np.where(l1 > 0, l1, np.float32(1.0))
    g = np.where(l1 > 0, (n2 / safe).astype(np.float32), np.float32(0.0)).astype(np.float32)
    return bits, g


def rabitq_pack_bits(bits: np.ndarray) -> np.ndarray:
    """Stored code: bit i of a key in byte i // 8, at bit position i % 8 -> [n][d / 8] uint8."""
    return np.packbits(np.asarray(bits, dtype=np.uint8), axis=-1, bitorder="little")


def rabitq_unpack_bits(packed: np.ndarray, d: int) -> np.ndarray:
    return np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=-1, count=d,
                         bitorder="little")


def rabitq_query(q_bits: np.ndarray, R: np.ndarray, u: np.ndarray):
    """The rotated group-mean query and its 4-bit code, all in float32.

    qbar_j = fp32(sum over heads in order of fp32(q_h,j)) / G (a rounded division);
    q' = qbar R (_rotate_f32); v_l = min q', v_r = max q';
    Delta = fp32(fp32(v_r - v_l) / 15); n_i = min(15, floor(fp32(fp32(fp32(q'_i - v_l) /
    Delta) + u_i))), with n = 0 everywhere when Delta = 0. u [d]: uniform draws in [0, 1).
    Returns (n [d] int64, Delta, v_l, qbar [d] float32).
    """
    q32 = F.bf16_to_f64(q_bits).astype(np.float32)
    acc = np.zeros(q32.shape[1], dtype=np.float32)
    for h in range(q32.shape[0]):
        acc = acc + q32[h]
    qbar = (acc / np.float32(q32.shape[0])).astype(np.float32)
    qr = _rotate_f32(qbar[None, :], R)[0]
    vl, vr = np.float32(qr.min()), np.float32(qr.max())
    delta = np.float32(np.float32(vr - vl) / np.float32(RQ_QUERY_LEVELS))
    if delta == 0:
        return np.zeros(qr.shape[0], dtype=np.int64), delta, vl, qbar
    t = ((qr - vl).astype(np.float32) / delta).astype(np.float32)
    n = np.floor((t + np.asarray(u, dtype=np.float32)).astype(np.float32)).astype(np.int64)
    return np.minimum(n, RQ_QUERY_LEVELS), delta, vl, qbar


def rabitq_scores(bits: np.ndarray, g: np.ndarray, n: np.ndarray, delta, vl, c: np.ndarray,
                  qbar: np.ndarray) -> np.ndarray:
    """Estimated scores [n_keys] (float64): g_t sum_i (2 b_ti - 1)(Delta n_i + v_l) + <c, qbar>."""
    qhat = np.float64(delta) * np.asarray(n, dtype=np.float64) + np.float64(vl)
    sgn = 2.0 * np.asarray(bits, dtype=np.float64) - 1.0
    shift = float(np.asarray(c, dtype=np.float64) @ np.asarray(qbar, dtype=np.float64))
    return np.asarray(g, dtype=np.float64) * (sgn @ qhat) + shift


def estimated_weights(s: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * s) over the given (valid) tokens, float64."""
    x = scale * np.asarray(s, dtype=np.float64)
    e = np.exp(x - x.max())
    return e / e.sum()


def block_mass(w: np.ndarray, S: int) -> np.ndarray:
    """Sum of the weights of each block's valid tokens -> [ceil(L / S)]."""
    L = w.shape[0]
    nb = (L + S - 1) // S
    pad = np.zeros(nb * S - L)
    return np.concatenate([w, pad]).reshape(nb, S).sum(axis=1)


def select_top_p(mass: np.ndarray, p: float, budget: int, forced: np.ndarray) -> np.ndarray:
    """Indices (ascending) of the forced blocks plus the fewest highest-mass others whose
    total mass, with the forced blocks', reaches p of the row's mass; at most ``budget``.

    Requires 0 < p <= 1 and |forced| <= budget. Blocks are added in order of decreasing
    mass, ties to the lower index; the running mass is summed in the order taken (forced
    blocks first, ascending) and compared with p * (sum of all masses).
    """
    if not (0.0 < p <= 1.0):
        raise ValueError("p must be in (0, 1]")
    forced = np.unique(np.asarray(forced, dtype=np.int64))
    if len(forced) > budget:
        raise ValueError("more forced blocks than the budget")
    nb = mass.shape[0]
    goal = p * float(mass.sum())
    taken = [int(j) for j in forced]
    acc = 0.0
    for j in taken:
        acc += float(mass[j])
    is_forced = np.zeros(nb, dtype=bool)
    is_forced[forced] = True
    rest = np.nonzero(~is_forced)[0]
    for j in rest[np.lexsort((rest, -mass[rest]))]:
        if len(taken) >= budget or acc >= goal:
            break
        taken.append(int(j))
        acc += float(mass[j])
    return np.sort(np.array(taken, dtype=np.int64))


def top_p_valid(mass: np.ndarray, p: float, budget: int, forced: np.ndarray, got: np.ndarray,
                rel_tol: float = 1e-4) -> tuple[bool, str]:
    """Is ``got`` a valid top-p selection, up to rounding of the masses and the goal?

    Valid iff it is strictly ascending, in range, holds every forced block and at most
    ``budget`` blocks; its non-forced blocks are the highest-mass ones up to near-ties
    (relative band rel_tol at the last one taken); and its size is right: either the goal
    p * total is reached (within rel_tol of the total) and dropping the lightest non-forced
    block would miss it, or the budget is full without reaching it.
    """
    got = np.asarray(got, dtype=np.int64)
    nb = mass.shape[0]
    forced = np.unique(np.asarray(forced, dtype=np.int64))
    if np.any(np.diff(got) <= 0):
        return False, "not strictly ascending"
    if got.size and (got[0] < 0 or got[-1] >= nb):
        return False, "index out of range"
    if not set(forced.tolist()) <= set(got.tolist()):
        return False, "forced block missing"
    if len(got) > budget:
        return False, f"{len(got)} blocks over the budget {budget}"
    total = float(mass.sum())
    tol = rel_tol * total
    goal = p * total
    extra = np.setdiff1d(got, forced)
    others = np.setdiff1d(np.arange(nb), got)
    if extra.size and others.size:
        lightest = float(mass[extra].min())
        band = rel_tol * max(abs(lightest), 1e-300)
        if float(mass[others].max()) > lightest + band:
            return False, "an unchosen block outweighs a chosen one"
    have = float(mass[got].sum())
    if have >= goal - tol:
        if extra.size and have - float(mass[extra].min()) >= goal + tol:
            return False, "not minimal: the goal is met without the lightest block"
        return True, "goal reached"
    if len(got) == budget or others.size == 0:
        return True, "budget full"
    return False, f"mass {have} short of the goal {goal}"


# ============================================================================================
# Semantic blocks: clustered, non-contiguous key blocks  [CSB, Abstract]
# The page builds a key index for the prompt: its keys are clustered into large blocks of
# tokens from anywhere in the prompt; a query scores each block by its centroid and attends
# to the original keys and values of the blocks it selects. The abstract gives no
# clustering algorithm. Readings:
#   * clustering = Lloyd's k-means in Euclidean distance on the stored keys (float64), with
#     C = ceil(L0 / S) clusters for a prompt of L0 tokens and a target block size S, seeded
#     with the keys at the evenly spaced positions floor(i * L0 / C), for a fixed number of
#     iterations; a token joins its nearest centroid (ties: the lower cluster index); an
#     empty cluster keeps its centroid;
#   * block score = qbar . centroid, the centroid being the mean of the member keys (so the
#     score is the mean of the members' exact group-mean scores);
#   * the budget counts clusters; ties go to the lower cluster index;
#   * tokens after the prompt (decoded after the index was built) are always attended.
# The clustering definition is parity unpinned (a reading); its implementation is pinned by
# the properties of Lloyd's algorithm.
# ============================================================================================


def kmeans_keys(k_bits: np.ndarray, C: int, iters: int):
    """Cluster keys [L0][d] (BF16) into C groups: (assign [L0] int64, centroids [C][d]).

    Centroids start at the keys at positions floor(i * L0 / C); each iteration assigns every
    key to its nearest centroid (squared Euclidean distance, ties to the lower index), then
    moves every non-empty cluster's centroid to the mean of its members.
    """
    x = F.bf16_to_f64(k_bits)
    L0 = x.shape[0]
    if not (1 <= C <= L0):
        raise ValueError("need 1 <= C <= L0")
    cent = x[(np.arange(C) * L0) // C].copy()
    assign = np.zeros(L0, dtype=np.int64)
    for _ in range(max(iters, 1)):
        d2 = ((x[:, None, :] - cent[None, :, :]) ** 2).sum(axis=2)          # [L0][C]
        assign = np.argmin(d2, axis=1)                                       # first minimum
        for j in range(C):
            members = x[assign == j]
            if len(members):
                cent[j] = members.mean(axis=0)
    return assign, cent


def kmeans_objective(k_bits: np.ndarray, assign: np.ndarray, cent: np.ndarray) -> float:
    """Sum over keys of the squared distance to the assigned centroid."""
    x = F.bf16_to_f64(k_bits)
    return float(((x - cent[assign]) ** 2).sum())


def semantic_block_scores(q_bits: np.ndarray, cent: np.ndarray) -> np.ndarray:
    """beta_j = qbar . centroid_j (float64); q_bits: the group's BF16 queries [G][d]."""
    return cent @ F.bf16_to_f64(q_bits).mean(axis=0)


def semantic_tokens(assign: np.ndarray, sel: np.ndarray, L0: int, L: int) -> np.ndarray:
    """The attended positions, ascending: the members of the selected clusters, then every
    token after the prompt (L0 <= t < L)."""
    members = np.nonzero(np.isin(assign, np.asarray(sel, dtype=np.int64)))[0]
    return np.concatenate([members, np.arange(L0, L)]).astype(np.int64)


def kmeans_keys_f32(k_bits: np.ndarray, C: int, iters: int):
    """kmeans_keys with every decision taken in float32 in a fixed order, as a kernel takes
    it: (assign [L0] int64, centroids [C][d] float32).

    x = fp32(k). Seeds: the keys at floor(i * L0 / C). Per iteration:
      * distance d_tj = sum over i ascending of fp32((x_ti - c_ji)^2), each difference,
        square and partial sum rounded to float32; a key joins the smallest d_tj (ties:
        the lower cluster index);
      * a non-empty cluster's centroid becomes fp32(fp32 sum of its members in token order,
        dimension by dimension, one rounding per add) / fp32(count); an empty one keeps
        its centroid.
    """
    x = F.bf16_to_f64(k_bits).astype(np.float32)
    L0, d = x.shape
    if not (1 <= C <= L0):
        raise ValueError("need 1 <= C <= L0")
    cent = x[(np.arange(C) * L0) // C].copy()
    assign = np.zeros(L0, dtype=np.int64)
    for _ in range(max(iters, 1)):
        acc = np.zeros((L0, C), dtype=np.float32)
        for i in range(d):
            diff = (x[:, i:i + 1] - cent[None, :, i]).astype(np.float32)
            acc = (acc + (diff * diff).astype(np.float32)).astype(np.float32)
        assign = np.argmin(acc, axis=1)                                      # first minimum
        for j in range(C):
            members = np.nonzero(assign == j)[0]
            if len(members) == 0:
                continue
            s = np.zeros(d, dtype=np.float32)
            for t in members:                                                # token order
                s = (s + x[t]).astype(np.float32)
            cent[j] = (s / np.float32(len(members))).astype(np.float32)
    return assign, cent
