/*
 * qs.h - C ABI of libqs: score-then-select sparse attention for one decode step (sm_100a).
 *
 * The decode step, per row = (sequence b, KV head g):
 *   1. score  - a cheap proxy score of the current query against the row's whole key
 *               history, reduced to one score per block of S tokens (max over the block;
 *               with the binary proxy, the log of the block's estimated attention mass;
 *               with semantic blocks, one score per cluster of the prompt's keys);
 *   2. select - the top-k blocks per row (forced blocks first), ties to the lower index;
 *               with the binary proxy, the fewest blocks whose estimated mass reaches p;
 *   3. attend - exact softmax attention of each of the group's query heads over the
 *               selected original keys and values only, FP32 accumulation, split over the
 *               selection and finished by a log-sum-exp combine.
 *
 * Sources:
 *   "Joint Subspace Sparse Attention for Efficient Long-Context Decoding"
 *     Figure 1: the mean of a KV head's query heads scores a projected-key cache in a
 *     shared low-dimensional subspace; the top-B positions are shared by the group's query
 *     heads; gather-free indexed attention reads the original keys/values at them.
 *     Abstract: distinct per-KV-head selections under the standard GQA cache layout.
 *     Figure 9: the step's stages are scoring preparation, candidate scoring, top-B
 *     selection and sparse attention.
 *     Figure 10: the projected scoring cache may be kept at reduced precision while the
 *     full KV cache and the final attention stay BF16.
 *   "Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention"
 *     Full text: NVFP4 scoring keys scanned densely on FP4 tensor cores; 128-token blocks;
 *     FP16 value aggregation with FP32 accumulation; calibrated key centring; at most two
 *     blocks kept at BF16 per sequence; the cache is packed directly from BF16 activations.
 *   "Coarse Semantic Blocks for Efficient Training-Free Sparse Attention" (Abstract): a
 *     prompt-specific key index: the prompt's keys clustered into large blocks of
 *     non-contiguous tokens, scored by their centroids; the selected blocks' original keys
 *     and values are attended.
 *   "RaBitQCache" (Abstract): keys scored through randomly rotated binary codes with
 *     binary-INT4 arithmetic (an unbiased estimate of q . k) and a top-p budget that grows
 *     the attended set until the estimated attention mass reaches p. The estimator is the
 *     published RaBitQ one: J. Gao and C. Long, "RaBitQ: Quantizing High-Dimensional
 *     Vectors with a Theoretical Error Bound for Approximate Nearest Neighbor Search",
 *     SIGMOD 2024, section 3.
 *
 * Conventions (all entry points):
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise; the caller owns
 *     every buffer (caches, inputs, outputs and the workspace). The library allocates no
 *     device memory and keeps no pointer after the call returns.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream) and never
 *     synchronise, except qs_device_status.
 *   - Arguments are validated on the host before any launch. On failure the call returns
 *     QS_ERR_INVALID_ARG (bad pointer/size) or QS_ERR_UNSUPPORTED (a shape the library does
 *     not implement) and launches nothing. There is no fallback path.
 *   - Cache tensors (K, V, proxy) and q must be 16-byte aligned (q may be 4-byte aligned
 *     for qs_score on the rank-r path).
 *   - Values that live on the device (sequence lengths, page-table entries, n_new, the
 *     selection) are checked by the kernels: an out-of-range value skips the access and
 *     records QS_ERR_DEVICE_BOUNDS in the workspace status word, which qs_device_status
 *     reads. Waits inside kernels are bounded; running out records QS_ERR_DEVICE_TIMEOUT.
 *   - A launch error is returned as QS_ERR_CUDA (the CUDA error is left for
 *     cudaGetLastError by the caller).
 *   - Entry points are re-entrant; two calls that share a workspace must not overlap on
 *     the GPU. The library keeps only process-wide caches, each guarded by a mutex or
 *     atomic: encoded TMA tensor maps (keyed by tensor address and shape, 16 entries),
 *     the kernels' shared-memory limits (set once per kernel and device) and the SM
 *     count of each device. One process may drive several GPUs (the current device at
 *     the call is used).
 *
 * Memory layouts (row-major, innermost last):
 *   K, V pages      [num_pages][Hkv][page_size][head_dim]   BF16 (V may be FP16)
 *   proxy (rank r)  [num_pages][Hkv][page_size][r]          F32, BF16 or E4M3 (FP8: sign,
 *                                                           4 exponent bits with bias 7,
 *                                                           3 mantissa bits; largest 448;
 *                                                           one byte per entry)
 *   proxy (NVFP4)   [num_pages][Hkv] x 8192 bytes (head_dim 128, page_size 128) of E2M1
 *                   codes, chunk-major: element e (0..127) of token slot m (0..127) is in
 *                   byte (e / 32) * 2048 + m * 16 + (e % 32) / 2, in the low nibble when e
 *                   is even and the high nibble when it is odd. Each 32-element chunk of a
 *                   token is one 16-byte row, so a contiguous copy of the page lands as the
 *                   K-major operand of the FP4 tensor-core MMA (8-token x 16-byte core
 *                   matrices, chunks 2048 bytes apart).
 *   proxy_scale     [num_pages][Hkv] x 1024 bytes of UE4M3 scales: the scale of elements
 *                   16j .. 16j+15 (j = 0..7) of token slot m is byte
 *                   (j / 4) * 512 + 16 * (m % 32) + 4 * (m / 32) + j % 4, the order in
 *                   which the tensor cores' scale-factor copy (tcgen05.cp 32x128b.warpx4)
 *                   expects a 128-token tile's scales.
 *   proxy (centroid)[num_pages][Hkv][page_size/S][head_dim] F32: the sum of the keys of each
 *                                                           S-token block of the page
 *   proxy (binary)  [num_pages][Hkv] x (page_size * head_dim/8 bytes of code bits, then
 *                                       page_size F32 factors g): token slot s has bits
 *                                       at byte s * head_dim/8 (bit i of the key in byte
 *                                       i / 8, position i % 8) and g at index s
 *   page_table      [batch][max_pages_per_seq]              int32 physical page ids
 *   seq_lens        [batch]                                 int32 tokens in the cache
 *   P               [Hkv][head_dim][r]                      F32
 *   R (binary)      [Hkv][head_dim][head_dim]               F32 rotation, y = x . R
 *   q, out          [batch][Hq][head_dim]                   q BF16; out F32 or BF16
 *   k_new, v_new    [batch][Hkv][max_new][head_dim]         K BF16, V as v_dtype
 *   block scores    [batch][Hkv][nb_stride]  F32, nb_stride = ceil(max_context / page_size)
 *                                                                 * (page_size / block_size)
 *   sel             [batch][Hkv][budget]     int32 ascending block ids, padded with -1
 *   n_sel           [batch][Hkv]             int32 = min(budget, ceil(seq_len / block_size))
 *                                            (top-p: the number of blocks taken)
 * Query head h belongs to KV head h / (Hq / Hkv).
 */
#ifndef QS_H
#define QS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *qs_stream_t; /* a cudaStream_t */

typedef enum {
  QS_OK = 0,
  QS_ERR_INVALID_ARG = 1,
  QS_ERR_UNSUPPORTED = 2,
  QS_ERR_CUDA = 3,
  QS_ERR_DEVICE_BOUNDS = 4,
  QS_ERR_DEVICE_TIMEOUT = 5
} qs_status;

typedef enum {
  QS_F32 = 0, QS_BF16 = 1, QS_F16 = 2, QS_NVFP4 = 3, QS_E4M3 = 4,
  QS_CENTROID = 5,  /* proxy_dtype only: per-block FP32 key sums (centroid scoring), r = 0 */
  QS_RABITQ = 6,    /* proxy_dtype only: binary codes of rotated centred keys, r = 0      */
  QS_SEMANTIC = 7   /* proxy_dtype only: semantic-block index outside the cache, r = 0   */
} qs_dtype;

/* Problem statement of one attention layer's decode step. */
typedef struct {
  int32_t n_q_heads;      /* Hq; Hq % Hkv == 0 and the group G = Hq / Hkv <= 8          */
  int32_t n_kv_heads;     /* Hkv                                                          */
  int32_t head_dim;       /* d: 64 or 128 (NVFP4 scoring needs 128)                       */
  int32_t page_size;      /* tokens per cache page: 128                                   */
  int32_t block_size;     /* S: a power of two dividing page_size (1 = token level)       */
  int32_t budget;         /* k: blocks selected per row, >= 1                             */
  int32_t proxy_rank;     /* r > 0: projected-key proxy; 0: NVFP4, centroid or binary     */
  int32_t proxy_dtype;    /* qs_dtype: F32, BF16 or E4M3 (rank r); NVFP4, CENTROID, RABITQ
                             or SEMANTIC (r 0)                                            */
  int32_t v_dtype;        /* qs_dtype of stored V: BF16 or F16                            */
  int32_t v_agg_dtype;    /* precision of the P.V operands: BF16 or F16 (FP32 accumulate) */
  int32_t out_dtype;      /* F32 or BF16                                                  */
  int32_t force_sink;     /* 1: block 0 is always selected                                */
  int32_t force_last;     /* 1: the block holding the newest token is always selected     */
  int32_t n_keep_hp;      /* NVFP4: 0..2 blocks with the largest quantisation error are
                             kept at full precision and always selected                  */
  float softmax_scale;    /* 0 => 1/sqrt(d)                                               */
  int32_t attn_path;      /* attention kernel: 0 chosen per shape (the tile pipeline when
                             block_size >= 8 and there are >= 40 tiles of 64 selected slots
                             per resident CTA, else the gather kernel); 1 tile pipeline
                             (needs block_size >= 8); 2 gather kernel. Same results up to
                             float32 summation order.                                    */
  int32_t key_storage;    /* the keys the attention reads ("Jet-QSparse ...", Full text: the
                             persistent cache keeps the attended keys in NVFP4, at most two
                             blocks per sequence at BF16). 0 (or QS_BF16): the BF16 key
                             pages. QS_NVFP4 (needs proxy_dtype QS_NVFP4, the tile pipeline,
                             head_dim 128): a token of one of the row's n_keep_hp kept blocks
                             is read from the BF16 key pages; every other token's key is its
                             NVFP4 scoring copy, decoded, un-centred and rounded to BF16 in
                             the kernel, bf16_rne(fp32(fp32(e * sigma) * g_k) + mu). The K
                             bytes read per token fall from 2 * head_dim to 72 (codes and
                             scales); a plain copy of the BF16 key pages is then needed only
                             for the kept blocks. Every call that attends then needs the
                             cache's proxy, proxy_scale, key_center (16-byte aligned),
                             key_gscale and, with n_keep_hp > 0, block_err
                             (QS_ERR_INVALID_ARG otherwise); qs_dense_attn always reads the
                             BF16 keys; qs_sparse_attn_noalloc returns QS_ERR_UNSUPPORTED. */
} qs_config;

/* The paged caches of one layer. All pointers are device pointers owned by the caller. */
typedef struct {
  void *k;                    /* K pages, BF16                                            */
  void *v;                    /* V pages, v_dtype                                         */
  void *proxy;                /* scoring cache (layout above)                             */
  uint8_t *proxy_scale;       /* NVFP4 only: UE4M3 scales; NULL otherwise                 */
  float *block_err;           /* NVFP4 only: [batch][Hkv][nb_stride] squared quantisation
                                 error of each complete block (written by qs_append_kv)   */
  const float *key_center;    /* NVFP4 and binary proxy: [batch][Hkv][d] centring mean    */
  const float *key_gscale;    /* NVFP4 only: 1 float, the key tensor scale g_k            */
  const int32_t *page_table;  /* [batch][max_pages_per_seq]                               */
  int32_t *seq_lens;          /* [batch]; advanced by qs_append_kv / qs_decode            */
  int32_t max_pages_per_seq;  /* row stride of page_table                                 */
  int32_t num_pages;          /* physical pages in k / v / proxy                          */
  int32_t max_context;        /* upper bound of every seq_len; sizes nb_stride           */
} qs_cache;

/* Bytes of workspace that the calls below need for `batch` sequences (host only, no
   device access). QS_ERR_INVALID_ARG / QS_ERR_UNSUPPORTED as for the other calls. */
qs_status qs_workspace_size(const qs_config *cfg, int32_t batch, int32_t max_context,
                            size_t *bytes /* host */);

/* Number of kernel launches qs_sparse_attn makes for this shape: 1 for the gather kernel
   (its log-sum-exp merge is in-kernel), 2 for the tile pipeline (then the row merge), 3 with
   key_storage QS_NVFP4 (the rows' kept blocks first). Host only. */
qs_status qs_attention_launches(const qs_config *cfg, int32_t batch, int32_t max_context,
                                int32_t *launches /* host */);

/* Zero the whole workspace (status word and counters; async on stream). Call once after
   allocating a workspace, before any other call uses it. */
qs_status qs_workspace_init(void *ws, size_t ws_bytes, qs_stream_t stream);

/* Append n_new[b] tokens to every KV head of sequence b, then advance seq_lens[b].
   Writes K/V into page slot seq_lens[b] + i and the row's scoring cache:
     rank r: proxy = k.P[g] in float32 (ascending index, one rounding per product and per
             sum), stored F32, rounded to nearest-even BF16, or rounded to nearest-even E4M3
             saturating at +-448 (the FP8 scoring cache of "Joint Subspace Sparse Attention
             ...", Figure 10);
     centroid: the block's FP32 key sum, continued in token order (one rounding per add;
             restarted at the block's first token): "Coarse Semantic Blocks ...", Abstract,
             scores blocks by their centroids;
     NVFP4:  x = float(k) - key_center[b][g] (float32), packed per 16 elements to UE4M3
             scale + E2M1 codes with the tensor scale g_k; each block of S tokens that this
             call completes gets block_err = sum of squared (x - dequant(x)).
     binary: o = float(k) - key_center[b][g] (float32), y = o . R[g] (R passed as P; y_i
             summed over j ascending, one rounding per product and per sum), code bits
             b_i = [y_i > 0] and g = fp32(sum_j o_j^2) / fp32(sum_i |y_i|) (both sums left to
             right; 0 when the second is 0): the RaBitQ code ("RaBitQCache", Abstract).
   k_new/v_new: [batch][Hkv][max_new][d]; n_new: device int32 [batch], each <= max_new;
   P: [Hkv][d][r] (NULL for NVFP4 and centroid; R [Hkv][d][d] for the binary proxy).
   Pages for the new tokens must be in page_table. */
qs_status qs_append_kv(const qs_config *cfg, const qs_cache *cache, const void *k_new,
                       const void *v_new, const int32_t *n_new, int32_t max_new,
                       const float *P, int32_t batch, void *ws, qs_stream_t stream);

/* Proxy block scores of every row (stage 1).
   rank r: qbar = mean of the group's query heads (float32), q~ = qbar.P[g] (float32),
           s_t = q~ . proxy_t (float32 accumulation), beta_j = max of s over the block's
           valid tokens (t < seq_len).
   centroid: qbar = mean of the group's query heads (float32); beta_j = qbar . sum_j /
           count_j (float32), count_j = valid tokens of block j (the mean of the block's
           exact group-mean scores);
   NVFP4:  the whole q tensor is packed with g_q = max|q| / 2688; per head h,
           s_{h,t} = g_q g_k sum_c sq_{h,c} sk_{t,c} sum_i eq_{h,16c+i} ek_{t,16c+i} on the
           block-scaled FP4 tensor cores; beta_j = max over the group's heads and the
           block's valid tokens.
   Blocks past ceil(seq_len / S) that share a page with valid tokens are written -inf;
   entries past the last page of a row are not written.
   q: [batch][Hq][d] BF16; P as in qs_append_kv; block_scores: [batch][Hkv][nb_stride].
   The binary proxy needs its rounding draws: qs_rabitq_score (QS_ERR_UNSUPPORTED here). */
qs_status qs_score(const qs_config *cfg, const qs_cache *cache, const void *q,
                   const float *P, int32_t batch, float *block_scores, void *ws,
                   qs_stream_t stream);

/* Top-k block selection of every row (stage 2).
   nb = ceil(seq_len / S). If nb <= budget every block is selected. Otherwise the forced
   set F (block 0 if force_sink, block nb-1 if force_last, and on the NVFP4 path the
   n_keep_hp complete blocks with the largest block_err, ties to the lower index) is taken
   first; the remaining budget - |F| blocks are the best-scoring others, ties to the lower
   index. A NaN or -inf score ranks as -FLT_MAX and +inf as FLT_MAX (ties between them and
   those values go to the lower index). Output ascending, padded with -1. */
qs_status qs_select_topk(const qs_config *cfg, const qs_cache *cache,
                         const float *block_scores, int32_t batch, int32_t *sel,
                         int32_t *n_sel, void *ws, qs_stream_t stream);

/* The same selection as qs_select_topk (same arguments, rules and output), computed by
   three counting passes over the order-preserving keys of the scores (their top 11, next
   11 and last 10 bits) instead of pairwise ranking: one CTA of 1,024 threads per row, a
   few streaming passes over the row's scores. For rows of many candidates (token-level
   selection at long context). One launch. */
qs_status qs_select_topk_radix(const qs_config *cfg, const qs_cache *cache,
                               const float *block_scores, int32_t batch, int32_t *sel,
                               int32_t *n_sel, void *ws, qs_stream_t stream);

/* Exact softmax attention over the selected blocks' valid tokens (stage 3).
   For every query head h of row (b, g): o_h = sum_t softmax_t(scale * q_h.k_t) v_t over
   t in the selected blocks (t < seq_len), normalised over those tokens only. Logits are
   float32 sums of BF16 products; P.V operands are v_agg_dtype, accumulated in float32.
   The selection is split across CTAs; partial (max, sum, o) states are merged by a
   log-sum-exp combine. out: [batch][Hq][d] in out_dtype. q is 16-byte aligned. */
qs_status qs_sparse_attn(const qs_config *cfg, const qs_cache *cache, const void *q,
                         const int32_t *sel, const int32_t *n_sel, int32_t batch, void *out,
                         void *ws, qs_stream_t stream);

/* One decode step: append one token per sequence (k_new/v_new: [batch][Hkv][d]), then
   score, select and attend over seq_len + 1 tokens. sel_out / n_sel_out may be NULL; the
   selection then stays in the workspace. The binary proxy with its top-p budget has its
   own step call, qs_decode_top_p; this call returns QS_ERR_UNSUPPORTED for it. */
qs_status qs_decode(const qs_config *cfg, const qs_cache *cache, const void *q,
                    const void *k_new, const void *v_new, const float *P, int32_t batch,
                    void *out, int32_t *sel_out, int32_t *n_sel_out, void *ws,
                    qs_stream_t stream);

/* ---- Binary proxy with a top-p budget ("RaBitQCache", Abstract) -------------------------
   Per row (b, g), with the rotation R[g] and the draws u[b][g] (uniform in [0, 1)):
     qbar_i = fp32(sum over the group's heads, in order) / G;  q' = qbar . R[g] (j
       ascending, one rounding per product and per sum); v_l = min q', Delta =
       fp32(max q' - v_l) / 15; code n_i = min(15, floor(fp32(fp32((q'_i - v_l) / Delta) +
       u_i))), all 0 when Delta = 0 (every step a rounded float32 operation);
     s_t = g_t sum_i (2 b_ti - 1)(Delta n_i + v_l) + key_center[b][g] . qbar, computed as
       g_t (Delta (2A - Q) + v_l (2B - d)) + c . qbar with A = sum_p 2^p popc(b & plane_p),
       B = popc(b), Q = sum n_i (the RaBitQ estimate of qbar . k_t);
     block_scores[b][g][j] = log sum_{t in block j, t < seq_len} e^(scale * s_t), the
       natural log of the block's estimated attention mass up to the row's normaliser
       (-inf for blocks with no valid token that share a page with valid ones; entries past
       the last page of a row are not written).
   q: [batch][Hq][d] BF16 (4-byte aligned); R: [Hkv][d][d] (16-byte aligned); u: [batch]
   [Hkv][d] F32. Two launches (query codes into the workspace, then the scan). cfg must
   have proxy_dtype QS_RABITQ (else QS_ERR_UNSUPPORTED) and cache->key_center set. */
qs_status qs_rabitq_score(const qs_config *cfg, const qs_cache *cache, const void *q,
                          const float *R, const float *u, int32_t batch, float *block_scores,
                          void *ws, qs_stream_t stream);

/* Top-p block selection of every row (one launch). block_scores hold natural-log block
   masses (as qs_rabitq_score writes them); with M = the row's largest, block j weighs
   w_j = e^(score_j - M), held in fixed point (units of 2^-40, so sums are exact). Over the
   nb = ceil(seq_len / S) blocks, Z = sum w, goal = min(Z, ceil(p Z)). The forced blocks
   (block 0 if force_sink, block nb-1 if force_last) are taken first and their mass
   counts; the others follow in order of decreasing score, ties to the lower index, until
   the taken mass reaches the goal or budget blocks are taken. A NaN score counts as -inf
   (mass 0) and +inf as FLT_MAX. sel: ascending block ids padded with -1; n_sel: the count.
   0 < p <= 1 and budget >= force_sink + force_last, else QS_ERR_INVALID_ARG. Any proxy
   kind's configuration is accepted; only its block size, budget and forced blocks are
   used. */
qs_status qs_select_top_p(const qs_config *cfg, const qs_cache *cache,
                          const float *block_scores, float p, int32_t batch, int32_t *sel,
                          int32_t *n_sel, void *ws, qs_stream_t stream);

/* One decode step with the binary proxy, as qs_decode is for the others: append one token
   per sequence (k_new / v_new: [batch][Hkv][d]; the binary writer with R), then
   qs_rabitq_score, qs_select_top_p with p, and qs_sparse_attn over seq_len + 1 tokens, in
   stream order (5 launches, plus the row merge when the tile pipeline runs). The block
   scores live in the workspace; sel_out / n_sel_out may both be NULL, the selection then
   stays in the workspace too. Arguments and statuses as in the four calls. */
qs_status qs_decode_top_p(const qs_config *cfg, const qs_cache *cache, const void *q,
                          const void *k_new, const void *v_new, const float *R,
                          const float *u, float p, int32_t batch, void *out,
                          int32_t *sel_out, int32_t *n_sel_out, void *ws,
                          qs_stream_t stream);

/* ---- Semantic blocks ("Coarse Semantic Blocks ...", Abstract) ---------------------------
   The index covers each sequence's prompt (L0 = prompt_lens[b] tokens already in the
   cache); it is built once, and every decode step scores it. With cfg->proxy_dtype =
   QS_SEMANTIC (rank 0), cfg->block_size S is the target cluster size and cfg->budget the
   number of clusters selected. C_b = ceil(L0_b / S) clusters; C_max = ceil(max_context / S).
   Index of row (b, g) = b * Hkv + g:
     centroids [rows][C_max][head_dim] F32;
     offsets   [rows][C_max + 1] int32: cluster j's members are members[offsets[j] ..
               offsets[j + 1]) of the row;
     members   [rows][max_context] int32 token positions, grouped by cluster, ascending
               within a cluster.
   The clustering is Lloyd's k-means with every decision in float32 in a fixed order:
     seeds c_j = fp32(key at floor(j * L0 / C)); then, `iters` times,
     assign: d_tj = sum over i ascending of fp32((x_ti - c_ji)^2) (one rounding per
             difference, square and add); key t joins the smallest d_tj, ties to the lower j;
     update: c_j = fp32(sum of the members' keys in token order) / fp32(count); an empty
             cluster keeps its centroid.
   Tokens appended after the index was built are not in it: qs_append_kv with this
   proxy_dtype writes their K/V only, and qs_semantic_select always adds them. */

/* Workspace bytes for qs_semantic_index (host only): 256 + 4 * rows * (max_context +
   C_max). QS_ERR_UNSUPPORTED unless proxy_dtype is QS_SEMANTIC. */
qs_status qs_semantic_index_workspace_size(const qs_config *cfg, int32_t batch,
                                           int32_t max_context, size_t *bytes /* host */);

/* Build the index of every row from the cached keys (K pages only; the cache's proxy
   fields are not read). prompt_lens: device int32 [batch], each <= cache->max_context
   (larger values are clamped). iters >= 1. Outputs as laid out above; entries past a row's
   C_b clusters or L0 members are not written. ws: qs_semantic_index_workspace_size bytes,
   256-byte aligned, its first 256 bytes zeroed once (qs_workspace_init). 1 + 3 * iters
   launches. A page-table entry that is not mapped records QS_ERR_DEVICE_BOUNDS (kernel
   id 9). */
qs_status qs_semantic_index(const qs_config *cfg, const qs_cache *cache,
                            const int32_t *prompt_lens, int32_t iters, float *centroids,
                            int32_t *offsets, int32_t *members, int32_t batch, void *ws,
                            qs_stream_t stream);

/* One decode step's selection over the index (3 launches):
     beta_j = qbar . c_j (float32; qbar = the mean of the group's query heads), for
       j < C_b;
     the cfg->budget best clusters, ties to the lower index (all of them if C_b <= budget;
       no forced clusters);
     tokens[row] = the members of the selected clusters (clusters in ascending order, each
       cluster's members ascending), then every token L0 <= t < seq_len; n_tokens[row] =
       their count; the rest of the row is padded with -1.
   Attend with qs_sparse_attn on a configuration equal to cfg except block_size = 1 and
   budget = max_tokens (and a workspace sized for it), passing tokens / n_tokens as the
   selection. tokens: [rows][max_tokens] int32; a row needing more than max_tokens entries
   is cut and records QS_ERR_DEVICE_BOUNDS (kernel id 9). ws: qs_workspace_size(cfg, ...)
   bytes. q: [batch][Hq][head_dim] BF16, 4-byte aligned. */
qs_status qs_semantic_select(const qs_config *cfg, const qs_cache *cache, const void *q,
                             const int32_t *prompt_lens, const float *centroids,
                             const int32_t *offsets, const int32_t *members, int32_t batch,
                             int32_t *tokens, int32_t *n_tokens, int32_t max_tokens, void *ws,
                             qs_stream_t stream);

/* ---- Comparison kernels: full-KV attention and gather-then-attend -----------------------
   "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 2 (b) and
   Figure 6 (a), compare the sparse attention stage with attention over the whole cache
   (full-KV) and with a two-step variant that first copies the selected tokens into a
   contiguous buffer and then runs ordinary attention over it (gather-then-attend). These
   calls rebuild those comparisons on the same caches; they are not part of qs_decode. */

/* Workspace bytes that qs_dense_attn needs for caches of up to max_context tokens per
   sequence (host only). Same statuses as qs_workspace_size; max_context <= 131072. */
qs_status qs_dense_workspace_size(const qs_config *cfg, int32_t batch, int32_t max_context,
                                  size_t *bytes /* host */);

/* Full-KV decode attention: for every query head h of row (b, g),
     o_h = sum_{t < len} softmax_t(scale * q_h.k_t) v_t,
   len = row_lens[b * Hkv + g] if row_lens is not NULL, else seq_lens[b]; a row of length 0
   gives zeros. Heads, types, softmax scale and output type come from cfg (its block size,
   budget, forced blocks and attn_path are not used); the cache's proxy fields are not
   read. Logits are float32 sums of BF16 products, P.V operands v_agg_dtype, float32
   accumulation; the row is split over the tile-pipeline attention kernel and merged by
   the log-sum-exp combine (2 launches). Every len must be <= cache->max_context (a row
   that needs more than ceil(max_context / 128) pages records QS_ERR_DEVICE_BOUNDS). ws: qs_dense_workspace_size(cfg, batch,
   cache->max_context) bytes, initialised by qs_workspace_init. q is 16-byte aligned. */
qs_status qs_dense_attn(const qs_config *cfg, const qs_cache *cache, const void *q,
                        const int32_t *row_lens, int32_t batch, void *out, void *ws,
                        qs_stream_t stream);

/* Gather the selected blocks of every row into a compact paged buffer (one launch).
   With P = ceil(budget * block_size / 128) pages per sequence, k_dst and v_dst are
   [batch * P][Hkv][128][head_dim] (K BF16, V as v_dtype; 16-byte aligned). Gathered slot
   i * S + u of row (b, g) receives token sel[i] * S + u of that row, for i < n_sel; it is
   stored at page b * P + slot / 128, row slot % 128. Only a selected last block can be cut
   by seq_len, so the valid tokens form a prefix: row_lens[b * Hkv + g] (device int32
   [batch * Hkv]) receives its length, and slots after it are not written.
   qs_dense_attn over a qs_cache whose k / v are these buffers, whose page_table maps
   page i of sequence b to b * P + i and whose max_context is P * 128, with these
   row_lens, attends over exactly the selected tokens. A selection entry outside
   [0, ceil(seq_len / S)) or an unmapped page records QS_ERR_DEVICE_BOUNDS (kernel id 8)
   and skips the copy. */
qs_status qs_gather_kv(const qs_config *cfg, const qs_cache *cache, const int32_t *sel,
                       const int32_t *n_sel, int32_t batch, void *k_dst, void *v_dst,
                       int32_t *row_lens, void *ws, qs_stream_t stream);

/* The gather of the NVFP4 storage variant ("Jet-QSparse ...", Full text: the persistent
   cache keeps the keys in NVFP4 and at most two blocks per sequence at BF16). As
   qs_gather_kv (same arguments, layout and row_lens; one launch), except for the keys of
   blocks that are not kept: a kept block is one of the n_keep_hp complete blocks with the
   largest block_err, ties to the lower index; its keys are copied from the BF16 K pages.
   Every other selected token's key is read from the NVFP4 scoring cache and written as
     bf16_rne(fp32(fp32(e * sigma * g_k) + key_center[b][g][i]))   per element i
   (e * sigma is exact in float32). qs_dense_attn over the compact buffer then attends the
   way the storage variant does. cfg must be the NVFP4 configuration (else
   QS_ERR_UNSUPPORTED); block_err is needed when n_keep_hp > 0. */
qs_status qs_gather_kv_nvfp4k(const qs_config *cfg, const qs_cache *cache, const int32_t *sel,
                              const int32_t *n_sel, int32_t batch, void *k_dst, void *v_dst,
                              int32_t *row_lens, void *ws, qs_stream_t stream);

/* ---- Calibration of the scoring basis (once, before decoding) ----------------------------
   "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Abstract and
   Table 9: the shared subspace minimises a tractable bound on the token-score preservation
   error with a spectral solution, and unit-trace-normalised group-mean moments are
   compared with raw ones. The bound is not on the pages; the reading built here is
     M = C_q / tr(C_q) + C_k / tr(C_k)   (per KV head),
     C_q = mean over positions of qbar qbar^T, qbar = mean of the group's query heads,
     C_k = mean over positions of k k^T,
     P = the r eigenvectors of M with the largest eigenvalues, descending, each column
         signed so that its largest-magnitude entry (lowest index on ties) is positive.
   Moments are summed in FP64; the eigenvectors come from a cyclic Jacobi iteration on M in
   FP64 with the rotations accumulated in FP32 (one CTA per KV head). */

/* Workspace bytes for qs_calibrate_basis (host only): 256 + 2 * Hkv * d * d * 8. */
qs_status qs_calib_workspace_size(const qs_config *cfg, size_t *bytes /* host */);

/* Compute P [Hkv][d][r] (FP32, the layout qs_append_kv and qs_score take) from n calibration
   positions: q [n][Hq][d] BF16 queries and k [n][Hkv][d] BF16 keys. eigvals [Hkv][r] (FP32,
   may be NULL) receives the eigenvalues of M in the same order. r = cfg->proxy_rank (> 0,
   else QS_ERR_UNSUPPORTED). ws: qs_calib_workspace_size bytes, 256-byte aligned (no
   initialisation needed). Two launches; asynchronous on stream. */
qs_status qs_calibrate_basis(const qs_config *cfg, const void *q, const void *k, int32_t n,
                             float *P, float *eigvals, void *ws, qs_stream_t stream);

/* Synchronise `stream`, return the first device-side error recorded in the workspace
   since the last call (QS_OK if none) and clear it. `detail` (HOST pointer, may be NULL)
   receives {kernel id, index} of that error. Returns QS_ERR_CUDA if the synchronisation
   or the read-back fails. Kernel ids: 1 append, 2 block error, 3 scoring prep, 4 score,
   5 select, 6 attention (with its log-sum-exp combine), 7 the wait self-test,
   8 the gather of gather-then-attend, 9 the semantic-block index and expansion. The binary
   proxy's writer, scan and top-p selection report as 1, 4 and 5. */
qs_status qs_device_status(void *ws, qs_stream_t stream, uint32_t *detail);

/* Sparse attention without a workspace, for callers that cannot allocate device memory:
   for example a plugin of a host framework that owns all device memory and hands its
   kernels only their inputs and outputs, or a decode loop that may not call cudaMalloc
   because the allocation would synchronise the device. The pages describe no such call;
   it exists for these callers only.
   Computes exactly what qs_sparse_attn computes, with the same kernels; its partials and
   counters live in one static device array of QS_ATTN_STATIC_SCRATCH_BYTES
   inside the library (each GPU that loads the library holds it until the process exits),
   so the call allocates nothing and takes no workspace. The first call on a device looks
   up that array's device address (once per device, with the device current); make that
   first call before any stream capture. Every call clears the array's counters before
   its kernel runs, and all calls on a device share the array: calls whose work overlaps
   on the GPU (different streams, or different threads without ordering) race and must
   not be issued. Device-side bounds checks still skip invalid accesses, but their status
   word is not reported by this call.
   Returns QS_ERR_UNSUPPORTED if batch * Hq * parts * (head_dim + 2) * 4 bytes of partials
   plus batch * Hkv * 4 bytes of counters exceed QS_ATTN_STATIC_SCRATCH_BYTES (parts per
   query head is what qs_sparse_attn plans for the shape: chunks of the tile pipeline or
   splits of the gather kernel), and QS_ERR_CUDA if the address lookup or a launch fails;
   other arguments as for qs_sparse_attn. */
#define QS_ATTN_STATIC_SCRATCH_BYTES (4u << 20)
qs_status qs_sparse_attn_noalloc(const qs_config *cfg, const qs_cache *cache, const void *q,
                                 const int32_t *sel, const int32_t *n_sel, int32_t batch,
                                 void *out, qs_stream_t stream);

/* Static string naming a status code. */
const char *qs_status_string(qs_status s);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t qs_version(void);

/* Diagnostic: launch one kernel whose bounded wait (the same mbarrier wait the library's
   kernels use) waits for an arrival that never comes; it must give up after a short limit
   and record QS_ERR_DEVICE_TIMEOUT in the workspace status word (kernel id 7), which
   qs_device_status then returns. The pages describe no such call: it lets a caller check on
   a given GPU that a lost arrival ends in a reported error, not a hang, and that the
   context stays usable. ws: a workspace as for the other calls (only its status word is
   used). */
qs_status qs_selftest_wait_timeout(void *ws, qs_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* QS_H */
