// semantic.h - host/device definitions of the semantic-block index and its decode side.
//
// "Coarse Semantic Blocks for Efficient Training-Free Sparse Attention" (Abstract): the
// prompt's keys are clustered into large blocks of non-contiguous tokens; a query scores
// each block by its centroid and attends to the original keys and values of the blocks it
// selects. The clustering is Lloyd's k-means with every decision taken in float32 in a
// fixed order (the oracle's kmeans_keys_f32):
//   seeds: the keys at floor(j * L0 / C), C = ceil(L0 / S);
//   assign: d_tj = sum over i ascending of fp32((x_ti - c_ji)^2), one rounding per
//           difference, square and sum; the smallest d_tj wins, ties to the lower j;
//   update: c_j = fp32(sum of the members' keys in token order) / fp32(count), an empty
//           cluster keeping its centroid.
// The index of one row (sequence b, KV head g): centroids [C_max][d] f32, member offsets
// [C_max + 1] (CSR) and members [L_max] (token positions, by cluster, ascending within).
#pragma once

#include "qs_internal.h"

namespace qs {

constexpr ProxyKind PK_SEMANTIC = ProxyKind(4);   // QS_SEMANTIC, rank 0
constexpr uint32_t KID_SEMANTIC = 9;              // status-word kernel id

struct SemIndexParams {
  const uint16_t* k;            // K pages, BF16
  const int32_t* page_table;
  const int32_t* prompt_lens;   // [batch]: L0 of each sequence
  float* cent;                  // [rows][c_max][d]
  int32_t* offsets;             // [rows][c_max + 1]
  int32_t* members;             // [rows][l_max]
  int32_t* assign;              // workspace [rows][l_max]
  int32_t* cursor;              // workspace [rows][c_max]
  uint32_t* hdr;
  int batch, Hkv, d, S, c_max, l_max, max_pages_per_seq, num_pages;
};

struct SemSelectParams {
  const uint16_t* q;            // [batch][Hq][d] BF16
  const int32_t* prompt_lens;   // [batch]
  const int32_t* seq_lens;      // [batch]
  const float* cent;
  const int32_t* offsets;
  const int32_t* members;
  float* scores;                // workspace [rows][c_max]
  int32_t* n_clusters;          // workspace [batch]: C of each sequence
  const int32_t* csel;          // [rows][budget] selected clusters (from the select kernel)
  const int32_t* n_csel;        // [rows]
  int32_t* tokens;              // [rows][max_tokens]
  int32_t* n_tokens;            // [rows]
  uint32_t* hdr;
  int batch, Hkv, G, d, S, c_max, l_max, budget, max_tokens;
};

cudaError_t launch_sem_index(const SemIndexParams& a, int iters, cudaStream_t s);
cudaError_t launch_sem_score(const SemSelectParams& a, cudaStream_t s);
cudaError_t launch_sem_expand(const SemSelectParams& a, cudaStream_t s);

}  // namespace qs
