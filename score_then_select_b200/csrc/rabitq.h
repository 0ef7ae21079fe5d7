// rabitq.h - host/device definitions of the binary-code scoring proxy with a top-p budget.
//
// "RaBitQCache" (Abstract): keys are scored through 1-bit codes of their randomly rotated
// directions and a 4-bit code of the rotated query, and the attended set grows until the
// estimated attention mass reaches p. The estimator is the published RaBitQ one (J. Gao
// and C. Long, SIGMOD 2024, section 3): with o = k - c and y = o R,
//   <o, q> ~= (|o|^2 / |y|_1) sum_i (2 b_i - 1) (q R)_i,   b_i = [y_i > 0],
// unbiased over a uniformly random rotation R and a uniformly random rounding of the
// query to its 4-bit grid.
//
// Scoring cache of one (page, KV head): 128 x d/8 bytes of code bits (token slot s at
// byte s * d/8; bit i of the key at byte i / 8, position i % 8), then 128 FP32 factors
// g = |o|^2 / |y|_1.
#pragma once

#include "qs_internal.h"

namespace qs {

constexpr ProxyKind PK_RABITQ = ProxyKind(3);   // QS_RABITQ, rank 0
constexpr int kRqBits = 4;                       // bits of the query code
constexpr int kRqLevels = (1 << kRqBits) - 1;    // codes 0 .. 15
constexpr int kRqRowWords = 32;                  // workspace words per row's query code

// Bytes of one (page, KV head) of the scoring cache.
inline int rq_page_bytes(int d) { return kPage * (d / 8) + kPage * 4; }

// Query code of one row in the workspace (kRqRowWords uint32 words):
//   [0, 4 * d/32)   bit planes: plane p, word w holds bit p of the codes of dims 32w..32w+31
//   [24]            Delta (float bits)       [25] v_l (float bits)
//   [26]            Q = sum of the codes     [27] c . qbar (float bits)
//   [28]            the row's largest block score, as its order-preserving key (0: none),
//                   reset by the query-code kernel and raised by the scan
constexpr int kRqDelta = 24, kRqVl = 25, kRqQsum = 26, kRqShift = 27, kRqRowMax = 28;

struct RqPrepParams {
  const uint16_t* q;          // [batch][Hq][d] BF16
  const float* R;             // [Hkv][d][d]
  const float* u;             // [batch][Hkv][d] rounding draws in [0, 1)
  const float* key_center;    // [batch][Hkv][d]
  uint32_t* qcode;            // [batch][Hkv][kRqRowWords]
  int batch, Hkv, G, d;
};

struct RqScoreParams {
  const uint8_t* proxy;       // scoring cache pages
  uint32_t* qcode;            // read; word kRqRowMax of each row raised
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* scores;              // [batch][Hkv][nb_stride]: log of each block's mass
  uint32_t* hdr;
  int batch, Hkv, d, S, nb_stride, max_pages_per_seq, num_pages, max_context;
  float scale;                // softmax scale
};

struct TopPParams {
  const float* scores;        // [rows][nb_stride] natural-log block masses
  const int32_t* seq_lens;
  int32_t* sel;               // [rows][budget]
  int32_t* n_sel;             // [rows]
  uint32_t* hdr;
  // the rows' largest scores as order-preserving keys, written by the scan that produced
  // `scores` (row r's at row_max[r * row_max_stride]); null: the select finds them itself
  const uint32_t* row_max;
  int row_max_stride;
  int rows, Hkv, S, nb_stride, budget, force_sink, force_last;
  float p;
};

cudaError_t launch_rq_prep(const RqPrepParams& a, cudaStream_t s);
cudaError_t launch_rq_score(const RqScoreParams& a, cudaStream_t s);
cudaError_t launch_top_p(const TopPParams& a, cudaStream_t s);

}  // namespace qs
