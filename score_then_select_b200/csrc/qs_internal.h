// qs_internal.h - parameter blocks and launchers shared by the libqs translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <utility>

#include "../../include/qs.h"

namespace qs {

// kernel ids recorded with device-side errors (documented in qs.h)
enum KernelId : uint32_t {
  KID_APPEND = 1,
  KID_BLOCKERR = 2,
  KID_PREP = 3,
  KID_SCORE = 4,
  KID_SELECT = 5,
  KID_ATTN = 6,
  KID_SELFTEST = 7,
  KID_GATHER = 8
};

constexpr int kPage = 128;          // tokens per page (the only page size built)
constexpr int kMaxBatch = 1024;     // sequences per call
constexpr int kMaxGroup = 8;        // query heads per KV head
constexpr int kMaxSelectBlocks = 131072;  // 32768 per CTA, clusters of 4 CTAs beyond
constexpr int kHdrWords = 64;       // workspace header (256 bytes)
constexpr int kCtrAppend = 16;      // header word: append "last CTA" counter
constexpr int kAttnCtasPerSm = 2;   // resident attention CTAs per SM (shared-memory bound)
constexpr int kAttnTmaMinRun = 8;   // shorter selected runs (block size) use the gather kernel
constexpr int kChunkTilesMax = 8;   // attention work unit: up to 8 tiles (512 slots) of one row
constexpr int kChunksPerCta = 6;    // chunk size target: about this many chunks per CTA
constexpr int kTmaMinTilesPerCta = 40;  // auto path: tile pipeline from this much work per CTA
constexpr int kCtrAttnNext = 17;    // header word: next attention chunk to claim

// Workspace carve-up (byte offsets); computed identically by qs_workspace_size and calls.
struct WsLayout {
  size_t qt = 0;        // rank r: q~ [batch][Hkv][r] f32
  size_t qtile = 0;     // NVFP4: query tiles [batch][Hkv][kQTileBytes]
  size_t qgscale = 0;   // NVFP4: g_q (1 float)
  size_t scores = 0;    // [batch][Hkv][nb_stride] f32
  size_t sel = 0;       // [batch][Hkv][budget] i32
  size_t nsel = 0;      // [batch][Hkv] i32
  size_t part_ml = 0;   // [batch][Hq][parts_per_head][2] f32 attention partials (m, l)
  size_t part_o = 0;    // [batch][Hq][parts_per_head][d] f32 attention partials o
  size_t row_ctr = 0;   // [batch][Hkv] u32 attention segments finished per row
  size_t kept = 0;      // NVFP4 key storage: [batch][Hkv][2] i32 kept blocks (-1: none)
  size_t total = 0;
  int nb_stride = 0;
  int attn_ctas = 0;     // attention grid (persistent; chunks claimed dynamically)
  int tiles_per_row = 0; // 64-token tiles of selected slots per row
  int chunk_tiles = 0;   // tiles per attention chunk: min(8, 32 / runs per tile)
  int chunks_per_row = 0;  // chunks per row (one partial each)
  int gsplits = 0;      // gather kernel: splits per row
  int g_tokens_per_split = 0;
  int parts_per_head = 0;  // attention partials per query head in the workspace
};

// Scoring proxy of a configuration
enum ProxyKind : int { PK_RANKR = 0, PK_NVFP4 = 1, PK_CENTROID = 2 };

struct Plan {
  int batch, Hq, Hkv, G, d, S, budget, r, nb_stride;
  int kind;             // ProxyKind
  bool attn_tma;        // attention by the tile pipeline (else the gather kernel)
  int proxy_dtype, v_dtype, v_agg_dtype, out_dtype;
  int force_sink, force_last, n_keep;
  bool key_nvfp4 = false;   // attention reads the NVFP4 keys (kept blocks BF16)
  float scale;
  WsLayout ws;
};

// ------------------------------------------------------------ kernel parameter blocks
struct AppendParams {
  const uint16_t* k_new;   // [batch][Hkv][max_new][d]
  const uint16_t* v_new;
  const int32_t* n_new;    // [batch] or nullptr (=> 1 token each)
  const float* P;          // [Hkv][d][r]
  uint16_t* k;             // cache pages
  uint16_t* v;
  void* proxy;
  uint8_t* proxy_scale;
  const float* key_center;
  const float* key_gscale;
  const int32_t* page_table;
  int32_t* seq_lens;
  uint32_t* hdr;
  // fused scoring prep (rank r): q~ of each row, or nullptr
  const uint16_t* q;
  float* qt;
  int batch, Hkv, G, d, r, max_new, max_pages_per_seq, num_pages, max_context;
  int S;                     // block size (centroid sums)
};

struct BlockErrParams {
  const uint16_t* k;
  const float* key_center;
  const float* key_gscale;
  const int32_t* page_table;
  const int32_t* seq_lens;  // already advanced
  const int32_t* n_new;     // [batch] or nullptr (=> 1)
  float* block_err;
  uint32_t* hdr;
  int batch, Hkv, d, S, nb_stride, max_pages_per_seq, num_pages, max_blocks_per_call;
};

struct PrepParams {          // rank r scoring prep (standalone qs_score)
  const uint16_t* q;
  const float* P;
  float* qt;
  int batch, Hkv, G, d, r;
};

struct QPackParams {         // NVFP4 query packing
  const uint16_t* q;
  uint8_t* tiles;            // [batch * Hkv][kQTileBytes]
  float* gscale;
  int n;                     // batch * Hq * d
  int rows, Hkv, G;
};

// ---- NVFP4 layouts (d = 128; documented in include/qs.h) -----------------------------
// Codes of one (page, KV head): [4 chunks][128 tokens][16 bytes]; chunk c of a token holds
// its elements 32c .. 32c+31 (two per byte, even element in the low nibble). A plain
// contiguous copy of the 8 KiB lands in shared memory as the K-major, no-swizzle operand
// of the FP4 tensor-core MMA (8-token x 16-byte core matrices).
constexpr int kNvfp4PageCodeBytes = 128 * 64;
// Scales of one (page, KV head): two 512-byte blocks (elements 0..63 and 64..127); in a
// block, token m's 4 scales sit at 16 * (m % 32) + 4 * (m / 32): the order the tensor
// cores' scale-factor copy expects.
constexpr int kNvfp4PageScaleBytes = 1024;
// Query tile of one row: 512 bytes of B-operand codes [4 chunks][8 heads][16 B] and two
// 512-byte scale blocks (head n's 4 scales at 16 * n).
constexpr int kQTileBytes = 512 + 1024;

__host__ __device__ inline int nvfp4_code_off(int token, int group) {
  return (group >> 1) * 2048 + token * 16 + (group & 1) * 8;
}
__host__ __device__ inline int nvfp4_scale_off(int token, int group) {
  return (group >> 2) * 512 + 16 * (token & 31) + 4 * (token >> 5) + (group & 3);
}
__host__ __device__ inline int qtile_code_off(int head, int group) {
  return (group >> 1) * 128 + head * 16 + (group & 1) * 8;
}
__host__ __device__ inline int qtile_scale_off(int head, int group) {
  return 512 + (group >> 2) * 512 + 16 * head + (group & 3);
}

struct ScoreParams {
  const uint16_t* q;         // centroid scoring: the queries [batch][Hq][d]
  const void* proxy;
  const uint8_t* proxy_scale;
  const float* qt;           // rank r: [batch][Hkv][r]
  const uint8_t* qtile;      // NVFP4: [batch][Hkv][kQTileBytes]
  const float* qgscale;
  const float* key_gscale;
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* scores;
  uint32_t* hdr;
  int batch, Hkv, G, d, S, nb_stride, max_pages_per_seq, num_pages, max_context;
  // 1: the kernel before this one (launched in stream order, without overlap) writes only
  // the query side (q~, or the NVFP4 query tiles and g_q), so the page stream may start
  // before waiting for it; 0: wait for it first (it may still be writing seq_lens)
  int early_stream;
};

struct SelectParams {
  const float* scores;
  const float* block_err;    // NVFP4 kept blocks, or nullptr
  const int32_t* seq_lens;
  int32_t* sel;
  int32_t* n_sel;
  uint32_t* hdr;
  int rows, Hkv, S, nb_stride, budget, force_sink, force_last, n_keep;
};

struct AttnParams {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* sel;        // nullptr: full KV (every block of the row, in order)
  const int32_t* n_sel;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* row_lens;   // [batch * Hkv] tokens per row, or nullptr (=> seq_lens[b])
  float* part_ml;
  float* part_o;
  uint32_t* row_ctr;         // [batch * Hkv] segments finished (self-resetting)
  void* out;
  uint32_t* hdr;
  int rows, Hkv, G, S, budget, tiles_per_row, chunk_tiles, chunks_per_row, max_pages_per_seq,
      num_pages;
  int run_h;                 // min(S, 64): rows of one box copy
  int log2_S, log2_run;
  int gsplits, g_tokens_per_split;   // gather kernel split plan
  int out_bf16;
  float scale_log2;          // softmax scale * log2(e)
  // NVFP4 key storage: keys from the scoring cache (codes, scales, g_k, the row's centre),
  // except the row's kept blocks (kept[row][0..1], -1: none), which come from k
  const uint8_t* k_codes;
  const uint8_t* k_scales;
  const float* key_center;
  const float* key_gscale;
  const int32_t* kept;
};

struct GatherParams {        // gather-then-attend: selected blocks -> compact pages
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* sel;
  const int32_t* n_sel;
  const int32_t* page_table;
  const int32_t* seq_lens;
  uint16_t* k_dst;           // [batch * dst_pages_per_seq][Hkv][128][d]
  uint16_t* v_dst;
  int32_t* row_lens;         // [batch * Hkv] gathered valid tokens
  uint32_t* hdr;
  int rows, Hkv, log2_S, budget, dst_pages_per_seq, max_pages_per_seq, num_pages;
};

struct CalibParams {        // calibration of the scoring basis (calib.cu)
  const uint16_t* q;         // [n][Hq][d] BF16
  const uint16_t* k;         // [n][Hkv][d] BF16
  double* mq;                // [Hkv][d][d] sum of qbar qbar^T
  double* mk;                // [Hkv][d][d] sum of k k^T
  float* P;                  // [Hkv][d][r]
  float* eig;                // [Hkv][r] or nullptr
  int n, Hkv, G, d, r;
};

// Launch `kern` on `s`; with `pdl` the launch may overlap the tail of the previous kernel
// in the stream (the kernel must call pdl_wait() before reading that kernel's results).
template <typename... P, typename... A>
inline cudaError_t launch_k(void (*kern)(P...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t s, bool pdl, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// ------------------------------------------------------------ launchers (return launch error)
cudaError_t launch_append(const Plan& p, const AppendParams& a, cudaStream_t s);
cudaError_t launch_block_err(const Plan& p, const BlockErrParams& a, cudaStream_t s);
cudaError_t launch_prep(const Plan& p, const PrepParams& a, cudaStream_t s);
cudaError_t launch_qpack(const Plan& p, const QPackParams& a, cudaStream_t s, bool pdl);
cudaError_t launch_score(const Plan& p, const ScoreParams& a, cudaStream_t s, bool pdl);
cudaError_t launch_select(const Plan& p, const SelectParams& a, cudaStream_t s, bool pdl);
cudaError_t launch_attn_gather(const Plan& p, const AttnParams& a, cudaStream_t s, bool pdl);
cudaError_t launch_attn(const Plan& p, const AttnParams& a, cudaStream_t s, bool pdl);
cudaError_t launch_gather_kv(const Plan& p, const GatherParams& a, cudaStream_t s);
cudaError_t launch_calibrate(const CalibParams& a, cudaStream_t s);
size_t calib_ws_bytes(int Hkv, int d);

int num_sms();   // SM count of the current device (cached per device)

// Raise `kern`'s dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device): function attributes are per device, and one process may drive several
// GPUs. Thread-safe.
cudaError_t set_smem_limit(const void* kern, int bytes);
template <typename... P>
inline cudaError_t set_smem_limit(void (*kern)(P...), int bytes) {
  return set_smem_limit(reinterpret_cast<const void*>(kern), bytes);
}

// host-side validation and launch planning (api.cu)
qs_status make_plan(const qs_config* c, int batch, int max_context, Plan& p);
qs_status check_cache(const Plan& p, const qs_cache* c, bool need_proxy);

}  // namespace qs
