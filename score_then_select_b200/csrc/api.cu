// api.cu - the C ABI of libqs: argument validation, launch plans, workspace layout and
// the entry points declared in include/qs.h. No device memory is allocated here.
#include <atomic>
#include <cmath>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "qs_internal.h"
#include "rabitq.h"
#include "semantic.h"
#include "nvfp4k.h"

namespace qs {
cudaError_t launch_select_radix(const SelectParams& a, cudaStream_t s);
}

namespace qs {

int num_sms() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cached[kMaxDevices] = {};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  if (dev >= 0 && dev < kMaxDevices && cached[dev].load() > 0) return cached[dev].load();
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  if (dev >= 0 && dev < kMaxDevices) cached[dev].store(n);
  return n;
}

cudaError_t set_smem_limit(const void* kern, int bytes) {
  struct Done { const void* kern; int dev, bytes; };
  static std::mutex mu;
  static std::vector<Done> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Done& d : done)
    if (d.kern == kern && d.dev == dev && d.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back(Done{kern, dev, bytes});
  return e;
}

static bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Split plan of the gather kernel (selections of runs shorter than 8 slots): splits per row
// so the (row, split) grid fills whole waves of resident CTAs (2 per SM) as evenly as
// possible; tokens per split is a multiple of the 64-token tile.
static void plan_gather_splits(int rows, int slots, int& splits, int& tps) {
  const int slots_per_wave = 2 * num_sms();
  double best = 1e30;
  splits = 1;
  tps = 64;
  for (int s = 1; s <= 64; ++s) {
    int t = (slots + s - 1) / s;
    t = (t + 63) / 64 * 64;
    if (t > 2048) continue;
    if ((s - 1) * t >= slots && s > 1) break;  // later splits would be empty
    const long long ctas = (long long)rows * s;
    const long long waves = (ctas + slots_per_wave - 1) / slots_per_wave;
    // time model: waves x tokens per CTA, plus a small per-CTA fixed cost
    const double cost = double(waves) * (t + 96.0);
    if (cost < best - 1e-9) {
      best = cost;
      splits = s;
      tps = t;
    }
  }
}

// Attention work plan (runs of >= 8 slots): each row's selected slots form
// ceil(budget * S / 64) tiles, cut into chunks of up to kChunkTilesMax tiles (one partial
// each; a chunk's runs of min(S, 64) slots must fit one warp's lanes);
// a persistent grid of kAttnCtasPerSm CTAs per SM (no more CTAs than chunks) claims them.
static void plan_attention(int rows, long long slots, int S, WsLayout& w) {
  const long long tpr = (slots + 63) / 64;
  const int runs_per_tile = S >= 64 ? 1 : 64 / S;         // a chunk's runs fit one warp
  const int kt_max = std::max(1, std::min(kChunkTilesMax, 32 / runs_per_tile));
  // about kChunksPerCta chunks per CTA, so the dynamic claims can even out the CTAs' speeds
  const long long ctas = (long long)kAttnCtasPerSm * num_sms();
  const long long want = rows * tpr / (ctas * kChunksPerCta);
  const int kt = int(std::max(1LL, std::min<long long>(kt_max, want)));
  const long long cpr = (tpr + kt - 1) / kt;
  const long long chunks = rows * cpr;                   // < 2^31: checked by the caller
  long long C = ctas;
  if (C > chunks) C = chunks;
  w.tiles_per_row = int(tpr);
  w.chunk_tiles = kt;
  w.chunks_per_row = int(cpr);
  w.attn_ctas = int(C);
}

qs_status make_plan(const qs_config* c, int batch, int max_context, Plan& p) {
  if (!c) return QS_ERR_INVALID_ARG;
  if (batch < 1 || batch > kMaxBatch || max_context < 1) return QS_ERR_INVALID_ARG;
  if (c->n_kv_heads < 1 || c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads) return QS_ERR_INVALID_ARG;
  if (c->budget < 1 || c->page_size < 1 || c->block_size < 1) return QS_ERR_INVALID_ARG;
  if (!is_pow2(c->block_size) || c->page_size % c->block_size) return QS_ERR_INVALID_ARG;
  if (c->force_sink < 0 || c->force_sink > 1 || c->force_last < 0 || c->force_last > 1)
    return QS_ERR_INVALID_ARG;
  if (c->n_keep_hp < 0 || c->n_keep_hp > 2) return QS_ERR_INVALID_ARG;
  if (!(c->softmax_scale >= 0.0f) || !std::isfinite(c->softmax_scale)) return QS_ERR_INVALID_ARG;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (G > kMaxGroup) return QS_ERR_UNSUPPORTED;
  if (c->page_size != kPage) return QS_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return QS_ERR_UNSUPPORTED;
  const int r = c->proxy_rank;
  if (r < 0) return QS_ERR_INVALID_ARG;
  p.kind = r > 0 ? PK_RANKR
         : c->proxy_dtype == QS_CENTROID ? PK_CENTROID
         : c->proxy_dtype == QS_RABITQ   ? PK_RABITQ
         : c->proxy_dtype == QS_SEMANTIC ? PK_SEMANTIC
                                         : PK_NVFP4;
  if (p.kind == PK_CENTROID || p.kind == PK_RABITQ || p.kind == PK_SEMANTIC) {
    if (c->n_keep_hp != 0) return QS_ERR_INVALID_ARG;
  } else if (r > 0) {
    const bool ok = (c->proxy_dtype == QS_F32 && (r == 16 || (r == 32 && c->head_dim == 128))) ||
                    ((c->proxy_dtype == QS_BF16 || c->proxy_dtype == QS_E4M3) &&
                     (r == 32 || (r == 64 && c->head_dim == 128)));
    if (!ok) return QS_ERR_UNSUPPORTED;
    if (c->n_keep_hp != 0) return QS_ERR_INVALID_ARG;
  } else {
    if (c->proxy_dtype != QS_NVFP4) return QS_ERR_INVALID_ARG;
    if (c->head_dim != 128) return QS_ERR_UNSUPPORTED;
    if (c->block_size != kPage) return QS_ERR_UNSUPPORTED;
  }
  if (c->v_dtype != QS_BF16 && c->v_dtype != QS_F16) return QS_ERR_INVALID_ARG;
  if (c->v_agg_dtype != QS_BF16 && c->v_agg_dtype != QS_F16) return QS_ERR_INVALID_ARG;
  if (c->v_dtype == QS_F16 && c->v_agg_dtype != QS_F16) return QS_ERR_UNSUPPORTED;
  if (c->out_dtype != QS_F32 && c->out_dtype != QS_BF16) return QS_ERR_INVALID_ARG;
  if (c->key_storage != 0 && c->key_storage != QS_BF16 && c->key_storage != QS_NVFP4)
    return QS_ERR_INVALID_ARG;
  p.key_nvfp4 = c->key_storage == QS_NVFP4;
  if (p.key_nvfp4) {
    // the scoring copy must be NVFP4 (d = 128, 128-token blocks, checked above); the
    // decode happens in the tile pipeline
    if (p.kind != PK_NVFP4) return QS_ERR_INVALID_ARG;
    if (c->attn_path == 2) return QS_ERR_UNSUPPORTED;
  }

  p.batch = batch;
  p.Hq = c->n_q_heads;
  p.Hkv = c->n_kv_heads;
  p.G = G;
  p.d = c->head_dim;
  p.S = c->block_size;
  p.budget = c->budget;
  p.r = r;
  p.proxy_dtype = c->proxy_dtype;
  p.v_dtype = c->v_dtype;
  p.v_agg_dtype = c->v_agg_dtype;
  p.out_dtype = c->out_dtype;
  p.force_sink = c->force_sink;
  p.force_last = c->force_last;
  p.n_keep = c->n_keep_hp;
  p.scale = c->softmax_scale > 0.0f ? c->softmax_scale : 1.0f / std::sqrt(float(c->head_dim));
  const long long pages = (max_context + kPage - 1) / kPage;
  const long long nbs = pages * (kPage / p.S);
  if (nbs > kMaxSelectBlocks) return QS_ERR_UNSUPPORTED;
  if (nbs > 32768 && c->n_keep_hp > 0) return QS_ERR_UNSUPPORTED;  // kept blocks: one CTA per row
  p.nb_stride = int(nbs);
  const long long slots = (long long)p.budget * p.S;
  if (slots > 64LL * 2048) return QS_ERR_UNSUPPORTED;

  WsLayout& w = p.ws;
  w.nb_stride = p.nb_stride;
  if ((long long)batch * p.Hkv * ((slots + 63) / 64) >= (1LL << 31)) return QS_ERR_UNSUPPORTED;
  if (c->attn_path < 0 || c->attn_path > 2) return QS_ERR_INVALID_ARG;
  if (c->attn_path == 1 && p.S < kAttnTmaMinRun) return QS_ERR_UNSUPPORTED;
  {
    const long long tiles = (long long)batch * p.Hkv * ((slots + 63) / 64);
    const long long ctas = (long long)kAttnCtasPerSm * num_sms();
    p.attn_tma = c->attn_path == 1 || p.key_nvfp4 ||
                 (c->attn_path == 0 && p.S >= kAttnTmaMinRun && tiles >= kTmaMinTilesPerCta * ctas);
  }
  if (p.attn_tma) {
    plan_attention(batch * p.Hkv, slots, p.S, w);
    w.parts_per_head = w.chunks_per_row;
  } else {
    plan_gather_splits(batch * p.Hkv, int(slots), w.gsplits, w.g_tokens_per_split);
    w.parts_per_head = w.gsplits;
  }
  size_t off = size_t(kHdrWords) * 4;
  const size_t rows = size_t(batch) * p.Hkv, rows_q = size_t(batch) * p.Hq;
  // the self-resetting row counters first: at the same place for every batch, so a
  // workspace initialised for `batch` sequences serves calls of fewer sequences too
  w.row_ctr = off; off = align_up(off + rows * 4, 256);
  w.qt = off;      off = align_up(off + rows * (r > 0 ? r : (p.kind == PK_RABITQ ? kRqRowWords : 1)) * 4, 256);
  w.qtile = off;   off = align_up(off + (p.kind == PK_NVFP4 ? rows * kQTileBytes : 0), 256);
  w.qgscale = off; off = align_up(off + 16, 256);
  w.scores = off;  off = align_up(off + rows * p.nb_stride * 4, 256);
  w.sel = off;     off = align_up(off + rows * p.budget * 4, 256);
  w.nsel = off;    off = align_up(off + rows * 4, 256);
  w.part_ml = off; off = align_up(off + rows_q * w.parts_per_head * 2 * 4, 256);
  w.part_o = off;  off = align_up(off + rows_q * w.parts_per_head * p.d * 4, 256);
  w.kept = off;    off = align_up(off + (p.key_nvfp4 ? rows * 2 * 4 : 0), 256);
  w.total = off;
  return QS_OK;
}

// Plan of full-KV attention: the configuration's heads, types and scale, with every
// 128-token block of a row selected in order (block size = page size, budget = pages of
// max_context), always on the tile pipeline. The configuration itself must be valid.
static qs_status make_dense_plan(const qs_config* c, int batch, int max_context, Plan& p) {
  qs_status st = make_plan(c, batch, max_context, p);
  if (st != QS_OK) return st;
  qs_config d = *c;
  d.block_size = kPage;
  d.budget = (max_context + kPage - 1) / kPage;
  d.force_sink = d.force_last = 0;
  d.n_keep_hp = 0;
  d.attn_path = 1;
  d.key_storage = 0;            // the full-KV comparison reads the BF16 key pages
  return make_plan(&d, batch, max_context, p);
}

qs_status check_cache(const Plan& p, const qs_cache* c, bool need_proxy) {
  if (!c || !c->k || !c->v || !c->page_table || !c->seq_lens) return QS_ERR_INVALID_ARG;
  if (c->max_pages_per_seq < 1 || c->num_pages < 1 || c->max_context < 1) return QS_ERR_INVALID_ARG;
  if ((long long)c->num_pages * p.Hkv * kPage >= (1LL << 31)) return QS_ERR_UNSUPPORTED;
  if (!aligned(c->k, 16) || !aligned(c->v, 16)) return QS_ERR_INVALID_ARG;
  if (need_proxy && p.kind != PK_SEMANTIC) {      // the semantic index lives outside the cache
    if (!c->proxy || !aligned(c->proxy, 16)) return QS_ERR_INVALID_ARG;
    if (p.kind == PK_NVFP4 && (!c->proxy_scale || !c->key_center || !c->key_gscale))
      return QS_ERR_INVALID_ARG;
    if (p.kind == PK_RABITQ && !c->key_center) return QS_ERR_INVALID_ARG;
  }
  // attention over the NVFP4 keys reads the codes, scales and centres by bulk copies and
  // the block errors for the kept blocks, whatever the call
  if (p.key_nvfp4) {
    if (!c->proxy || !c->proxy_scale || !c->key_center || !c->key_gscale) return QS_ERR_INVALID_ARG;
    if (p.n_keep > 0 && !c->block_err) return QS_ERR_INVALID_ARG;
    if (!aligned(c->proxy, 16) || !aligned(c->proxy_scale, 16) || !aligned(c->key_center, 16))
      return QS_ERR_INVALID_ARG;
  }
  return QS_OK;
}

static uint32_t* hdr_of(void* ws) { return reinterpret_cast<uint32_t*>(ws); }
template <typename T>
static T* ws_at(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(ws) + off);
}

static qs_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QS_OK : QS_ERR_CUDA; }

// ------------------------------------------------------------ stage bodies (validated input)
static qs_status do_append(const Plan& p, const qs_cache* c, const void* k_new, const void* v_new,
                           const int32_t* n_new, int max_new, const float* P, const void* q,
                           void* ws, cudaStream_t s) {
  AppendParams a{};
  a.k_new = static_cast<const uint16_t*>(k_new);
  a.v_new = static_cast<const uint16_t*>(v_new);
  a.n_new = n_new;
  a.P = P;
  a.k = static_cast<uint16_t*>(c->k);
  a.v = static_cast<uint16_t*>(c->v);
  a.proxy = c->proxy;
  a.proxy_scale = c->proxy_scale;
  a.key_center = c->key_center;
  a.key_gscale = c->key_gscale;
  a.page_table = c->page_table;
  a.seq_lens = c->seq_lens;
  a.hdr = hdr_of(ws);
  a.q = (p.r > 0) ? static_cast<const uint16_t*>(q) : nullptr;
  a.qt = ws_at<float>(ws, p.ws.qt);
  a.batch = p.batch;
  a.Hkv = p.Hkv;
  a.G = p.G;
  a.d = p.d;
  a.r = p.r;
  a.max_new = max_new;
  a.max_pages_per_seq = c->max_pages_per_seq;
  a.num_pages = c->num_pages;
  a.max_context = c->max_context;
  a.S = p.S;
  qs_status st = cuda_status(launch_append(p, a, s));
  if (st != QS_OK || p.kind != PK_NVFP4) return st;
  BlockErrParams e{};
  e.k = a.k;
  e.key_center = c->key_center;
  e.key_gscale = c->key_gscale;
  e.page_table = c->page_table;
  e.seq_lens = c->seq_lens;
  e.n_new = n_new;
  e.block_err = c->block_err;
  e.hdr = a.hdr;
  e.batch = p.batch;
  e.Hkv = p.Hkv;
  e.d = p.d;
  e.S = p.S;
  e.nb_stride = p.nb_stride;
  e.max_pages_per_seq = c->max_pages_per_seq;
  e.num_pages = c->num_pages;
  e.max_blocks_per_call = max_new / p.S + 1;
  return cuda_status(launch_block_err(p, e, s));
}

static qs_status do_prep(const Plan& p, const void* q, const float* P, void* ws, cudaStream_t s,
                         bool pdl) {
  if (p.kind == PK_CENTROID) return QS_OK;          // the scan averages the queries itself
  if (p.r > 0) {
    PrepParams a{static_cast<const uint16_t*>(q), P, ws_at<float>(ws, p.ws.qt),
                 p.batch, p.Hkv, p.G, p.d, p.r};
    return cuda_status(launch_prep(p, a, s));
  }
  QPackParams a{static_cast<const uint16_t*>(q), ws_at<uint8_t>(ws, p.ws.qtile),
                ws_at<float>(ws, p.ws.qgscale), p.batch * p.Hq * p.d, p.batch * p.Hkv, p.Hkv,
                p.G};
  return cuda_status(launch_qpack(p, a, s, pdl));
}

static qs_status do_score(const Plan& p, const qs_cache* c, const void* q, float* scores, void* ws,
                          cudaStream_t s, bool pdl, bool early_stream = false) {
  ScoreParams a{};
  a.early_stream = early_stream ? 1 : 0;
  a.q = static_cast<const uint16_t*>(q);
  a.proxy = c->proxy;
  a.proxy_scale = c->proxy_scale;
  a.qt = ws_at<float>(ws, p.ws.qt);
  a.qtile = ws_at<uint8_t>(ws, p.ws.qtile);
  a.qgscale = ws_at<float>(ws, p.ws.qgscale);
  a.key_gscale = c->key_gscale;
  a.page_table = c->page_table;
  a.seq_lens = c->seq_lens;
  a.scores = scores;
  a.hdr = hdr_of(ws);
  a.batch = p.batch;
  a.Hkv = p.Hkv;
  a.G = p.G;
  a.d = p.d;
  a.S = p.S;
  a.nb_stride = p.nb_stride;
  a.max_pages_per_seq = c->max_pages_per_seq;
  a.num_pages = c->num_pages;
  a.max_context = c->max_context;
  return cuda_status(launch_score(p, a, s, pdl));
}

static qs_status do_select(const Plan& p, const qs_cache* c, const float* scores, int32_t* sel,
                           int32_t* n_sel, void* ws, cudaStream_t s, bool pdl) {
  SelectParams a{};
  a.scores = scores;
  a.block_err = (p.kind == PK_NVFP4 && p.n_keep > 0) ? c->block_err : nullptr;
  a.seq_lens = c->seq_lens;
  a.sel = sel;
  a.n_sel = n_sel;
  a.hdr = hdr_of(ws);
  a.rows = p.batch * p.Hkv;
  a.Hkv = p.Hkv;
  a.S = p.S;
  a.nb_stride = p.nb_stride;
  a.budget = p.budget;
  a.force_sink = p.force_sink;
  a.force_last = p.force_last;
  a.n_keep = a.block_err ? p.n_keep : 0;
  return cuda_status(launch_select(p, a, s, pdl));
}

static qs_status do_attend(const Plan& p, const qs_cache* c, const void* q, const int32_t* sel,
                           const int32_t* n_sel, void* out, void* ws, cudaStream_t s, bool pdl,
                           const int32_t* row_lens = nullptr) {
  AttnParams a{};
  a.row_lens = row_lens;
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(c->k);
  a.v = static_cast<const uint16_t*>(c->v);
  a.sel = sel;
  a.n_sel = n_sel;
  a.page_table = c->page_table;
  a.seq_lens = c->seq_lens;
  a.part_ml = ws_at<float>(ws, p.ws.part_ml);
  a.part_o = ws_at<float>(ws, p.ws.part_o);
  a.row_ctr = ws_at<uint32_t>(ws, p.ws.row_ctr);
  a.out = out;
  a.out_bf16 = p.out_dtype == QS_BF16 ? 1 : 0;
  a.hdr = hdr_of(ws);
  a.rows = p.batch * p.Hkv;
  a.Hkv = p.Hkv;
  a.G = p.G;
  a.S = p.S;
  a.budget = p.budget;
  a.tiles_per_row = p.ws.tiles_per_row;
  a.chunk_tiles = p.ws.chunk_tiles;
  a.chunks_per_row = p.ws.chunks_per_row;
  a.gsplits = p.ws.gsplits;
  a.g_tokens_per_split = p.ws.g_tokens_per_split;
  a.max_pages_per_seq = c->max_pages_per_seq;
  a.num_pages = c->num_pages;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  if (p.key_nvfp4) {
    // NVFP4 keys: the row's kept blocks first (one CTA per row), then the attention
    a.k_codes = static_cast<const uint8_t*>(c->proxy);
    a.k_scales = c->proxy_scale;
    a.key_center = c->key_center;
    a.key_gscale = c->key_gscale;
    int32_t* kept = ws_at<int32_t>(ws, p.ws.kept);
    a.kept = kept;
    KeptParams kp{c->block_err, c->seq_lens, kept, p.batch * p.Hkv, p.Hkv, p.nb_stride,
                  p.n_keep};
    const qs_status st = cuda_status(launch_kept_blocks(kp, s, pdl));
    if (st != QS_OK) return st;
    pdl = true;
  }
  return cuda_status(launch_attn(p, a, s, pdl));
}

}  // namespace qs

using namespace qs;

extern "C" {

int32_t qs_version(void) { return 10000; }

const char* qs_status_string(qs_status s) {
  switch (s) {
    case QS_OK: return "ok";
    case QS_ERR_INVALID_ARG: return "invalid argument";
    case QS_ERR_UNSUPPORTED: return "unsupported shape or type";
    case QS_ERR_CUDA: return "CUDA error";
    case QS_ERR_DEVICE_BOUNDS: return "device-side bounds check failed";
    case QS_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

qs_status qs_workspace_size(const qs_config* cfg, int32_t batch, int32_t max_context, size_t* bytes) {
  if (!bytes) return QS_ERR_INVALID_ARG;
  Plan p;
  qs_status st = make_plan(cfg, batch, max_context, p);
  if (st != QS_OK) return st;
  *bytes = p.ws.total;
  return QS_OK;
}

qs_status qs_attention_launches(const qs_config* cfg, int32_t batch, int32_t max_context,
                                int32_t* launches) {
  Plan p;
  const qs_status st = make_plan(cfg, batch, max_context, p);
  if (st != QS_OK) return st;
  if (!launches) return QS_ERR_INVALID_ARG;
  // gather kernel: 1 (its merge is in-kernel); tile pipeline: 2 (the row merge follows),
  // 3 with NVFP4 keys (the rows' kept blocks first)
  *launches = p.attn_tma ? (p.key_nvfp4 ? 3 : 2) : 1;
  return QS_OK;
}

qs_status qs_workspace_init(void* ws, size_t ws_bytes, qs_stream_t stream) {
  if (!ws || ws_bytes < size_t(kHdrWords) * 4 || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, stream));
}

qs_status qs_append_kv(const qs_config* cfg, const qs_cache* cache, const void* k_new,
                       const void* v_new, const int32_t* n_new, int32_t max_new, const float* P,
                       int32_t batch, void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if ((st = check_cache(p, cache, true)) != QS_OK) return st;
  if (!k_new || !v_new || !n_new || max_new < 1 || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return QS_ERR_INVALID_ARG;
  if ((p.r > 0 || p.kind == PK_RABITQ) && (!P || !aligned(P, 16))) return QS_ERR_INVALID_ARG;
  if (p.kind == PK_NVFP4 && !cache->block_err) return QS_ERR_INVALID_ARG;
  return do_append(p, cache, k_new, v_new, n_new, max_new, P, nullptr, ws, stream);
}

qs_status qs_score(const qs_config* cfg, const qs_cache* cache, const void* q, const float* P,
                   int32_t batch, float* block_scores, void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if ((st = check_cache(p, cache, true)) != QS_OK) return st;
  if (!q || !aligned(q, 4) || !block_scores || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  if (p.r > 0 && (!P || !aligned(P, 16))) return QS_ERR_INVALID_ARG;
  if (p.r == 0 && !aligned(q, 16)) return QS_ERR_INVALID_ARG;
  if (p.kind == PK_RABITQ) return QS_ERR_UNSUPPORTED;     // qs_rabitq_score takes its draws
  if (p.kind == PK_SEMANTIC) return QS_ERR_UNSUPPORTED;   // qs_semantic_select scores clusters
  if (p.kind == PK_CENTROID) return do_score(p, cache, q, block_scores, ws, stream, false);
  // the prep kernel runs in stream order and writes only the query side, so the scan
  // overlaps it and starts streaming pages before it waits for the query
  if ((st = do_prep(p, q, P, ws, stream, false)) != QS_OK) return st;
  return do_score(p, cache, q, block_scores, ws, stream, true, true);
}

qs_status qs_select_topk(const qs_config* cfg, const qs_cache* cache, const float* block_scores,
                         int32_t batch, int32_t* sel, int32_t* n_sel, void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if (!cache || !cache->seq_lens) return QS_ERR_INVALID_ARG;
  if (!block_scores || !sel || !n_sel || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  if (p.kind == PK_NVFP4 && p.n_keep > 0 && !cache->block_err) return QS_ERR_INVALID_ARG;
  return do_select(p, cache, block_scores, sel, n_sel, ws, stream, false);
}

qs_status qs_sparse_attn(const qs_config* cfg, const qs_cache* cache, const void* q,
                         const int32_t* sel, const int32_t* n_sel, int32_t batch, void* out,
                         void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if ((st = check_cache(p, cache, false)) != QS_OK) return st;
  if (!q || !aligned(q, 16) || !sel || !n_sel || !out || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  return do_attend(p, cache, q, sel, n_sel, out, ws, stream, false);
}

qs_status qs_dense_workspace_size(const qs_config* cfg, int32_t batch, int32_t max_context,
                                  size_t* bytes) {
  if (!bytes) return QS_ERR_INVALID_ARG;
  Plan p;
  const qs_status st = make_dense_plan(cfg, batch, max_context, p);
  if (st != QS_OK) return st;
  *bytes = p.ws.total;
  return QS_OK;
}

qs_status qs_dense_attn(const qs_config* cfg, const qs_cache* cache, const void* q,
                        const int32_t* row_lens, int32_t batch, void* out, void* ws,
                        qs_stream_t stream) {
  Plan p;
  qs_status st = make_dense_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if ((st = check_cache(p, cache, false)) != QS_OK) return st;
  if (!q || !aligned(q, 16) || !out || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  return do_attend(p, cache, q, nullptr, nullptr, out, ws, stream, false, row_lens);
}

qs_status qs_gather_kv(const qs_config* cfg, const qs_cache* cache, const int32_t* sel,
                       const int32_t* n_sel, int32_t batch, void* k_dst, void* v_dst,
                       int32_t* row_lens, void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if ((st = check_cache(p, cache, false)) != QS_OK) return st;
  if (!sel || !n_sel || !k_dst || !v_dst || !row_lens || !ws || !aligned(ws, 256))
    return QS_ERR_INVALID_ARG;
  if (!aligned(k_dst, 16) || !aligned(v_dst, 16)) return QS_ERR_INVALID_ARG;
  GatherParams a{};
  a.k = static_cast<const uint16_t*>(cache->k);
  a.v = static_cast<const uint16_t*>(cache->v);
  a.sel = sel;
  a.n_sel = n_sel;
  a.page_table = cache->page_table;
  a.seq_lens = cache->seq_lens;
  a.k_dst = static_cast<uint16_t*>(k_dst);
  a.v_dst = static_cast<uint16_t*>(v_dst);
  a.row_lens = row_lens;
  a.hdr = hdr_of(ws);
  a.rows = p.batch * p.Hkv;
  a.Hkv = p.Hkv;
  a.log2_S = 0;
  while ((1 << a.log2_S) < p.S) ++a.log2_S;
  a.budget = p.budget;
  a.dst_pages_per_seq = (p.budget * p.S + kPage - 1) / kPage;
  a.max_pages_per_seq = cache->max_pages_per_seq;
  a.num_pages = cache->num_pages;
  return cuda_status(launch_gather_kv(p, a, stream));
}

qs_status qs_calib_workspace_size(const qs_config* cfg, size_t* bytes) {
  Plan p;
  const qs_status st = make_plan(cfg, 1, 1, p);
  if (st != QS_OK) return st;
  if (!bytes) return QS_ERR_INVALID_ARG;
  if (p.r <= 0) return QS_ERR_UNSUPPORTED;
  *bytes = calib_ws_bytes(p.Hkv, p.d);
  return QS_OK;
}

qs_status qs_calibrate_basis(const qs_config* cfg, const void* q, const void* k, int32_t n,
                             float* P, float* eigvals, void* ws, qs_stream_t stream) {
  Plan p;
  const qs_status st = make_plan(cfg, 1, 1, p);
  if (st != QS_OK) return st;
  if (p.r <= 0) return QS_ERR_UNSUPPORTED;
  if (!q || !k || n < 1 || !P || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  CalibParams a{};
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k);
  a.mq = ws_at<double>(ws, size_t(kHdrWords) * 4);
  a.mk = a.mq + size_t(p.Hkv) * p.d * p.d;
  a.P = P;
  a.eig = eigvals;
  a.n = n;
  a.Hkv = p.Hkv;
  a.G = p.G;
  a.d = p.d;
  a.r = p.r;
  return cuda_status(launch_calibrate(a, stream));
}

qs_status qs_decode(const qs_config* cfg, const qs_cache* cache, const void* q, const void* k_new,
                    const void* v_new, const float* P, int32_t batch, void* out, int32_t* sel_out,
                    int32_t* n_sel_out, void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if ((st = check_cache(p, cache, true)) != QS_OK) return st;
  if (p.kind == PK_RABITQ || p.kind == PK_SEMANTIC) return QS_ERR_UNSUPPORTED;  // own calls
  if (!q || !aligned(q, 16) || !k_new || !v_new || !out || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return QS_ERR_INVALID_ARG;
  if (p.r > 0 && (!P || !aligned(P, 16))) return QS_ERR_INVALID_ARG;
  if (p.kind == PK_NVFP4 && !cache->block_err) return QS_ERR_INVALID_ARG;
  if ((sel_out == nullptr) != (n_sel_out == nullptr)) return QS_ERR_INVALID_ARG;
  int32_t* sel = sel_out ? sel_out : ws_at<int32_t>(ws, p.ws.sel);
  int32_t* nsel = n_sel_out ? n_sel_out : ws_at<int32_t>(ws, p.ws.nsel);
  float* scores = ws_at<float>(ws, p.ws.scores);
  // append (+ fused scoring prep on the rank-r path, query packing on the NVFP4 path), then
  // the stages in stream order, each launched behind the one before
  if ((st = do_append(p, cache, k_new, v_new, nullptr, 1, P, q, ws, stream)) != QS_OK) return st;
  if (p.kind == PK_NVFP4 && (st = do_prep(p, q, P, ws, stream, true)) != QS_OK) return st;
  if ((st = do_score(p, cache, q, scores, ws, stream, true)) != QS_OK) return st;
  if ((st = do_select(p, cache, scores, sel, nsel, ws, stream, true)) != QS_OK) return st;
  return do_attend(p, cache, q, sel, nsel, out, ws, stream, true);
}

}  // extern "C"

// ------------------------------------------------------------ binary proxy (validated input)
namespace qs {

static qs_status do_rq_score(const Plan& p, const qs_cache* c, const void* q, const float* R,
                             const float* u, float* scores, void* ws, cudaStream_t s) {
  uint32_t* qcode = ws_at<uint32_t>(ws, p.ws.qt);
  RqPrepParams a{static_cast<const uint16_t*>(q), R, u, c->key_center, qcode,
                 p.batch, p.Hkv, p.G, p.d};
  const qs_status st = cuda_status(launch_rq_prep(a, s));
  if (st != QS_OK) return st;
  RqScoreParams b{};
  b.proxy = static_cast<const uint8_t*>(c->proxy);
  b.qcode = qcode;
  b.page_table = c->page_table;
  b.seq_lens = c->seq_lens;
  b.scores = scores;
  b.hdr = hdr_of(ws);
  b.batch = p.batch;
  b.Hkv = p.Hkv;
  b.d = p.d;
  b.S = p.S;
  b.nb_stride = p.nb_stride;
  b.max_pages_per_seq = c->max_pages_per_seq;
  b.num_pages = c->num_pages;
  b.max_context = c->max_context;
  b.scale = p.scale;
  return cuda_status(launch_rq_score(b, s));
}

// row_max: the rows' largest scores as recorded by the scan that wrote `scores` (the step
// call), or null (scores from the caller: the select finds them)
static qs_status do_top_p(const Plan& p, const qs_cache* c, const float* scores, float p_mass,
                          int32_t* sel, int32_t* n_sel, void* ws, cudaStream_t s,
                          const uint32_t* row_max = nullptr) {
  TopPParams a{};
  a.scores = scores;
  a.row_max = row_max;
  a.row_max_stride = kRqRowWords;
  a.seq_lens = c->seq_lens;
  a.sel = sel;
  a.n_sel = n_sel;
  a.hdr = hdr_of(ws);
  a.rows = p.batch * p.Hkv;
  a.Hkv = p.Hkv;
  a.S = p.S;
  a.nb_stride = p.nb_stride;
  a.budget = p.budget;
  a.force_sink = p.force_sink;
  a.force_last = p.force_last;
  a.p = p_mass;
  return cuda_status(launch_top_p(a, s));
}

static bool top_p_args_ok(const Plan& p, float p_mass) {
  return p_mass > 0.0f && p_mass <= 1.0f && p.budget >= p.force_sink + p.force_last;
}

}  // namespace qs

extern "C" {

qs_status qs_rabitq_score(const qs_config* cfg, const qs_cache* cache, const void* q,
                          const float* R, const float* u, int32_t batch, float* block_scores,
                          void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if (p.kind != PK_RABITQ) return QS_ERR_UNSUPPORTED;
  if ((st = check_cache(p, cache, true)) != QS_OK) return st;
  if (!q || !aligned(q, 4) || !R || !aligned(R, 16) || !u || !block_scores || !ws ||
      !aligned(ws, 256))
    return QS_ERR_INVALID_ARG;
  return do_rq_score(p, cache, q, R, u, block_scores, ws, stream);
}

qs_status qs_select_top_p(const qs_config* cfg, const qs_cache* cache, const float* block_scores,
                          float p_mass, int32_t batch, int32_t* sel, int32_t* n_sel, void* ws,
                          qs_stream_t stream) {
  Plan p;
  const qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if (!cache || !cache->seq_lens) return QS_ERR_INVALID_ARG;
  if (!block_scores || !sel || !n_sel || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  if (!top_p_args_ok(p, p_mass)) return QS_ERR_INVALID_ARG;
  return do_top_p(p, cache, block_scores, p_mass, sel, n_sel, ws, stream);
}

qs_status qs_decode_top_p(const qs_config* cfg, const qs_cache* cache, const void* q,
                          const void* k_new, const void* v_new, const float* R, const float* u,
                          float p_mass, int32_t batch, void* out, int32_t* sel_out,
                          int32_t* n_sel_out, void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if (p.kind != PK_RABITQ) return QS_ERR_UNSUPPORTED;
  if ((st = check_cache(p, cache, true)) != QS_OK) return st;
  if (!q || !aligned(q, 16) || !k_new || !v_new || !out || !ws || !aligned(ws, 256))
    return QS_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return QS_ERR_INVALID_ARG;
  if (!R || !aligned(R, 16) || !u) return QS_ERR_INVALID_ARG;
  if (!top_p_args_ok(p, p_mass)) return QS_ERR_INVALID_ARG;
  if ((sel_out == nullptr) != (n_sel_out == nullptr)) return QS_ERR_INVALID_ARG;
  int32_t* sel = sel_out ? sel_out : ws_at<int32_t>(ws, p.ws.sel);
  int32_t* nsel = n_sel_out ? n_sel_out : ws_at<int32_t>(ws, p.ws.nsel);
  float* scores = ws_at<float>(ws, p.ws.scores);
  if ((st = do_append(p, cache, k_new, v_new, nullptr, 1, R, nullptr, ws, stream)) != QS_OK)
    return st;
  if ((st = do_rq_score(p, cache, q, R, u, scores, ws, stream)) != QS_OK) return st;
  const uint32_t* row_max = ws_at<uint32_t>(ws, p.ws.qt) + kRqRowMax;
  if ((st = do_top_p(p, cache, scores, p_mass, sel, nsel, ws, stream, row_max)) != QS_OK)
    return st;
  return do_attend(p, cache, q, sel, nsel, out, ws, stream, false);
}

// ---- top-k by histogram passes (the same result as qs_select_topk)
qs_status qs_select_topk_radix(const qs_config* cfg, const qs_cache* cache,
                               const float* block_scores, int32_t batch, int32_t* sel,
                               int32_t* n_sel, void* ws, qs_stream_t stream) {
  Plan p;
  const qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if (!cache || !cache->seq_lens) return QS_ERR_INVALID_ARG;
  if (!block_scores || !sel || !n_sel || !ws || !aligned(ws, 256)) return QS_ERR_INVALID_ARG;
  if (p.kind == PK_NVFP4 && p.n_keep > 0 && !cache->block_err) return QS_ERR_INVALID_ARG;
  SelectParams a{};
  a.scores = block_scores;
  a.block_err = (p.kind == PK_NVFP4 && p.n_keep > 0) ? cache->block_err : nullptr;
  a.seq_lens = cache->seq_lens;
  a.sel = sel;
  a.n_sel = n_sel;
  a.hdr = hdr_of(ws);
  a.rows = p.batch * p.Hkv;
  a.Hkv = p.Hkv;
  a.S = p.S;
  a.nb_stride = p.nb_stride;
  a.budget = p.budget;
  a.force_sink = p.force_sink;
  a.force_last = p.force_last;
  a.n_keep = a.block_err ? p.n_keep : 0;
  return cuda_status(launch_select_radix(a, stream));
}

// ---- the NVFP4 storage variant's attended keys ("Jet-QSparse ...", Full text)
qs_status qs_gather_kv_nvfp4k(const qs_config* cfg, const qs_cache* cache, const int32_t* sel,
                              const int32_t* n_sel, int32_t batch, void* k_dst, void* v_dst,
                              int32_t* row_lens, void* ws, qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if (p.kind != PK_NVFP4) return QS_ERR_UNSUPPORTED;
  if ((st = check_cache(p, cache, true)) != QS_OK) return st;
  if (!sel || !n_sel || !k_dst || !v_dst || !row_lens || !ws || !aligned(ws, 256))
    return QS_ERR_INVALID_ARG;
  if (!aligned(k_dst, 16) || !aligned(v_dst, 16)) return QS_ERR_INVALID_ARG;
  if (p.n_keep > 0 && !cache->block_err) return QS_ERR_INVALID_ARG;
  GatherNvParams a{};
  a.base.k = static_cast<const uint16_t*>(cache->k);
  a.base.v = static_cast<const uint16_t*>(cache->v);
  a.base.sel = sel;
  a.base.n_sel = n_sel;
  a.base.page_table = cache->page_table;
  a.base.seq_lens = cache->seq_lens;
  a.base.k_dst = static_cast<uint16_t*>(k_dst);
  a.base.v_dst = static_cast<uint16_t*>(v_dst);
  a.base.row_lens = row_lens;
  a.base.hdr = hdr_of(ws);
  a.base.rows = p.batch * p.Hkv;
  a.base.Hkv = p.Hkv;
  a.base.log2_S = 7;                                  // the NVFP4 path has S = 128
  a.base.budget = p.budget;
  a.base.dst_pages_per_seq = p.budget;                // one 128-token page per block
  a.base.max_pages_per_seq = cache->max_pages_per_seq;
  a.base.num_pages = cache->num_pages;
  a.codes = static_cast<const uint8_t*>(cache->proxy);
  a.scales = cache->proxy_scale;
  a.key_center = cache->key_center;
  a.key_gscale = cache->key_gscale;
  a.block_err = p.n_keep > 0 ? cache->block_err : nullptr;
  a.nb_stride = p.nb_stride;
  a.n_keep = p.n_keep;
  return cuda_status(launch_gather_kv_nvfp4k(p, a, stream));
}

// ---- semantic blocks ("Coarse Semantic Blocks ...", Abstract)
static int sem_c_max(const Plan& p, int max_context) { return (max_context + p.S - 1) / p.S; }

static size_t sem_index_ws_bytes(const Plan& p, int max_context) {
  const size_t rows = size_t(p.batch) * p.Hkv;
  return size_t(kHdrWords) * 4 + rows * size_t(max_context) * 4 +
         rows * size_t(sem_c_max(p, max_context)) * 4;
}

qs_status qs_semantic_index_workspace_size(const qs_config* cfg, int32_t batch,
                                           int32_t max_context, size_t* bytes) {
  if (!bytes) return QS_ERR_INVALID_ARG;
  Plan p;
  const qs_status st = make_plan(cfg, batch, max_context, p);
  if (st != QS_OK) return st;
  if (p.kind != PK_SEMANTIC) return QS_ERR_UNSUPPORTED;
  *bytes = sem_index_ws_bytes(p, max_context);
  return QS_OK;
}

qs_status qs_semantic_index(const qs_config* cfg, const qs_cache* cache,
                            const int32_t* prompt_lens, int32_t iters, float* centroids,
                            int32_t* offsets, int32_t* members, int32_t batch, void* ws,
                            qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if (p.kind != PK_SEMANTIC) return QS_ERR_UNSUPPORTED;
  if ((st = check_cache(p, cache, false)) != QS_OK) return st;
  if (!prompt_lens || !centroids || !offsets || !members || !ws || !aligned(ws, 256) ||
      iters < 1)
    return QS_ERR_INVALID_ARG;
  const int l_max = cache->max_context, c_max = sem_c_max(p, l_max);
  const size_t rows = size_t(p.batch) * p.Hkv;
  SemIndexParams a{};
  a.k = static_cast<const uint16_t*>(cache->k);
  a.page_table = cache->page_table;
  a.prompt_lens = prompt_lens;
  a.cent = centroids;
  a.offsets = offsets;
  a.members = members;
  a.assign = ws_at<int32_t>(ws, size_t(kHdrWords) * 4);
  a.cursor = a.assign + rows * l_max;
  a.hdr = hdr_of(ws);
  a.batch = p.batch;
  a.Hkv = p.Hkv;
  a.d = p.d;
  a.S = p.S;
  a.c_max = c_max;
  a.l_max = l_max;
  a.max_pages_per_seq = cache->max_pages_per_seq;
  a.num_pages = cache->num_pages;
  return cuda_status(launch_sem_index(a, iters, stream));
}

qs_status qs_semantic_select(const qs_config* cfg, const qs_cache* cache, const void* q,
                             const int32_t* prompt_lens, const float* centroids,
                             const int32_t* offsets, const int32_t* members, int32_t batch,
                             int32_t* tokens, int32_t* n_tokens, int32_t max_tokens, void* ws,
                             qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if (p.kind != PK_SEMANTIC) return QS_ERR_UNSUPPORTED;
  if (!cache || !cache->seq_lens) return QS_ERR_INVALID_ARG;
  if (!q || !aligned(q, 4) || !prompt_lens || !centroids || !offsets || !members || !tokens ||
      !n_tokens || max_tokens < 1 || !ws || !aligned(ws, 256))
    return QS_ERR_INVALID_ARG;
  const int l_max = cache->max_context, c_max = sem_c_max(p, l_max);
  SemSelectParams a{};
  a.q = static_cast<const uint16_t*>(q);
  a.prompt_lens = prompt_lens;
  a.seq_lens = cache->seq_lens;
  a.cent = centroids;
  a.offsets = offsets;
  a.members = members;
  a.scores = ws_at<float>(ws, p.ws.scores);          // rows x nb_stride >= rows x c_max
  a.n_clusters = ws_at<int32_t>(ws, p.ws.qt);        // batch <= rows entries
  a.csel = ws_at<int32_t>(ws, p.ws.sel);
  a.n_csel = ws_at<int32_t>(ws, p.ws.nsel);
  a.tokens = tokens;
  a.n_tokens = n_tokens;
  a.hdr = hdr_of(ws);
  a.batch = p.batch;
  a.Hkv = p.Hkv;
  a.G = p.G;
  a.d = p.d;
  a.S = p.S;
  a.c_max = c_max;
  a.l_max = l_max;
  a.budget = p.budget;
  a.max_tokens = max_tokens;
  if ((st = cuda_status(launch_sem_score(a, stream))) != QS_OK) return st;
  // the top clusters: the select kernel over C_b candidates per row (block size 1)
  SelectParams sp{};
  sp.scores = a.scores;
  sp.block_err = nullptr;
  sp.seq_lens = a.n_clusters;
  sp.sel = ws_at<int32_t>(ws, p.ws.sel);
  sp.n_sel = ws_at<int32_t>(ws, p.ws.nsel);
  sp.hdr = a.hdr;
  sp.rows = p.batch * p.Hkv;
  sp.Hkv = p.Hkv;
  sp.S = 1;
  sp.nb_stride = c_max;
  sp.budget = p.budget;
  sp.force_sink = 0;
  sp.force_last = 0;
  sp.n_keep = 0;
  if ((st = cuda_status(launch_select(p, sp, stream, false))) != QS_OK) return st;
  return cuda_status(launch_sem_expand(a, stream));
}

qs_status qs_device_status(void* ws, qs_stream_t stream, uint32_t* detail) {
  if (!ws) return QS_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return QS_ERR_CUDA;
  uint32_t h[3] = {0, 0, 0};
  if (cudaMemcpy(h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return QS_ERR_CUDA;
  if (detail) {
    detail[0] = h[1];
    detail[1] = h[2];
  }
  if (h[0] != 0) {
    if (cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return QS_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return QS_ERR_CUDA;
  }
  return static_cast<qs_status>(h[0]);
}

}  // extern "C"
