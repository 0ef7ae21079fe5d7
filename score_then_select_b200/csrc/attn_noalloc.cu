// attn_noalloc.cu - sparse attention for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a plugin of a host framework that owns all device
// memory and passes its kernels only their inputs and outputs, or a decode loop that must
// not allocate because cudaMalloc may synchronise the device. qs_sparse_attn_noalloc runs
// the same attention kernel as qs_sparse_attn, with its scratch (split partials and the
// per-row split counters) in one file-scope static device array instead of a
// caller-provided workspace. The array is 4 MiB; every GPU that loads the library holds
// it until the process exits. All calls on a device share it, so calls that overlap on
// the GPU race.
#include <mutex>

#include "qs_device.cuh"

namespace qs {

constexpr size_t kStaticScratch = QS_ATTN_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t qs_attn_scratch[kStaticScratch];

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu;
static void* g_scratch_ptr[kMaxDevices];   // device address of qs_attn_scratch, per device

// Once per device, with that device current: look up the array's device address. In host
// code the symbol name is only a host-side stand-in, never a device address.
static qs_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, qs_attn_scratch) != cudaSuccess || p == nullptr)
      return QS_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return QS_OK;
}

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace qs

using namespace qs;

extern "C" qs_status qs_sparse_attn_noalloc(const qs_config* cfg, const qs_cache* cache,
                                            const void* q, const int32_t* sel,
                                            const int32_t* n_sel, int32_t batch, void* out,
                                            qs_stream_t stream) {
  Plan p;
  qs_status st = make_plan(cfg, batch, cache ? cache->max_context : 0, p);
  if (st != QS_OK) return st;
  if ((st = check_cache(p, cache, false)) != QS_OK) return st;
  if (p.key_nvfp4) return QS_ERR_UNSUPPORTED;      // its kept blocks live in a workspace
  if (!q || (reinterpret_cast<uintptr_t>(q) & 15) || !sel || !n_sel || !out) return QS_ERR_INVALID_ARG;
  // carve the static array: status header | row counters | partial (m, l) | partial o
  const size_t rows = size_t(batch) * p.Hkv, rows_q = size_t(batch) * p.Hq;
  const size_t hdr_bytes = size_t(kHdrWords) * 4;
  const size_t ctr_off = hdr_bytes;
  const size_t ml_off = up256(ctr_off + rows * 4);
  const size_t o_off = up256(ml_off + rows_q * p.ws.parts_per_head * 2 * 4);
  const size_t need = o_off + rows_q * p.ws.parts_per_head * p.d * 4;
  if (need > kStaticScratch) return QS_ERR_UNSUPPORTED;
  void* base = nullptr;
  if ((st = scratch_address(&base)) != QS_OK) return st;
  uint8_t* s8 = static_cast<uint8_t*>(base);
  // the counters and the status word must start at zero for every call
  if (cudaMemsetAsync(s8, 0, ml_off, stream) != cudaSuccess) return QS_ERR_CUDA;

  AttnParams a{};
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(cache->k);
  a.v = static_cast<const uint16_t*>(cache->v);
  a.sel = sel;
  a.n_sel = n_sel;
  a.page_table = cache->page_table;
  a.seq_lens = cache->seq_lens;
  a.part_ml = reinterpret_cast<float*>(s8 + ml_off);
  a.part_o = reinterpret_cast<float*>(s8 + o_off);
  a.row_ctr = reinterpret_cast<uint32_t*>(s8 + ctr_off);
  a.out = out;
  a.out_bf16 = p.out_dtype == QS_BF16 ? 1 : 0;
  a.hdr = reinterpret_cast<uint32_t*>(s8);
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
  a.max_pages_per_seq = cache->max_pages_per_seq;
  a.num_pages = cache->num_pages;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  return launch_attn(p, a, stream, false) == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}
