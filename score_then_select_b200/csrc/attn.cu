// attn.cu - sparse attention over the selected blocks with its LSE combine: the tile
// pipeline for selected runs of >= 8 slots and enough work per CTA (otherwise
// attn_gather.cu).
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1 and
// Abstract: gather-free indexed attention reads the original full-dimensional keys and
// values of the selected positions straight from the standard GQA paged cache, with a
// distinct selection per KV head shared by that head's query heads.
// "Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention", Full
// text: value aggregation in FP16 with FP32 accumulation over contiguous block tiles.
//
// Full-KV attention (the dense baseline the pages compare the sparse stage with) runs the
// same kernel without a selection: every 128-token block of the row in order, optionally
// over per-row lengths (the compact buffer of gather-then-attend, gather.cu).
//
// Work decomposition (persistent grid, dynamic): a row (sequence, KV head) holds
// `tiles_per_row` 64-token tiles of selected slots, cut into chunks of `chunk_tiles` tiles;
// CTA c starts with chunks c and c + C, then claims the rest in order from a workspace
// counter, so CTAs that the memory system serves faster simply take more chunks.
//
// Warp roles (warp-specialised; no block-wide barrier in the loop):
//   * producer warp (warp 4): claims chunks ahead and resolves the chunk's runs
//     (a run is min(S, 64) slots of one selected block: lane = run) through selection
//     entry -> page table in a pipeline one chunk apart per stage; then fills one stage of
//     the shared-memory ring per tile: full and empty runs move as 64-element x run-height
//     boxes by the TMA unit (tensor maps over the K and V caches, 128-byte swizzle; empty
//     runs read zeros from outside the tensor), a ragged last block by 16-byte cp.async
//     with zero fill (counted on the stage's ragged-copy barrier), and the first tile of a
//     chunk also brings the row's queries (a bulk copy). The box and bulk copies are counted
//     on the stage's `full` barrier by their bytes; per-stage metadata carries
//     the valid-slot mask and the chunk's identity. After the last chunk it posts an end
//     marker.
//   * consumer warps (warps 0-3): each owns 16 tokens of every tile and keeps its own
//     online-softmax state (base 2, scale * log2 e folded into the logits). At the end of
//     a chunk the four states are merged in a fixed order into the chunk's partial
//     (max, sum, o).
// attn_combine_kernel, launched behind this grid, merges each (row, query head)'s chunk
// partials by log-sum-exp into the output (one CTA per row and head: the merge's L2 reads
// are spread over the whole GPU instead of adding a serial tail to one CTA's work).
//
// Tensor-core mapping and online softmax: attn_warp_tile (attn_core.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "attn_core.cuh"

namespace qs {

constexpr int kTileT = 64;
constexpr int kAttnStages = 3;
constexpr int kConsumerWarps = 4;
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kAttnThreads = kConsumerThreads + 32;
constexpr int kHalfBytes = kTileT * 128;         // 64 rows x 64 elements (one swizzled box column)

template <int D>
struct AttnSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kHalves * kHalfBytes;           // one of K or V
  static constexpr int kQBytes = (kMaxGroup * D * 2 + 1023) / 1024 * 1024;
  static constexpr int kStageBytes = 2 * kTileBytes + kQBytes;      // multiple of 1024
  static constexpr int kMetaOff = kAttnStages * kStageBytes;        // u32 [stages][4]
  static constexpr int kBarOff = kMetaOff + kAttnStages * 16;       // u64 full[], empty[], rag[]
  static constexpr int kMlOff = kBarOff + 3 * kAttnStages * 8;      // f32 [2][m [4][8], l [4][8]]
  static constexpr int kMiscOff = kMlOff + 2 * 64 * 4;              // i32 abort, u64 barrier
  static constexpr int kScrOff = kMiscOff + 16;                     // merge buffer
  static constexpr int kBufStride = D + 4;                          // floats per head (merge)
  static constexpr int kUsed = kScrOff + 2 * 8 * kBufStride * 4;
  static constexpr int kTotal = kUsed + 1024;                       // + alignment slack
};
static_assert(AttnSmem<128>::kTotal + 1024 <= 228 * 1024 / kAttnCtasPerSm,
              "kAttnCtasPerSm CTAs must fit one SM");

// Byte offset of (token row r, 16-byte chunk c) inside a K or V tile: the 128-byte
// swizzle of the TMA unit, column halves of 64 elements 8 KiB apart.
QS_DEV uint32_t swz(int r, int c) {
  return uint32_t((c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Bounded mbarrier wait that also gives up once another warp of the CTA has given up
// (`abort` set): no wait in this kernel can outlast the others.
QS_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < (1u << 22); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 63 && *abort) return false;
  }
  *abort = 1;
  return false;
}

// Per-stage metadata word 3: chunk-in-row | first-tile flag | last-tile flag | ragged-copy
// flag | phase parity of the stage's ragged-copy barrier.
constexpr uint32_t kMetaFirst = 1u << 16, kMetaLast = 1u << 17;
constexpr uint32_t kMetaRag = 1u << 18, kMetaRagPhase = 1u << 19;
// NVFP4 key storage: the tile's K region holds NVFP4 codes, scales and the row's centre
// (else BF16 keys); the tile covers page slots 64..127 (else 0..63)
constexpr uint32_t kMetaRawK = 1u << 20, kMetaHalf = 1u << 21;
// NVFP4 key storage: layout of the K region of a stage for a tile of NVFP4 keys
constexpr int kRawCodes = 0, kRawScales = 4096;
constexpr uint32_t kRawBytes = 4096 + 1024;

// Barrier of the four consumer warps on an mbarrier (count 4), bounded like every wait
// here: a warp that gives up cannot leave the others waiting on a hardware barrier.
QS_DEV void consumer_sync(uint64_t* bar, uint32_t& phase, int lane, volatile int* abort) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  wait_or_abort(bar, phase, abort);
  phase ^= 1u;
  __syncwarp();
}

// ======================= consumers: online softmax, chunk partials, row merge ==========
template <int D, bool V_F16, bool AGG_F16, bool KQ4>
QS_DEV void attn_consume(const AttnParams& a, uint8_t* smem, uint32_t* meta, uint64_t* full,
                         uint64_t* empty, uint64_t* rag, float* s_ml, volatile int* s_abort,
                         uint64_t* cbar, float* s_buf) {
  using SM = AttnSmem<D>;
  constexpr int KS = D / 16;
  constexpr int NS = kAttnStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = a.Hkv * a.G;
  const int cpr = a.chunks_per_row;
  const float gk = KQ4 ? *a.key_gscale : 0.0f;            // NVFP4 key tensor scale
  uint32_t cphase = 0, mpar = 0;
  const int h0 = 2 * (lane & 3);                           // this lane's heads h0, h0 + 1
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
  float o[KS][4];
#pragma unroll
  for (int m = 0; m < KS; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.0f;
  uint32_t qb[KS][2];
  // NVFP4 keys: q 2^-qexp as FP16 fragments, 2^qexp g_k, and q . mu of heads h0, h0 + 1
  uint32_t qh[KS][2];
  float gks = 0.0f, qmu0 = 0.0f, qmu1 = 0.0f;
  for (int t = 0;; ++t) {
    const int s = t % NS;
    if (!wait_or_abort(&full[s], (t / NS) & 1, s_abort)) break;
    const uint32_t lo = meta[4 * s], hi = meta[4 * s + 1];
    const int row = int(meta[4 * s + 2]);
    const uint32_t info = meta[4 * s + 3];
    if (row < 0 || row >= a.rows || int(info & 0xffffu) >= cpr) break;   // end marker
    if ((info & kMetaRag) && !wait_or_abort(&rag[s], (info & kMetaRagPhase) ? 1u : 0u, s_abort)) break;
    const uint8_t* st = smem + s * SM::kStageBytes;
    if (info & kMetaFirst) {
      // query fragments (B operand of S^T): head = lane/4, dims 2*(lane%4)+{0,1}
      const int h = lane >> 2;
      const uint16_t* qs = reinterpret_cast<const uint16_t*>(st + 2 * SM::kTileBytes) + h * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int d0 = ks * 16 + 2 * (lane & 3);
        qb[ks][0] = h < a.G ? *reinterpret_cast<const uint32_t*>(qs + d0) : 0u;
        qb[ks][1] = h < a.G ? *reinterpret_cast<const uint32_t*>(qs + d0 + 8) : 0u;
      }
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.0f;
#pragma unroll
      for (int m = 0; m < KS; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.0f;
      if constexpr (KQ4) {
        // q . mu of heads h0 and h0 + 1: lane slice j = lane / 4 covers dims 16j .. 16j + 15,
        // the eight slices summed by shuffles (every lane of a t = lane % 4 class agrees)
        const int j = lane >> 2;
        const float4* mu4 = reinterpret_cast<const float4*>(a.key_center + size_t(row) * D + 16 * j);
        const uint16_t* qsb = reinterpret_cast<const uint16_t*>(st + 2 * SM::kTileBytes);
        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const float4 mv = __ldg(mu4 + i4);
          const float mu[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int d = 16 * j + 4 * i4 + e;
            if (h0 < a.G) s0 = fmaf(bf16_to_f32(qsb[h0 * D + d]), mu[e], s0);
            if (h0 + 1 < a.G) s1 = fmaf(bf16_to_f32(qsb[(h0 + 1) * D + d]), mu[e], s1);
          }
        }
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) {
          s0 += __shfl_xor_sync(kFull, s0, o2);
          s1 += __shfl_xor_sync(kFull, s1, o2);
        }
        qmu0 = s0;
        qmu1 = s1;
        // qexp puts the group's largest |q| in [2^14, 2^15): every BF16 query element then
        // converts to FP16 exactly unless it is below 2^-28 of that maximum (FP16 subnormals)
        uint32_t mx = 0u;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
          mx = max(mx, max(max(qb[ks][0] & 0x7fff7fffu, qb[ks][1] & 0x7fff7fffu) >> 16,
                           max(qb[ks][0] & 0x7fffu, qb[ks][1] & 0x7fffu)));
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) mx = max(mx, __shfl_xor_sync(kFull, mx, o2));
        const int e = int(mx >> 7);                        // biased exponent of max |q|
        const int qexp = mx == 0u ? 0 : max(-60, min(100, e - 127 - 14));
        const float down = __uint_as_float(uint32_t(127 - qexp) << 23);
        gks = gk * __uint_as_float(uint32_t(127 + qexp) << 23);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
#pragma unroll
          for (int i = 0; i < 2; ++i)
            qh[ks][i] = pack_f16x2(bf16_lo(qb[ks][i]) * down, bf16_hi(qb[ks][i]) * down);
      }
    }
    const uint32_t kst = smem_u32(st), vst = smem_u32(st + SM::kTileBytes);

    const int tl = warp * 16 + (lane >> 2);       // tokens tl and tl + 8 (same 32-slot word)
    const uint32_t vm = warp < 2 ? lo : hi;
    const bool v0 = (vm >> (tl & 31)) & 1u, v1 = (vm >> ((tl + 8) & 31)) & 1u;
    const auto sw = [](int r, int c) { return swz(r, c); };
    if (KQ4 && (info & kMetaRawK)) {
      const KFragNvfp4<KS> kf(st + kRawCodes, st + kRawScales, qh, gks, qmu0, qmu1,
                              (info & kMetaHalf) ? 64 : 0, warp, lane);
      attn_warp_tile<D, V_F16, AGG_F16>(kf, vst, qb, v0, v1, a.scale_log2, m0, m1, l0, l1, o,
                                        warp, lane, sw);
    } else {
      attn_warp_tile<D, V_F16, AGG_F16>(KFragLdsm<decltype(sw)>{kst, warp, lane, sw}, vst, qb, v0,
                                        v1, a.scale_log2, m0, m1, l0, l1, o, warp, lane, sw);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);        // this warp is done with the stage
    if (!(info & kMetaLast)) continue;

    // ---------------- end of a chunk: merge the four warps (fixed order) into its partial.
    // The (max, sum) exchange alternates between two buffers so that a warp already at the
    // next chunk's end cannot overwrite what warp 0 still reads.
    float* s_m = s_ml + 64 * mpar;
    float* s_l = s_m + 32;
    mpar ^= 1;
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(kFull, l0, o2);
      l1 += __shfl_xor_sync(kFull, l1, o2);
    }
    if (lane < 4) {
      s_m[warp * 8 + h0] = m0;
      s_m[warp * 8 + h0 + 1] = m1;
    }
    consumer_sync(cbar, cphase, lane, s_abort);
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      M0 = fmaxf(M0, s_m[w * 8 + h0]);
      M1 = fmaxf(M1, s_m[w * 8 + h0 + 1]);
    }
    {
      const float f0 = ex2(m0 - (M0 == -INFINITY ? 0.0f : M0));
      const float f1 = ex2(m1 - (M1 == -INFINITY ? 0.0f : M1));
#pragma unroll
      for (int m = 0; m < KS; ++m) {
        o[m][0] *= f0;
        o[m][1] *= f1;
        o[m][2] *= f0;
        o[m][3] *= f1;
      }
      if (lane < 4) {
        s_l[warp * 8 + h0] = l0 * f0;
        s_l[warp * 8 + h0 + 1] = l1 * f1;
      }
    }
    auto park = [&](float* dst) {
#pragma unroll
      for (int m = 0; m < KS; ++m) {
        const int d0 = m * 16 + (lane >> 2);
        dst[h0 * SM::kBufStride + d0] = o[m][0];
        dst[(h0 + 1) * SM::kBufStride + d0] = o[m][1];
        dst[h0 * SM::kBufStride + d0 + 8] = o[m][2];
        dst[(h0 + 1) * SM::kBufStride + d0 + 8] = o[m][3];
      }
    };
    auto add = [&](const float* src) {
#pragma unroll
      for (int m = 0; m < KS; ++m) {
        const int d0 = m * 16 + (lane >> 2);
        o[m][0] += src[h0 * SM::kBufStride + d0];
        o[m][1] += src[(h0 + 1) * SM::kBufStride + d0];
        o[m][2] += src[h0 * SM::kBufStride + d0 + 8];
        o[m][3] += src[(h0 + 1) * SM::kBufStride + d0 + 8];
      }
    };
    float* slot0 = s_buf;
    float* slot1 = s_buf + 8 * SM::kBufStride;
    if (warp >= 2) park(warp == 2 ? slot0 : slot1);        // o2 -> slot 0, o3 -> slot 1
    consumer_sync(cbar, cphase, lane, s_abort);
    if (warp < 2) add(warp == 0 ? slot0 : slot1);          // o0 + o2, o1 + o3
    consumer_sync(cbar, cphase, lane, s_abort);
    if (warp == 1) park(slot0);
    consumer_sync(cbar, cphase, lane, s_abort);
    if (warp == 0) {
      add(slot0);                                          // (o0 + o2) + (o1 + o3)
      const int ci = int(info & 0xffffu);
      const size_t rq0 = size_t(row / a.Hkv) * Hq + (row % a.Hkv) * a.G;
      const size_t p0i = (rq0 + h0) * cpr + ci, p1i = (rq0 + h0 + 1) * cpr + ci;
#pragma unroll
      for (int m = 0; m < KS; ++m) {
        const int d0 = m * 16 + (lane >> 2);
        if (h0 < a.G) {
          __stcg(a.part_o + p0i * D + d0, o[m][0]);
          __stcg(a.part_o + p0i * D + d0 + 8, o[m][2]);
        }
        if (h0 + 1 < a.G) {
          __stcg(a.part_o + p1i * D + d0, o[m][1]);
          __stcg(a.part_o + p1i * D + d0 + 8, o[m][3]);
        }
      }
      if (lane < 4) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int h = h0 + k;
          if (h < a.G) {
            const size_t pi = (rq0 + h) * cpr + ci;
            const float M = fmaxf(fmaxf(s_m[h], s_m[8 + h]), fmaxf(s_m[16 + h], s_m[24 + h]));
            const float L = (s_l[h] + s_l[16 + h]) + (s_l[8 + h] + s_l[24 + h]);
            __stcg(a.part_ml + pi * 2, M);
            __stcg(a.part_ml + pi * 2 + 1, L);
          }
        }
      }
    }
  }
}

template <int D, bool V_F16, bool AGG_F16, bool KQ4>
__global__ void __launch_bounds__(kAttnThreads, kAttnCtasPerSm)
    attn_kernel(const __grid_constant__ AttnParams a, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v) {
  using SM = AttnSmem<D>;
  constexpr int CH = D / 8;        // 16-byte chunks per row
  constexpr int NS = kAttnStages;
  extern __shared__ uint8_t smem_raw[];
  // the swizzled boxes need 1024-byte aligned stages
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint32_t* meta = reinterpret_cast<uint32_t*>(smem + SM::kMetaOff);   // [stage][mask lo, hi, row, info]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint64_t* empty = full + NS;
  uint64_t* rag = empty + NS;       // ragged-run copies of a stage (one cp.async arrival per lane)
  float* s_ml = reinterpret_cast<float*>(smem + SM::kMlOff);         // [2][m [4][8], l [4][8]]
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + SM::kMiscOff);
  uint64_t* cbar = reinterpret_cast<uint64_t*>(smem + SM::kMiscOff + 8);
  float* s_buf = reinterpret_cast<float*>(smem + SM::kScrOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);                 // producer lane 0 (with the stage's byte count)
      mbar_init(&empty[s], kConsumerWarps);
      mbar_init(&rag[s], 32);
      meta[4 * s + 2] = 0xffffffffu;          // an unfilled stage reads as the end marker
    }
    mbar_init(cbar, kConsumerWarps);
    *s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();      // the selection comes from the kernel before
  pdl_trigger();   // the next kernel may be scheduled now; it waits for this grid to finish

  const int Hq = a.Hkv * a.G;
  const int tpr = a.tiles_per_row, cpr = a.chunks_per_row, ktiles = a.chunk_tiles;
  const int nchunks = a.rows * cpr;

  if (warp == kConsumerWarps) {
    // ======================= producer: chunk claims, run table, copies ================
    // A run is hb = min(S, 64) consecutive slots of a tile: one selected block, or one half
    // of a 128-slot block; lane u of a chunk's table holds run u (tile u / rpt, run u % rpt).
    // Three stages a chunk apart: A loads the selection entry and the row's n_sel / length;
    // B validates and loads the page-table entry; C yields the cache row of the run's first
    // slot and its valid count (0: empty; hb: full; else a ragged last block).
    const int hb = a.run_h, lg_hb = a.log2_run, rpt = kTileT >> lg_hb, lgS = a.log2_S;
    uint32_t* next_ctr = a.hdr + kCtrAttnNext;
    struct RunA { int row, sl, blk, n, L, k0, k1; };
    struct RunB { int pg, t0, g, cnt, row, raw; };
    auto stage_a = [&](int c) {
      RunA r{0, 0, -1, 0, 0, -1, -1};
      if (c < nchunks) {
        r.row = c / cpr;
        const int tin0 = (c - r.row * cpr) * ktiles, j = lane >> (6 - lg_hb);
        if (j < min(ktiles, tpr - tin0)) {
          r.sl = (tin0 + j) * kTileT + ((lane & (rpt - 1)) << lg_hb);
          r.L = a.row_lens ? a.row_lens[r.row] : a.seq_lens[r.row / a.Hkv];
          const int e = r.sl >> lgS;
          if constexpr (KQ4) {                             // the row's kept (BF16) blocks
            r.k0 = a.kept[2 * r.row];
            r.k1 = a.kept[2 * r.row + 1];
          }
          if (a.sel) {
            r.n = a.n_sel[r.row];
            if (e < a.budget) r.blk = a.sel[size_t(r.row) * a.budget + e];
          } else {                                         // full KV: every block, in order
            r.n = int((static_cast<long long>(r.L) + (1 << lgS) - 1) >> lgS);
            r.blk = e;
          }
        } else {
          r.n = -2;                                        // no such run in this chunk
        }
      }
      return r;
    };
    auto stage_b = [&](int c, const RunA& x) {
      RunB r{-1, 0, 0, 0, x.row, 0};
      if (c >= nchunks || x.n == -2) return r;
      const int b = x.row / a.Hkv;
      r.g = x.row - b * a.Hkv;
      if (x.n < 0 || x.n > a.budget || x.L < 0) {
        flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_ATTN, uint32_t(x.row));
        return r;
      }
      if (x.sl >= (x.n << lgS)) return r;                  // beyond the row's selection
      const int nbr = (x.L + (1 << lgS) - 1) >> lgS;
      if (x.blk < 0 || x.blk >= nbr) {
        flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_ATTN, uint32_t(x.row));
        return r;
      }
      r.t0 = (x.blk << lgS) + (x.sl & ((1 << lgS) - 1));
      if (r.t0 >= x.L) return r;                           // ragged tail of the last block
      r.cnt = min(hb, x.L - r.t0);
      r.raw = KQ4 && x.blk != x.k0 && x.blk != x.k1;       // keys from the NVFP4 cache
      const int pi = r.t0 >> 7;                            // kPage = 128
      r.pg = pi < a.max_pages_per_seq ? a.page_table[size_t(b) * a.max_pages_per_seq + pi] : -1;
      return r;                                            // pg is checked once it has landed
    };
    auto stage_c = [&](const RunB& x, int& y, int& cnt, int& raw) {
      cnt = x.cnt;
      y = -1;
      raw = 0;
      if (cnt == 0) return;
      if (x.pg < 0 || x.pg >= a.num_pages) {
        flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_ATTN, uint32_t(x.row));
        cnt = 0;
        return;
      }
      y = (x.pg * a.Hkv + x.g) * kPage + (x.t0 & (kPage - 1));
      raw = x.raw;
    };

    // chunks: the first two of each CTA are fixed (blockIdx, blockIdx + C), the rest are
    // claimed from the counter (value + 2C), two claims in flight, each used two chunks
    // after it is issued (an atomic on the shared counter is slow under full HBM load)
    const unsigned C2 = 2u * gridDim.x;
    unsigned pend_a = 0, pend_b = 0;
    if (lane == 0) {
      pend_a = atomicAdd(next_ctr, 1u) + C2;
      pend_b = atomicAdd(next_ctr, 1u) + C2;
    }
    int c_cur = int(min(blockIdx.x, unsigned(nchunks)));
    int c_n1 = int(min(blockIdx.x + gridDim.x, unsigned(nchunks)));
    RunA pa = stage_a(c_n1);
    RunB pb = stage_b(c_cur, stage_a(c_cur));

    const uint8_t* kbase = reinterpret_cast<const uint8_t*>(a.k);
    const uint8_t* vbase = reinterpret_cast<const uint8_t*>(a.v);
    int t = 0;                                             // stages filled so far
    int kseq = 0;                                          // chunks started by this CTA
    uint32_t rag_uses = 0;                                 // bit s: parity of stage s's ragged uses
    bool ok = true;
    while (ok && c_cur < nchunks) {
      int run_y, run_cnt, run_raw;
      stage_c(pb, run_y, run_cnt, run_raw);
      pb = stage_b(c_n1, pa);
      // the two pending claims alternate by chunk parity: neither register is touched
      // until two chunks after its atomic was issued
      int c_n2;
      if ((kseq & 1) == 0) {
        c_n2 = int(min(__shfl_sync(kFull, pend_a, 0), unsigned(nchunks)));
        if (lane == 0) pend_a = c_n2 < nchunks ? atomicAdd(next_ctr, 1u) + C2 : unsigned(nchunks);
      } else {
        c_n2 = int(min(__shfl_sync(kFull, pend_b, 0), unsigned(nchunks)));
        if (lane == 0) pend_b = c_n2 < nchunks ? atomicAdd(next_ctr, 1u) + C2 : unsigned(nchunks);
      }
      ++kseq;
      pa = stage_a(c_n2);

      const int row = c_cur / cpr, ci = c_cur - row * cpr;
      const int nt = min(ktiles, tpr - ci * ktiles);
      const int b = row / a.Hkv, g = row - b * a.Hkv;
      // per-tile summary, lane j for tile j of the chunk: valid-slot mask, box bytes,
      // whether a ragged run needs the 16-byte copy path
      uint32_t t_lo = 0, t_hi = 0, t_bytes = 0, t_rag = 0;
      for (int r = 0; r < rpt; ++r) {
        const int cr = __shfl_sync(kFull, run_cnt, ((lane << (6 - lg_hb)) + r) & 31);
        if (cr > 0) {
          const unsigned long long m = (cr >= 64 ? ~0ull : ((1ull << cr) - 1)) << (r << lg_hb);
          t_lo |= uint32_t(m);
          t_hi |= uint32_t(m >> 32);
        }
        const int rr = __shfl_sync(kFull, run_raw, ((lane << (6 - lg_hb)) + r) & 31);
        // NVFP4 keys (rr): the K box is replaced by the tile's codes, scales and centre
        if (cr == 0 || cr == hb)
          t_bytes += rr ? uint32_t(SM::kHalves * hb * 128) + kRawBytes
                        : uint32_t(2 * SM::kHalves * hb * 128);
        else {
          t_rag = 1;
          if (rr) t_bytes += kRawBytes;
        }
      }
      const uint32_t q_bytes = uint32_t(a.G * D * 2);
      const uint16_t* qrow = a.q + (size_t(b) * Hq + g * a.G) * D;
      // box copy owned by this lane: run lane / (2 halves), column half, K or V
      const int box_r = lane / (2 * SM::kHalves), box_h = (lane >> 1) % SM::kHalves, box_v = lane & 1;
      const bool box_lane = lane < rpt * SM::kHalves * 2;
      for (int j = 0; j < nt; ++j, ++t) {
        const int s = t % NS;
        bool got = true;
        if (lane == 0 && t >= NS) got = wait_or_abort(&empty[s], ((t / NS) - 1) & 1, s_abort);
        ok = __shfl_sync(kFull, got, 0);
        __syncwarp();
        if (!ok) break;

        uint8_t* st = smem + s * SM::kStageBytes;
        const uint32_t lo = __shfl_sync(kFull, t_lo, j), hi = __shfl_sync(kFull, t_hi, j);
        const uint32_t bytes = __shfl_sync(kFull, t_bytes, j) + (j == 0 ? q_bytes : 0u);
        const bool ragged = __shfl_sync(kFull, t_rag, j) != 0;
        uint32_t rag_bits = 0;
        if (ragged) {
          // a ragged run: 16-byte copies of its valid rows, zeros for the rest, counted on
          // the stage's ragged-copy barrier (its phase parity travels in the metadata)
          rag_bits = kMetaRag | ((rag_uses >> s) & 1u ? kMetaRagPhase : 0u);
          rag_uses ^= 1u << s;
          for (int r = 0; r < rpt; ++r) {
            const int src = (j << (6 - lg_hb)) + r;
            const int cr = __shfl_sync(kFull, run_cnt, src), y0 = __shfl_sync(kFull, run_y, src);
            const int rr = __shfl_sync(kFull, run_raw, src);
            if (cr == 0 || cr == hb) continue;
            for (int i = lane; i < hb; i += 32) {
              const int rt = (r << lg_hb) + i;
              const bool v = i < cr;
              const size_t off = size_t(v ? y0 + i : 0) * (D * 2);
#pragma unroll
              for (int ch = 0; ch < CH; ++ch) {
                if (!rr) cp_async16_zfill(st + swz(rt, ch), kbase + off + ch * 16, v);
                cp_async16_zfill(st + SM::kTileBytes + swz(rt, ch), vbase + off + ch * 16, v);
              }
            }
          }
          cp_async_mbar_arrive_noinc(&rag[s]);
        }
        uint32_t kq4_bits = 0;
        if constexpr (KQ4) {                               // one run per tile (S = 128)
          const int src = (j << (6 - lg_hb)) & 31;
          const int yr = __shfl_sync(kFull, run_y, src), rr = __shfl_sync(kFull, run_raw, src);
          if (rr) kq4_bits = kMetaRawK | ((yr & 64) ? kMetaHalf : 0u);
        }
        if (lane == 0) {
          meta[4 * s] = lo;
          meta[4 * s + 1] = hi;
          meta[4 * s + 2] = uint32_t(row);
          meta[4 * s + 3] = uint32_t(ci) | (j == 0 ? kMetaFirst : 0u) | (j + 1 == nt ? kMetaLast : 0u) |
                            rag_bits | kq4_bits;
          mbar_arrive_expect_tx(&full[s], bytes);
        }
        __syncwarp();                                      // the byte count is posted first
        // full and empty runs: one box copy per lane (an empty run reads zeros from outside
        // the tensor); a chunk's first tile also brings the row's queries
        {
          const int src = ((j << (6 - lg_hb)) + box_r) & 31;
          const int ry = __shfl_sync(kFull, run_y, src), rc = __shfl_sync(kFull, run_cnt, src);
          const int rr = __shfl_sync(kFull, run_raw, src);
          if (box_lane && (rc == 0 || rc == hb) && !(rr && box_v == 0)) {
            const uint32_t off = (box_v ? SM::kTileBytes : 0) + box_h * kHalfBytes + ((box_r << lg_hb) << 7);
            tma_load_2d(st + off, box_v ? static_cast<const void*>(&tm_v) : static_cast<const void*>(&tm_k),
                        64 * box_h, rc ? ry : -hb, &full[s]);
          }
          if constexpr (KQ4) {
            // NVFP4 keys, by the two K lanes: the tile's 64 token rows of each of the 4 code
            // chunks (1 KB each) and the page's 1 KB of scales
            if (rr && box_lane && box_v == 0) {
              const size_t ph = size_t(ry >> 7);             // page * Hkv + head
              const uint8_t* cb = a.k_codes + ph * kNvfp4PageCodeBytes + (ry & 127) * 16;
              const int c0 = 2 * box_h;
              bulk_g2s(st + kRawCodes + c0 * 1024, cb + c0 * 2048, 1024u, &full[s]);
              bulk_g2s(st + kRawCodes + (c0 + 1) * 1024, cb + (c0 + 1) * 2048, 1024u, &full[s]);
              if (box_h == 0)
                bulk_g2s(st + kRawScales, a.k_scales + ph * kNvfp4PageScaleBytes, 1024u, &full[s]);
            }
          }
        }
        if (j == 0 && lane == 0) bulk_g2s(st + 2 * SM::kTileBytes, qrow, q_bytes, &full[s]);
      }
      c_cur = c_n1;
      c_n1 = c_n2;
    }
    // end marker: one more stage whose row is -1
    if (ok) {
      const int s = t % NS;
      bool got = true;
      if (lane == 0 && t >= NS) got = wait_or_abort(&empty[s], ((t / NS) - 1) & 1, s_abort);
      ok = __shfl_sync(kFull, got, 0);
      __syncwarp();
      if (ok) {
        if (lane == 0) {
          meta[4 * s + 2] = 0xffffffffu;
          mbar_arrive_expect_tx(&full[s], 0u);
        }
        ++t;
      }
    }
    // every copy issued must land before the CTA exits
    cp_async_commit();
    cp_async_wait<0>();
    if (lane == 0) {
      for (int j = t > NS ? t - NS : 0; j < t; ++j)
        if (!mbar_wait(&full[j % NS], (j / NS) & 1)) *s_abort = 1;
    }
    __syncwarp();
  } else {
    attn_consume<D, V_F16, AGG_F16, KQ4>(a, smem, meta, full, empty, rag, s_ml, s_abort, cbar,
                                         s_buf);
  }
  __syncthreads();
  if (tid == 0 && *s_abort) flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_ATTN, blockIdx.x);
}


// ---------------------------------------------------------------- combine
// One CTA per (row, query head): the head's chunk partials -> output by log-sum-exp,
//   out[d] = sum_p 2^(m_p - M) o_p[d] / sum_p 2^(m_p - M) l_p  (a row with no tokens -> 0).
// Thread d owns output element d; all of its partial loads are in flight together.
// Waits for the attention grid (programmatic dependent launch), then resets the chunk
// claim counter for the next attention launch.
template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(const AttnParams a) {
  extern __shared__ float s_w[];                           // [cpr] weights, then 1/den
  pdl_wait();
  const int row = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int cpr = a.chunks_per_row;
  if (row == 0 && h == 0 && tid == 0) a.hdr[kCtrAttnNext] = 0u;
  const size_t rq = size_t(row / a.Hkv) * (a.Hkv * a.G) + (row % a.Hkv) * a.G + h;
  const float* ml = a.part_ml + rq * cpr * 2;
  if (tid < 32) {
    float M = -INFINITY;
    for (int p = lane; p < cpr; p += 32) {
      const float2 v = __ldcg(reinterpret_cast<const float2*>(ml) + p);
      if (v.y > 0.0f) M = fmaxf(M, v.x);
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o2));
    float den = 0.0f;
    for (int p = lane; p < cpr; p += 32) {
      const float2 v = __ldcg(reinterpret_cast<const float2*>(ml) + p);
      const float w = v.y > 0.0f ? ex2(v.x - M) : 0.0f;
      s_w[p] = w;
      den += w * v.y;
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) den += __shfl_xor_sync(kFull, den, o2);
    if (lane == 0) s_w[cpr] = den > 0.0f ? 1.0f / den : 0.0f;
  }
  __syncthreads();
  const float* po = a.part_o + rq * cpr * D + tid;
  float acc = 0.0f;
  int p = 0;
  for (; p + 8 <= cpr; p += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldcg(po + size_t(p + u) * D);
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += s_w[p + u] * v[u];
  }
  for (; p < cpr; ++p) acc += s_w[p] * __ldcg(po + size_t(p) * D);
  const float r = acc * s_w[cpr];
  const size_t oi = rq * D + tid;
  if (a.out_bf16)
    reinterpret_cast<uint16_t*>(a.out)[oi] = f32_to_bf16_rn(r);
  else
    reinterpret_cast<float*>(a.out)[oi] = r;
}

// ------------------------------------------------------------------ tensor maps (host)
// A 2-D map over one cache tensor viewed as [num_pages * Hkv * 128 rows][d] 16-bit
// elements; boxes of 64 elements x `box_rows` rows, 128-byte swizzle. Maps are cached by
// (address, rows, d, box_rows): encoding is a host-only call but not free.
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

static bool cache_map(const void* base, uint64_t rows, int d, int box_rows, CUtensorMap* out) {
  struct Entry { const void* base; uint64_t rows; int d, box_rows; CUtensorMap map; };
  static std::mutex mu;
  static Entry entries[16];
  static int n_entries = 0, next = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_entries; ++i) {
    const Entry& e = entries[i];
    if (e.base == base && e.rows == rows && e.d == d && e.box_rows == box_rows) {
      *out = e.map;
      return true;
    }
  }
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn || rows == 0 || rows >= (1ull << 31)) return false;
  CUtensorMap m;
  const cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(d) * 2};
  const cuuint32_t box[2] = {64u, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  if (fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  Entry& e = entries[next];
  e = Entry{base, rows, d, box_rows, m};
  next = (next + 1) % 16;
  if (n_entries < 16) ++n_entries;
  *out = m;
  return true;
}

template <int D, bool VF, bool AF, bool KQ4 = false>
static cudaError_t launch_attn_t(const AttnParams& a, const CUtensorMap& mk, const CUtensorMap& mv,
                                 int grid, cudaStream_t s, bool pdl) {
  auto k = attn_kernel<D, VF, AF, KQ4>;
  const int smem = AttnSmem<D>::kTotal;
  const cudaError_t attr = set_smem_limit(k, smem);
  if (attr != cudaSuccess) return attr;
  cudaError_t e = launch_k(k, dim3(grid), dim3(kAttnThreads), smem, s, pdl, a, mk, mv);
  if (e != cudaSuccess) return e;
  // the row merge, launched behind the attention grid (it waits for it before reading)
  const size_t csmem = size_t(a.chunks_per_row + 1) * sizeof(float);
  return launch_k(attn_combine_kernel<D>, dim3(a.rows, a.G), dim3(D), csmem, s, true, a);
}

cudaError_t launch_attn(const Plan& p, const AttnParams& a_in, cudaStream_t s, bool pdl) {
  if (!p.attn_tma) return launch_attn_gather(p, a_in, s, pdl);
  AttnParams a = a_in;
  a.run_h = p.S < kTileT ? p.S : kTileT;
  a.log2_S = 0;
  while ((1 << a.log2_S) < p.S) ++a.log2_S;
  a.log2_run = a.log2_S < 6 ? a.log2_S : 6;
  CUtensorMap mk, mv;
  std::memset(&mk, 0, sizeof(mk));
  std::memset(&mv, 0, sizeof(mv));
  const uint64_t rows = uint64_t(a.num_pages) * a.Hkv * kPage;
  if (!cache_map(a.k, rows, p.d, a.run_h, &mk) || !cache_map(a.v, rows, p.d, a.run_h, &mv))
    return cudaErrorNotSupported;
  const bool vf = p.v_dtype == QS_F16, af = p.v_agg_dtype == QS_F16;
  const int grid = p.ws.attn_ctas;
  if (p.key_nvfp4) {                  // NVFP4 keys: d = 128, V and P.V in FP16
    if (p.d != 128 || !vf) return cudaErrorInvalidValue;
    return launch_attn_t<128, true, true, true>(a, mk, mv, grid, s, pdl);
  }
  if (p.d == 128) {
    if (vf) return launch_attn_t<128, true, true>(a, mk, mv, grid, s, pdl);
    if (af) return launch_attn_t<128, false, true>(a, mk, mv, grid, s, pdl);
    return launch_attn_t<128, false, false>(a, mk, mv, grid, s, pdl);
  }
  if (p.d == 64) {
    if (vf) return launch_attn_t<64, true, true>(a, mk, mv, grid, s, pdl);
    if (af) return launch_attn_t<64, false, true>(a, mk, mv, grid, s, pdl);
    return launch_attn_t<64, false, false>(a, mk, mv, grid, s, pdl);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qs
