// score_nvfp4.cu - proxy block scores by a dense FP4 scan of the NVFP4 key cache.
//
// "Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention", Full
// text: the centred keys are stored as NVFP4 and a dense scan scores the whole key history
// with native FP4 query-key products on Blackwell tensor cores; 128-token blocks are then
// selected. Per head h of the row's group and token t,
//   s[h,t] = g_q g_k sum_c sq[h,c] sk[t,c] sum_i eq[h,16c+i] ek[t,16c+i]      (FP32 accumulate)
// and a block's score is the maximum over the group's heads and the block's valid tokens.
//
// One (sequence, KV head, page) unit is one 128-token block: it is the M = 128 side of a
// block-scaled FP4 MMA (tcgen05.mma kind::mxf4nvf4, UE4M3 scale per 16 elements), the
// group's <= 8 heads are the N = 8 side, and K = 128 takes two MMAs of K = 64. The
// per-unit work is tiny next to its 9 KiB of HBM traffic, so the kernel is a bandwidth
// pipeline around the tensor cores:
//   warp 0      one lane streams each unit's page codes (8 KiB), page scales (1 KiB) and
//               the row's query tile (1.5 KiB, L2-resident) with bulk TMA copies into a
//               4-stage shared-memory ring (mbarrier transaction counts);
//   warp 1      one lane copies the stage's scale factors to tensor memory
//               (tcgen05.cp 32x128b.warpx4), issues the two MMAs into the stage's
//               accumulator columns and commits them to an mbarrier;
//   warps 2..5  read the 128 x 8 accumulator (tcgen05.ld, each warp its 32 lanes), take
//               the max over heads and tokens, and release the stage.
// The page layouts written by the NVFP4 writer make each copy land directly in the
// K-major, no-swizzle operand layout (see qs_internal.h).
#include "qs_device.cuh"

namespace qs {

constexpr int kF4Stages = 4;
constexpr int kF4Threads = 32 * 6;
constexpr int kF4CodeOff = 0;
constexpr int kF4ScaleOff = kNvfp4PageCodeBytes;                       // 8192
constexpr int kF4QCodeOff = kF4ScaleOff + kNvfp4PageScaleBytes;        // 9216
constexpr int kF4QScaleOff = kF4QCodeOff + 512;                        // 9728
constexpr int kF4SlotBytes = kF4QCodeOff + kQTileBytes;                // 10752
constexpr uint32_t kF4TmemCols = 128;
// accumulator of stage s: columns [8s, 8s+8); scale factors of stage s: 32 + 16s + {A kb0,
// A kb1, B kb0, B kb1} = +{0, 4, 8, 12}
constexpr uint32_t kF4SfBase = 32;
// instruction descriptor: A and B E2M1 (1), UE4M3 scales (0), both K-major, N = 8
// (n_dim = N >> 3 at bit 17), M = 128 (m_dim = M >> 4 at bit 24), dense K = 64
constexpr uint32_t kF4Idesc = (1u << 7) | (1u << 10) | (1u << 17) | (8u << 24);

struct F4Unit {
  int row, p, nv, page;
  bool ok;
};

// unit index -> (row, page index, valid tokens, physical page); lengths clamped
QS_DEV F4Unit f4_unit(const ScoreParams& a, const int* prefix, int u, int& b) {
  while (u >= prefix[b + 1]) ++b;
  F4Unit x;
  const int np = (prefix[b + 1] - prefix[b]) / a.Hkv;
  const int off = u - prefix[b];
  const int g = off / np;
  x.p = off % np;
  x.row = b * a.Hkv + g;
  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.max_context ? a.max_context : L);
  x.nv = min(kPage, L - x.p * kPage);
  x.ok = x.p < a.max_pages_per_seq;
  x.page = x.ok ? a.page_table[size_t(b) * a.max_pages_per_seq + x.p] : -1;
  x.ok = x.ok && x.page >= 0 && x.page < a.num_pages;
  return x;
}

QS_DEV void f4_prefix(const ScoreParams& a, int* prefix) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int carry = 0;
    if (lane == 0) prefix[0] = 0;
    for (int base = 0; base < a.batch; base += 32) {
      const int b = base + lane;
      int u = 0;
      if (b < a.batch) {
        int L = a.seq_lens[b];
        if (L < 0 || L > a.max_context) {
          flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(b));
          L = L < 0 ? 0 : a.max_context;
        }
        u = a.Hkv * ((L + kPage - 1) / kPage);
      }
      int x = u;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
      }
      if (b < a.batch) prefix[b + 1] = carry + x;
      carry += __shfl_sync(kFull, x, 31);
    }
  }
}

__global__ void __launch_bounds__(kF4Threads) score_nvfp4_kernel(const ScoreParams a) {
  constexpr int NST = kF4Stages;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* slots = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NST * kF4SlotBytes);
  uint64_t* empty = full + NST;
  uint64_t* dfull = empty + NST;
  uint64_t* rfull = dfull + NST;                                  // 4 warp maxima written
  int4* info = reinterpret_cast<int4*>(rfull + NST);
  float* red = reinterpret_cast<float*>(info + NST);              // [NST][4]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(red + NST * 4);
  int* prefix = reinterpret_cast<int*>(s_tmem + 4);               // [batch + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();      // the query tiles, g_q and seq_lens come from the kernels before
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);     // one arrival per epilogue warp
      mbar_init(&dfull[s], 1);     // one tcgen05.commit per unit
      mbar_init(&rfull[s], 4);     // one arrival per epilogue warp
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kF4TmemCols);
    tmem_relinquish();
  }
  f4_prefix(a, prefix);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *s_tmem;

  const long long U = prefix[a.batch];
  const int u0 = int(U * blockIdx.x / gridDim.x);
  const int u1 = int(U * (blockIdx.x + 1) / gridDim.x);
  const int n_units = u1 - u0;

  if (warp == 0) {
    // ---------------- producer: 32 lanes resolve 32 units, lane 0 issues their copies
    int b = 0;
    bool dead = false;
    for (int k0 = 0; k0 < n_units && !dead; k0 += 32) {
      F4Unit x{};
      x.ok = false;
      if (k0 + lane < n_units) x = f4_unit(a, prefix, u0 + k0 + lane, b);
      const int m = min(32, n_units - k0);
      for (int j = 0; j < m; ++j) {
        const int jrow = __shfl_sync(kFull, x.row, j);
        const int jp = __shfl_sync(kFull, x.p, j);
        const int jnv = __shfl_sync(kFull, x.nv, j);
        const int jok = __shfl_sync(kFull, int(x.ok), j);
        const int jpage = __shfl_sync(kFull, x.page, j);
        if (lane == 0) {
          const int k = k0 + j;
          const int s = k % NST;
          const uint32_t ph = uint32_t(k / NST) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) {
            flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
            dead = true;
          } else {
            info[s] = make_int4(jrow, jp, jnv, jok);
            uint8_t* slot = slots + s * kF4SlotBytes;
            if (jok) {
              const int g = jrow % a.Hkv;
              const size_t ph_idx = size_t(jpage) * a.Hkv + g;
              mbar_arrive_expect_tx(&full[s], uint32_t(kF4SlotBytes));
              bulk_g2s(slot + kF4CodeOff,
                       reinterpret_cast<const uint8_t*>(a.proxy) + ph_idx * kNvfp4PageCodeBytes,
                       kNvfp4PageCodeBytes, &full[s]);
              bulk_g2s(slot + kF4ScaleOff, a.proxy_scale + ph_idx * kNvfp4PageScaleBytes,
                       kNvfp4PageScaleBytes, &full[s]);
              bulk_g2s(slot + kF4QCodeOff, a.qtile + size_t(jrow) * kQTileBytes, kQTileBytes,
                       &full[s]);
            } else {
              flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(jrow));
              mbar_arrive(&full[s]);
            }
          }
        }
        dead = __shfl_sync(kFull, int(dead), 0) != 0;
        if (dead) break;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one lane)
    if (lane == 0) {
      int last = -1;
      for (int k = 0; k < n_units; ++k) {
        const int s = k % NST;
        const uint32_t ph = uint32_t(k / NST) & 1u;
        if (!mbar_wait(&full[s], ph)) {
          flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
          break;
        }
        tc_fence_after();
        const uint8_t* slot = slots + s * kF4SlotBytes;
        const uint32_t sf = tbase + kF4SfBase + 16u * s;
        // scale factors: 32 rows x 16 bytes each, 8-row core matrices 128 bytes apart
        tc_cp_32x128b_x4(sf + 0, smem_desc_kmajor(slot + kF4ScaleOff, 128, 128));
        tc_cp_32x128b_x4(sf + 4, smem_desc_kmajor(slot + kF4ScaleOff + 512, 128, 128));
        tc_cp_32x128b_x4(sf + 8, smem_desc_kmajor(slot + kF4QScaleOff, 128, 128));
        tc_cp_32x128b_x4(sf + 12, smem_desc_kmajor(slot + kF4QScaleOff + 512, 128, 128));
        const uint32_t d = tbase + 8u * s;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          // A: 128 tokens x 32 bytes: chunks 2kb, 2kb+1 (2048 bytes apart), 8-token groups
          // 128 bytes apart; B: 8 heads x 32 bytes: chunks 128 bytes apart
          const uint64_t adesc = smem_desc_kmajor(slot + kF4CodeOff + kb * 4096, 2048, 128);
          const uint64_t bdesc = smem_desc_kmajor(slot + kF4QCodeOff + kb * 256, 128, 512);
          tc_mma_nvf4(d, adesc, bdesc, kF4Idesc, sf + 4u * kb, sf + 8u + 4u * kb, kb > 0);
        }
        tc_commit(&dfull[s]);
        last = k;
      }
      // after a timeout, let the MMAs already issued finish before TMEM is released
      if (last >= 0 && last + 1 < n_units) {
        const int s = last % NST;
        mbar_wait(&dfull[s], uint32_t(last / NST) & 1u, 1u << 16);
      }
    }
  } else {
    // ---------------- epilogue warps: TMEM lanes 32*(warp%4) .. +31 = the unit's tokens
    const int q = warp & 3;
    const float gscale = __fmul_rn(*a.qgscale, *a.key_gscale);
    const uint32_t lane_addr = uint32_t(32 * q) << 16;
    for (int k = 0; k < n_units; ++k) {
      const int s = k % NST;
      const uint32_t ph = uint32_t(k / NST) & 1u;
      if (!mbar_wait(&dfull[s], ph)) {
        if (lane == 0) flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
        break;
      }
      tc_fence_after();
      const int4 x = info[s];
      uint32_t r[8];
      tc_ld_32x32b_x8(tbase + lane_addr + 8u * s, r);
      const int tok = 32 * q + lane;
      float v = -INFINITY;
      if (x.w && tok < x.z) {
#pragma unroll
        for (int n = 0; n < 8; ++n)
          if (n < a.G) v = fmaxf(v, __uint_as_float(r[n]));
        v *= gscale;
      }
      v = warp_max(v);
      tc_fence_before();
      if (lane == 0) {
        red[s * 4 + q] = v;
        mbar_arrive(&rfull[s]);
      }
      if (warp == 2 && lane == 0) {
        // the four warps' maxima -> the block score (one 128-token block per page)
        if (!mbar_wait(&rfull[s], ph)) {
          flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
        } else if (x.w) {
          const float m = fmaxf(fmaxf(red[s * 4 + 0], red[s * 4 + 1]),
                                fmaxf(red[s * 4 + 2], red[s * 4 + 3]));
          a.scores[size_t(x.x) * a.nb_stride + x.y] = m;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kF4TmemCols);
}

cudaError_t launch_score_nvfp4(const Plan& p, const ScoreParams& a, cudaStream_t s, bool pdl) {
  const size_t smem_max = size_t(kF4Stages) * kF4SlotBytes + 4 * kF4Stages * sizeof(uint64_t) +
                          kF4Stages * sizeof(int4) + kF4Stages * 4 * sizeof(float) + 16 +
                          size_t(kMaxBatch + 1) * sizeof(int);
  const size_t smem = smem_max - size_t(kMaxBatch - a.batch) * sizeof(int);
  auto k = score_nvfp4_kernel;
  static int per_sm = [&] {
    int n = 0;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max)) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kF4Threads, smem_max) != cudaSuccess)
      n = 0;
    return n;
  }();
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  // tensor memory: 512 columns per SM, kF4TmemCols per CTA
  const int resident = per_sm < int(512 / kF4TmemCols) ? per_sm : int(512 / kF4TmemCols);
  const long long units = (long long)a.batch * a.Hkv * ((a.max_context + kPage - 1) / kPage);
  long long grid = (long long)num_sms() * resident;
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  return launch_k(k, dim3(unsigned(grid)), dim3(kF4Threads), smem, s, pdl, a);
}

}  // namespace qs
