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
//               shared-memory ring (mbarrier transaction counts);
//   warp 1      one lane copies the stage's scale factors to tensor memory
//               (tcgen05.cp 32x128b.warpx4), issues the two MMAs into the stage's
//               accumulator columns and commits them to an mbarrier;
//   warps 2..9  two groups of four alternate over the units: each reads the 128 x 8
//               accumulator (tcgen05.ld, each warp its 32 lanes), takes the max over
//               heads and tokens, and releases the stage.
// Shared-memory stages are released by the MMA commit itself; accumulator slots are
// released by the epilogue, so the epilogue stays off the memory pipeline.
// The page layouts written by the NVFP4 writer make each copy land directly in the
// K-major, no-swizzle operand layout (see qs_internal.h).
#include "qs_device.cuh"

namespace qs {

// Several CTAs share an SM (one CTA's serial issue loop cannot stream an SM's share of
// HBM bandwidth): each holds a power-of-two share of the 512 tensor-memory columns and
// sizes its shared-memory ring so that exactly that many CTAs fit on an SM.
constexpr int kF4CtasPerSm = 3;
template <int K> struct F4Cfg;
template <> struct F4Cfg<2> { static constexpr int NS = 11, ND = 12; static constexpr uint32_t COLS = 256; };
template <> struct F4Cfg<3> { static constexpr int NS = 7, ND = 6; static constexpr uint32_t COLS = 128; };
template <> struct F4Cfg<4> { static constexpr int NS = 5, ND = 6; static constexpr uint32_t COLS = 128; };
constexpr int kF4Stages = F4Cfg<kF4CtasPerSm>::NS;   // shared-memory ring: page codes + scales
constexpr int kF4DStages = F4Cfg<kF4CtasPerSm>::ND;  // tensor-memory ring: accumulator + A scales
constexpr int kF4EpiGroups = 2;                 // 4-warp epilogue groups, alternate units
constexpr int kF4Threads = 32 * (2 + 4 * kF4EpiGroups);
constexpr int kF4CodeOff = 0;
constexpr int kF4ScaleOff = kNvfp4PageCodeBytes;                       // 8192
constexpr int kF4SlotBytes = kF4ScaleOff + kNvfp4PageScaleBytes;       // 9216
constexpr uint32_t kF4TmemCols = F4Cfg<kF4CtasPerSm>::COLS;
// TMEM: accumulator of D-stage d: columns [8d, 8d+8); A scales of D-stage d: 8 ND + 8d +
// {kb0, kb1} = +{0, 4}; the current row's B scales: 16 ND + {0, 4}
constexpr uint32_t kF4SfaBase = 8 * kF4DStages;
constexpr uint32_t kF4SfbBase = kF4SfaBase + 8 * kF4DStages;
static_assert(kF4SfbBase + 8 <= kF4TmemCols, "tensor-memory plan exceeds the allocation");
static_assert(kF4DStages % kF4EpiGroups == 0, "a D-stage must always go to the same group");
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
  constexpr int NS = kF4Stages, ND = kF4DStages;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* slots = smem;                                          // [NS][9216]
  uint8_t* btile = smem + NS * kF4SlotBytes;                      // [kQTileBytes] current row
  uint64_t* full = reinterpret_cast<uint64_t*>(btile + kQTileBytes);
  uint64_t* empty = full + NS;        // smem stage free: committed by the MMA lane
  uint64_t* dfull = empty + NS;       // accumulator ready: committed by the MMA lane
  uint64_t* dfree = dfull + ND;       // accumulator read: 4 epilogue warps
  uint64_t* rfull = dfree + ND;       // the 4 warp maxima written: 4 epilogue warps
  uint64_t* bbar = rfull + ND;        // [0] B tile landed, [1] MMAs drained
  int4* info = reinterpret_cast<int4*>(bbar + 2);                 // [NS] unit of a smem stage
  int4* dinfo = info + NS;                                        // [ND] unit of a TMEM slot
  float* red = reinterpret_cast<float*>(dinfo + ND);              // [ND][4]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(red + ND * 4);
  int* prefix = reinterpret_cast<int*>(s_tmem + 4);               // [batch + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (!a.early_stream) pdl_wait();   // query tiles, g_q and seq_lens: the kernels before
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int d = 0; d < ND; ++d) {
      mbar_init(&dfull[d], 2);     // the MMA lane's arrive (unit info) + its MMA commit
      mbar_init(&dfree[d], 4);
      mbar_init(&rfull[d], 4);
    }
    mbar_init(&bbar[0], 1);
    mbar_init(&bbar[1], 1);
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
    // ---------------- producer: 32 lanes resolve 32 units, lane 0 streams their pages
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
          const int s = k % NS;
          const uint32_t ph = uint32_t(k / NS) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) {
            flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
            dead = true;
          } else {
            info[s] = make_int4(jrow, jp, jnv, jok);
            uint8_t* slot = slots + s * kF4SlotBytes;
            if (jok) {
              const size_t ph_idx = size_t(jpage) * a.Hkv + (jrow % a.Hkv);
              mbar_arrive_expect_tx(&full[s], uint32_t(kF4SlotBytes));
              bulk_g2s(slot + kF4CodeOff,
                       reinterpret_cast<const uint8_t*>(a.proxy) + ph_idx * kNvfp4PageCodeBytes,
                       kNvfp4PageCodeBytes, &full[s]);
              bulk_g2s(slot + kF4ScaleOff, a.proxy_scale + ph_idx * kNvfp4PageScaleBytes,
                       kNvfp4PageScaleBytes, &full[s]);
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
    if (a.early_stream) pdl_wait();   // the query tiles come from the kernel before
    if (lane == 0) {
      int cur_row = -1;
      uint32_t bph0 = 0, bph1 = 0;     // parities of the B-tile and drain barriers
      bool issued = false;
      for (int k = 0; k < n_units; ++k) {
        const int s = k % NS, d = k % ND;
        if (!mbar_wait(&full[s], uint32_t(k / NS) & 1u)) {
          flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
          break;
        }
        const int row = info[s].x;
        if (row != cur_row) {
          // a new row: let every MMA on the old B tile finish, then load the row's tile
          // (B codes + B scales) and copy its scales to tensor memory
          bool ok = true;
          if (issued) {
            tc_commit(&bbar[1]);
            ok = mbar_wait(&bbar[1], bph1);
            bph1 ^= 1u;
          }
          if (ok) {
            mbar_arrive_expect_tx(&bbar[0], uint32_t(kQTileBytes));
            bulk_g2s(btile, a.qtile + size_t(row) * kQTileBytes, kQTileBytes, &bbar[0]);
            ok = mbar_wait(&bbar[0], bph0);
            bph0 ^= 1u;
          }
          if (!ok) {
            flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
            break;
          }
          tc_fence_after();
          tc_cp_32x128b_x4(tbase + kF4SfbBase + 0, smem_desc_kmajor(btile + 512, 128, 128));
          tc_cp_32x128b_x4(tbase + kF4SfbBase + 4, smem_desc_kmajor(btile + 1024, 128, 128));
          cur_row = row;
        }
        // the accumulator (and A-scale) slot d was read by the epilogue for unit k - ND
        if (!mbar_wait(&dfree[d], (uint32_t(k / ND) & 1u) ^ 1u)) {
          flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
          break;
        }
        tc_fence_after();
        dinfo[d] = info[s];          // published to the epilogue by this plain arrive
        mbar_arrive(&dfull[d]);
        const uint8_t* slot = slots + s * kF4SlotBytes;
        const uint32_t sfa = tbase + kF4SfaBase + 8u * d;
        // A scales: 32 rows x 16 bytes each, 8-row core matrices 128 bytes apart
        tc_cp_32x128b_x4(sfa + 0, smem_desc_kmajor(slot + kF4ScaleOff, 128, 128));
        tc_cp_32x128b_x4(sfa + 4, smem_desc_kmajor(slot + kF4ScaleOff + 512, 128, 128));
        const uint32_t dt = tbase + 8u * d;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          // A: 128 tokens x 32 bytes: chunks 2kb, 2kb+1 (2048 bytes apart), 8-token groups
          // 128 bytes apart; B: 8 heads x 32 bytes: chunks 128 bytes apart
          const uint64_t adesc = smem_desc_kmajor(slot + kF4CodeOff + kb * 4096, 2048, 128);
          const uint64_t bdesc = smem_desc_kmajor(btile + kb * 256, 128, 512);
          tc_mma_nvf4(dt, adesc, bdesc, kF4Idesc, sfa + 4u * kb, tbase + kF4SfbBase + 4u * kb,
                      kb > 0);
        }
        tc_commit(&empty[s]);      // the page's shared memory is free once the MMAs are done
        tc_commit(&dfull[d]);
        issued = true;
      }
      // let the MMAs issued so far finish before tensor memory is released
      if (issued) {
        tc_commit(&bbar[1]);
        mbar_wait(&bbar[1], bph1, 1u << 20);
      }
    }
  } else {
    // ---------------- epilogue groups: group eg takes units k = eg, eg + 2, ...; a warp
    // reads TMEM lanes 32*(warp%4) .. +31 = 32 of the unit's tokens
    const int eg = (warp - 2) >> 2;
    const int q = warp & 3;
    const bool leader = ((warp - 2) & 3) == 0;       // first warp of its group
    if (a.early_stream) pdl_wait();                   // g_q comes from the kernel before
    const float gscale = __fmul_rn(*a.qgscale, *a.key_gscale);
    const uint32_t lane_addr = uint32_t(32 * q) << 16;
    for (int k = eg; k < n_units; k += kF4EpiGroups) {
      const int d = k % ND;
      const uint32_t dph = uint32_t(k / ND) & 1u;
      if (!mbar_wait(&dfull[d], dph)) {
        if (lane == 0) flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
        break;
      }
      tc_fence_after();
      const int4 x = dinfo[d];         // {row, page index in row, valid tokens, ok}
      uint32_t r[8];
      tc_ld_32x32b_x8(tbase + lane_addr + 8u * d, r);
      tc_fence_before();
      const int tok = 32 * q + lane;
      float v = -INFINITY;
      if (x.w && tok < x.z) {
#pragma unroll
        for (int n = 0; n < 8; ++n)
          if (n < a.G) v = fmaxf(v, __uint_as_float(r[n]));
        v *= gscale;
      }
      v = warp_max(v);
      if (lane == 0) {
        red[d * 4 + q] = v;
        mbar_arrive(&rfull[d]);
        if (leader) {
          // the group's four warp maxima -> the block score (one 128-token block per page)
          if (!mbar_wait(&rfull[d], dph)) {
            flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
          } else if (x.w) {
            const float mx = fmaxf(fmaxf(red[d * 4 + 0], red[d * 4 + 1]),
                                   fmaxf(red[d * 4 + 2], red[d * 4 + 3]));
            a.scores[size_t(x.x) * a.nb_stride + x.y] = mx;
          }
        }
        // slot d (accumulator, A scales, dinfo, red) may be reused once all four warps
        // are past it; the leader only after reading the maxima
        mbar_arrive(&dfree[d]);
      }
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kF4TmemCols);
}

cudaError_t launch_score_nvfp4(const Plan& p, const ScoreParams& a, cudaStream_t s, bool pdl) {
  const size_t smem_max = size_t(kF4Stages) * kF4SlotBytes + kQTileBytes +
                          (2 * kF4Stages + 3 * kF4DStages + 2) * sizeof(uint64_t) +
                          (kF4Stages + kF4DStages) * sizeof(int4) +
                          kF4DStages * 4 * sizeof(float) + 16 +
                          size_t(kMaxBatch + 1) * sizeof(int);
  const size_t smem = smem_max - size_t(kMaxBatch - a.batch) * sizeof(int);
  auto k = score_nvfp4_kernel;
  const cudaError_t attr = set_smem_limit(k, int(smem_max));
  if (attr != cudaSuccess) return attr;
  // kF4CtasPerSm CTAs per SM, each with its share of the SM's tensor memory
  const long long units = (long long)a.batch * a.Hkv * ((a.max_context + kPage - 1) / kPage);
  long long grid = (long long)num_sms() * kF4CtasPerSm;
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  return launch_k(k, dim3(unsigned(grid)), dim3(kF4Threads), smem, s, pdl, a);
}

}  // namespace qs
