// score.cu - proxy block scores on the projected-key cache (the rank-r path).
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1: the
// mean of a KV head's query heads, projected into the shared subspace (q~ = qbar . P),
// scores every cached projected key; Figure 9 names this "candidate scoring" and the q~
// computation "scoring preparation". Each block of S tokens is reduced to the maximum of
// its valid tokens' scores (the reading taken for block selection, "Jet-QSparse",
// Full text, which selects 128-token blocks from a dense scan).
//
// The scan is bound by HBM bandwidth (r, 2r or 4r bytes and 2r flops per token for an FP8,
// BF16 or FP32 cache; "Joint Subspace Sparse Attention ...", Figure 10, keeps the
// projected-key cache at FP8 or BF16). Design:
//   - persistent grid; the (sequence, KV head, page) units of all rows are split evenly
//     over the CTAs, counting only pages that hold tokens (ragged batches balance);
//   - one elected producer lane per CTA streams each unit's contiguous page chunk
//     (128 tokens x r entries, 8 or 16 KiB) with a bulk TMA copy into a shared-memory
//     ring, completion tracked by mbarrier transaction counts;
//   - each consumer lane owns whole tokens: it reads the token's 16-byte chunks from shared
//     memory in a lane-rotated order (conflict-free 128-bit loads), dots them with q~ in
//     FP32 with one accumulator per chunk, and the block max is a warp-shuffle reduction.
#include "qs_device.cuh"

namespace qs {

template <typename PT, int R>
struct ProxyShape {
  static constexpr int kTokenBytes = R * int(sizeof(PT));   // 64 or 128
  static constexpr int kLPT = kTokenBytes / 16;             // lanes per token
  static constexpr int kTPW = 32 / kLPT;                    // tokens per warp step
  static constexpr int kEPL = 16 / int(sizeof(PT));         // elements per lane
  static constexpr int kIter = kPage / kTPW;                // warp steps per page
  static constexpr int kPageBytes = kPage * kTokenBytes;
  static constexpr int kStages = kPageBytes <= 8192 ? 8 : 4;
};

constexpr int kScoreConsumers = 4;
constexpr int kScoreThreads = 32 * (1 + kScoreConsumers);

// Per-sequence unit prefix: units(b) = Hkv * ceil(L_b / 128); lengths are clamped to
// [0, max_context] (an out-of-range length is recorded as a bounds error).
QS_DEV void unit_prefix(const ScoreParams& a, int* prefix) {
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

struct Unit {
  int b, g, p, L, nv, page;
  bool ok;
};

QS_DEV Unit decode_unit(const ScoreParams& a, const int* prefix, int u, int& b) {
  while (u >= prefix[b + 1]) ++b;
  Unit x;
  x.b = b;
  const int np = (prefix[b + 1] - prefix[b]) / a.Hkv;
  const int off = u - prefix[b];
  x.g = off / np;
  x.p = off % np;
  int L = a.seq_lens[b];
  L = L < 0 ? 0 : (L > a.max_context ? a.max_context : L);
  x.L = L;
  x.nv = min(kPage, L - x.p * kPage);
  x.ok = x.p < a.max_pages_per_seq;
  x.page = x.ok ? a.page_table[size_t(b) * a.max_pages_per_seq + x.p] : -1;
  x.ok = x.ok && x.page >= 0 && x.page < a.num_pages;
  return x;
}

template <typename PT, int R>
__global__ void __launch_bounds__(kScoreThreads, 3) score_rankr_kernel(const ScoreParams a) {
  using SH = ProxyShape<PT, R>;
  constexpr int NST = SH::kStages;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* slots = smem;                                          // [NST][page bytes]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NST * SH::kPageBytes);
  uint64_t* empty = full + NST;
  int4* info = reinterpret_cast<int4*>(empty + NST);              // [NST] {row, page idx, nv, ok}
  int* prefix = reinterpret_cast<int*>(info + NST);               // [batch + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (!a.early_stream) pdl_wait();   // q~ and seq_lens come from the kernel before
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  unit_prefix(a, prefix);
  __syncthreads();

  const long long U = prefix[a.batch];
  const int u0 = int(U * blockIdx.x / gridDim.x);
  const int u1 = int(U * (blockIdx.x + 1) / gridDim.x);
  const int n_units = u1 - u0;

  if (warp == 0) {
    // ---------------- producer warp: the 32 lanes resolve 32 units' pages in parallel,
    // then lane 0 issues their bulk copies in order
    int b = 0;
    bool dead = false;
    for (int k0 = 0; k0 < n_units && !dead; k0 += 32) {
      Unit x{};
      x.ok = false;
      x.nv = 0;
      if (k0 + lane < n_units) x = decode_unit(a, prefix, u0 + k0 + lane, b);
      const int row = x.b * a.Hkv + x.g;
      const int m = min(32, n_units - k0);
      for (int j = 0; j < m; ++j) {
        const int jrow = __shfl_sync(kFull, row, j);
        const int jp = __shfl_sync(kFull, x.p, j);
        const int jnv = __shfl_sync(kFull, x.nv, j);
        const int jok = __shfl_sync(kFull, int(x.ok), j);
        const int jpage = __shfl_sync(kFull, x.page, j);
        const int jg = __shfl_sync(kFull, x.g, j);
        if (lane == 0) {
          const int k = k0 + j;
          const int s = k % NST;
          const uint32_t ph = uint32_t(k / NST) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) {
            flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
            dead = true;
          } else {
            info[s] = make_int4(jrow, jp, jnv, jok);
            if (jok) {
              const uint32_t bytes = uint32_t(jnv) * SH::kTokenBytes;
              const uint8_t* src = reinterpret_cast<const uint8_t*>(a.proxy) +
                                   (size_t(jpage) * a.Hkv + jg) * size_t(SH::kPageBytes);
              mbar_arrive_expect_tx(&full[s], bytes);
              bulk_g2s(slots + s * SH::kPageBytes, src, bytes, &full[s]);
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
    return;
  }

  // ---------------- consumers: each lane owns whole tokens (token m*32 + lane, m < 4) and
  // reads its 16-byte chunks in a lane-rotated order so that every quarter-warp's
  // 128-bit shared loads hit distinct banks; one accumulator per chunk position.
  constexpr int CPT = SH::kTokenBytes / 16;           // 16-byte chunks per token: 4 or 8
  constexpr int EPC = SH::kEPL;                       // elements per chunk: 8 (bf16) / 4 (f32)
  const int c = warp - 1;
  // lanes that share a 128-byte bank window in a quarter-warp start at different chunks
  const int rot = lane / (128 / SH::kTokenBytes);
  float qr[CPT][EPC];                                 // q~ permuted by this lane's rotation
  int cur_row = -1;
  if (a.early_stream) pdl_wait();                     // q~ comes from the kernel before
  const int bpp = kPage / a.S;  // blocks per page
  for (int k = c; k < n_units; k += kScoreConsumers) {
    const int s = k % NST;
    const uint32_t ph = uint32_t(k / NST) & 1u;
    if (!mbar_wait(&full[s], ph)) {
      if (lane == 0) flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
      break;
    }
    const int4 x = info[s];                  // {row, page index in row, valid tokens, ok}
    const int row = x.x;
    if (x.w) {
      if (row != cur_row) {
        cur_row = row;
#pragma unroll
        for (int kk = 0; kk < CPT; ++kk) {
          const int ch = (kk + rot) & (CPT - 1);
#pragma unroll
          for (int e = 0; e < EPC; ++e) qr[kk][e] = a.qt[size_t(row) * R + ch * EPC + e];
        }
      }
      const uint8_t* slot = slots + s * SH::kPageBytes;
      float* out = a.scores + size_t(row) * a.nb_stride + size_t(x.y) * bpp;
      const int nv = x.z;
      float sc[kPage / 32];
#pragma unroll
      for (int m = 0; m < kPage / 32; ++m) {
        const int tok = m * 32 + lane;
        const uint8_t* tp = slot + tok * SH::kTokenBytes;
        float acc[CPT];
#pragma unroll
        for (int kk = 0; kk < CPT; ++kk) {
          const uint4 v = *reinterpret_cast<const uint4*>(tp + (((kk + rot) & (CPT - 1)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          float t = 0.0f;
          if constexpr (sizeof(PT) == 1) {            // FP8 E4M3, decoded exactly via FP16
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t h01 = e4m3x2_to_f16x2(w[e]), h23 = e4m3x2_to_f16x2(w[e] >> 16);
              t = fmaf(f16_lo(h01), qr[kk][4 * e], t);
              t = fmaf(f16_hi(h01), qr[kk][4 * e + 1], t);
              t = fmaf(f16_lo(h23), qr[kk][4 * e + 2], t);
              t = fmaf(f16_hi(h23), qr[kk][4 * e + 3], t);
            }
          } else if constexpr (sizeof(PT) == 2) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              t = fmaf(bf16_lo(w[e]), qr[kk][2 * e], t);
              t = fmaf(bf16_hi(w[e]), qr[kk][2 * e + 1], t);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) t = fmaf(__uint_as_float(w[e]), qr[kk][e], t);
          }
          acc[kk] = t;
        }
        float dot = 0.0f;
#pragma unroll
        for (int kk = 0; kk < CPT; ++kk) dot += acc[kk];
        sc[m] = tok < nv ? dot : -INFINITY;
      }
      if (a.S >= 32) {
        const int per = a.S / 32;                      // m-steps per block
        for (int blk = 0; blk < kPage / a.S; ++blk) {
          float mx = -INFINITY;
#pragma unroll
          for (int m = 0; m < kPage / 32; ++m)
            if (m / per == blk) mx = fmaxf(mx, sc[m]);
          mx = warp_max(mx);
          if (lane == 0) out[blk] = mx;
        }
      } else {
#pragma unroll
        for (int m = 0; m < kPage / 32; ++m) {
          float v2 = sc[m];
          for (int o = 1; o < a.S; o <<= 1) v2 = fmaxf(v2, __shfl_xor_sync(kFull, v2, o));
          if ((lane & (a.S - 1)) == 0) out[(m * 32 + lane) / a.S] = v2;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

template <typename PT, int R>
static cudaError_t launch_rankr_score(const ScoreParams& a, cudaStream_t st, bool pdl) {
  using SH = ProxyShape<PT, R>;
  const size_t smem_max = size_t(SH::kStages) * SH::kPageBytes +
                          2 * SH::kStages * sizeof(uint64_t) + SH::kStages * sizeof(int4) +
                          size_t(kMaxBatch + 1) * sizeof(int);
  const size_t smem = smem_max - size_t(kMaxBatch - a.batch) * sizeof(int);
  auto k = score_rankr_kernel<PT, R>;
  // the shared-memory limit is set once per device (sized for the largest batch); the
  // resident CTAs per SM follow from it and are the same on every B200
  const cudaError_t attr = set_smem_limit(k, int(smem_max));
  if (attr != cudaSuccess) return attr;
  static const int per_sm = [&] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kScoreThreads, smem_max) != cudaSuccess)
      n = 0;
    return n;
  }();
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  const long long units = (long long)a.batch * a.Hkv *
                          ((a.max_context + kPage - 1) / kPage);
  long long grid = (long long)num_sms() * (per_sm > 0 ? per_sm : 1);
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  return launch_k(k, dim3(unsigned(grid)), dim3(kScoreThreads), smem, st, pdl, a);
}

cudaError_t launch_score_nvfp4(const Plan& p, const ScoreParams& a, cudaStream_t s, bool pdl);
cudaError_t launch_score_centroid(const Plan& p, const ScoreParams& a, cudaStream_t s, bool pdl);

cudaError_t launch_score(const Plan& p, const ScoreParams& a, cudaStream_t s, bool pdl) {
  if (p.kind == PK_CENTROID) return launch_score_centroid(p, a, s, pdl);
  if (p.kind == PK_NVFP4) return launch_score_nvfp4(p, a, s, pdl);
  if (p.proxy_dtype == QS_E4M3) {
    if (p.r == 32) return launch_rankr_score<uint8_t, 32>(a, s, pdl);
    if (p.r == 64) return launch_rankr_score<uint8_t, 64>(a, s, pdl);
    return cudaErrorInvalidValue;
  }
  const bool f32 = p.proxy_dtype == QS_F32;
  if (f32 && p.r == 16) return launch_rankr_score<float, 16>(a, s, pdl);
  if (f32 && p.r == 32) return launch_rankr_score<float, 32>(a, s, pdl);
  if (!f32 && p.r == 32) return launch_rankr_score<uint16_t, 32>(a, s, pdl);
  if (!f32 && p.r == 64) return launch_rankr_score<uint16_t, 64>(a, s, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace qs
