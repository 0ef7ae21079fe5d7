// score.cu - proxy block scores on the projected-key cache (the rank-r path).
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1: the
// mean of a KV head's query heads, projected into the shared subspace (q~ = qbar . P),
// scores every cached projected key; Figure 9 names this "candidate scoring" and the q~
// computation "scoring preparation". Each block of S tokens is reduced to the maximum of
// its valid tokens' scores (the reading taken for block selection, "Jet-QSparse",
// Full text, which selects 128-token blocks from a dense scan).
//
// The scan is bound by HBM bandwidth (2r bytes and 2r flops per token). Design:
//   - persistent grid; the (sequence, KV head, page) units of all rows are split evenly
//     over the CTAs, counting only pages that hold tokens (ragged batches balance);
//   - one elected producer lane per CTA streams each unit's contiguous page chunk
//     (128 tokens x r entries, 8 or 16 KiB) with a bulk TMA copy into a shared-memory
//     ring, completion tracked by mbarrier transaction counts;
//   - consumer warps read 16-byte vectors from shared memory (LPT lanes per token),
//     dot them with their slice of q~ in FP32, sum across the token's lanes and reduce the
//     block max with warp shuffles.
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
__global__ void __launch_bounds__(kScoreThreads) score_rankr_kernel(const ScoreParams a) {
  using SH = ProxyShape<PT, R>;
  constexpr int NST = SH::kStages;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* slots = smem;                                          // [NST][page bytes]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NST * SH::kPageBytes);
  uint64_t* empty = full + NST;
  int* prefix = reinterpret_cast<int*>(empty + NST);              // [batch + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    // ---------------- producer: one lane issues the bulk copies
    if (lane == 0) {
      int b = 0;
      for (int k = 0; k < n_units; ++k) {
        const int s = k % NST;
        const uint32_t ph = uint32_t(k / NST) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u)) {
          flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
          break;
        }
        const Unit x = decode_unit(a, prefix, u0 + k, b);
        if (x.ok) {
          const uint32_t bytes = uint32_t(x.nv) * SH::kTokenBytes;
          const uint8_t* src = reinterpret_cast<const uint8_t*>(a.proxy) +
                               (size_t(x.page) * a.Hkv + x.g) * size_t(SH::kPageBytes);
          mbar_arrive_expect_tx(&full[s], bytes);
          bulk_g2s(slots + s * SH::kPageBytes, src, bytes, &full[s]);
        } else {
          flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(x.b));
          mbar_arrive(&full[s]);
        }
      }
    }
    return;
  }

  // ---------------- consumers
  const int c = warp - 1;
  const int part = lane % SH::kLPT;
  const int tok_in_step = lane / SH::kLPT;
  float qv[SH::kEPL];
  int cur_row = -1;
  int b = 0;
  const int bpp = kPage / a.S;  // blocks per page
  for (int k = c; k < n_units; k += kScoreConsumers) {
    const int s = k % NST;
    const uint32_t ph = uint32_t(k / NST) & 1u;
    const Unit x = decode_unit(a, prefix, u0 + k, b);
    if (!mbar_wait(&full[s], ph)) {
      if (lane == 0) flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
      break;
    }
    const int row = x.b * a.Hkv + x.g;
    if (x.ok) {
      if (row != cur_row) {
        cur_row = row;
#pragma unroll
        for (int e = 0; e < SH::kEPL; ++e) qv[e] = a.qt[size_t(row) * R + part * SH::kEPL + e];
      }
      const uint8_t* slot = slots + s * SH::kPageBytes;
      float* out = a.scores + size_t(row) * a.nb_stride + size_t(x.p) * bpp;
      float m_run = -INFINITY;
#pragma unroll
      for (int i = 0; i < SH::kIter; ++i) {
        const uint4 v = *reinterpret_cast<const uint4*>(slot + (i * 32 + lane) * 16);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float acc = 0.0f;
        if constexpr (sizeof(PT) == 2) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc = fmaf(bf16_lo(w[e]), qv[2 * e], acc);
            acc = fmaf(bf16_hi(w[e]), qv[2 * e + 1], acc);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) acc = fmaf(__uint_as_float(w[e]), qv[e], acc);
        }
#pragma unroll
        for (int o = 1; o < SH::kLPT; o <<= 1) acc += __shfl_xor_sync(kFull, acc, o);
        const int tok = i * SH::kTPW + tok_in_step;
        const float sc = tok < x.nv ? acc : -INFINITY;
        if (a.S >= SH::kTPW) {
          m_run = fmaxf(m_run, sc);
          if ((((i + 1) * SH::kTPW) & (a.S - 1)) == 0) {
#pragma unroll
            for (int o = SH::kLPT; o < 32; o <<= 1)
              m_run = fmaxf(m_run, __shfl_xor_sync(kFull, m_run, o));
            if (lane == 0) out[(i * SH::kTPW) / a.S] = m_run;
            m_run = -INFINITY;
          }
        } else {
          float v2 = sc;
          for (int o = SH::kLPT; o < SH::kLPT * a.S; o <<= 1)
            v2 = fmaxf(v2, __shfl_xor_sync(kFull, v2, o));
          if ((lane & (SH::kLPT * a.S - 1)) == 0) out[tok / a.S] = v2;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

template <typename PT, int R>
static cudaError_t launch_rankr_score(const ScoreParams& a, cudaStream_t st) {
  using SH = ProxyShape<PT, R>;
  const size_t smem = size_t(SH::kStages) * SH::kPageBytes + 2 * SH::kStages * sizeof(uint64_t) +
                      size_t(a.batch + 1) * sizeof(int);
  auto k = score_rankr_kernel<PT, R>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kScoreThreads, smem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)a.batch * a.Hkv *
                          ((a.max_context + kPage - 1) / kPage);
  long long grid = (long long)num_sms() * (per_sm > 0 ? per_sm : 1);
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  k<<<int(grid), kScoreThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_score_nvfp4(const Plan& p, const ScoreParams& a, cudaStream_t s);

cudaError_t launch_score(const Plan& p, const ScoreParams& a, cudaStream_t s) {
  if (p.r == 0) return launch_score_nvfp4(p, a, s);
  const bool f32 = p.proxy_dtype == QS_F32;
  if (f32 && p.r == 16) return launch_rankr_score<float, 16>(a, s);
  if (f32 && p.r == 32) return launch_rankr_score<float, 32>(a, s);
  if (!f32 && p.r == 32) return launch_rankr_score<uint16_t, 32>(a, s);
  if (!f32 && p.r == 64) return launch_rankr_score<uint16_t, 64>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace qs
