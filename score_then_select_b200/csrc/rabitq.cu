// rabitq.cu - the binary-code scan and the top-p selection ("RaBitQCache", Abstract).
//
//   rq_prep_kernel:  CTA = one row (sequence b, KV head g), thread i = dimension i. The
//                    group-mean query qbar (head sum in order, divided by G), q' = qbar R[g]
//                    (j ascending, one rounding per product and per sum), v_l = min q',
//                    Delta = (max q' - v_l) / 15, codes n_i = min(15, floor((q'_i - v_l) /
//                    Delta + u_i)) (all 0 when Delta = 0), stored as 4 bit planes, with
//                    Delta, v_l, sum n_i and c . qbar. Every step is a rounded float32
//                    operation, so the codes are those of the float32 definition.
//   rq_score_kernel: a warp scores one (row, page) unit at a time: lane l the token slots
//                    l + 32k, k < 4. With A = sum_p 2^p popc(b & plane_p) and B = popc(b),
//                      s = g (Delta (2A - Q) + v_l (2B - d)) + c . qbar
//                    = g sum_i (2 b_i - 1)(Delta n_i + v_l) + c . qbar (the RaBitQ estimate
//                    of q . k, Gao and Long, SIGMOD 2024, section 3), then each block's
//                    log-sum-exp of scale * s over its valid tokens (the log of its
//                    estimated attention mass up to the row's normaliser); the row's
//                    largest block score is recorded in its query-code record.
//   top_p_sorted_kernel, top_p_kernel: CTA = one row (budgets up to 4,096 blocks, and
//                    larger ones); see their comments.
#include <cfloat>

#include "qs_device.cuh"
#include "rabitq.h"

namespace qs {

// ============================================================ query code
template <int D>
__global__ void __launch_bounds__(D) rq_prep_kernel(const RqPrepParams a) {
  constexpr int W = D / 32;
  __shared__ float s_qbar[D];
  __shared__ float s_min[W], s_max[W], s_dot[W];
  __shared__ int s_sum[W];
  const int row = blockIdx.x, b = row / a.Hkv, g = row % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hq = a.Hkv * a.G;
  float acc = 0.0f;
  for (int h = 0; h < a.G; ++h)
    acc = __fadd_rn(acc, bf16_to_f32(a.q[(size_t(b) * Hq + size_t(g) * a.G + h) * D + tid]));
  const float qbar = __fdiv_rn(acc, float(a.G));
  s_qbar[tid] = qbar;
  __syncthreads();
  const float* Rg = a.R + size_t(g) * D * D;
  float y = 0.0f;
  for (int j0 = 0; j0 < D; j0 += 16) {                 // 16 loads of R in flight at a time
    float r[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) r[u] = __ldg(Rg + size_t(j0 + u) * D + tid);
#pragma unroll
    for (int u = 0; u < 16; ++u) y = __fadd_rn(y, __fmul_rn(s_qbar[j0 + u], r[u]));
  }

  float mn = y, mx = y, dot = __fmul_rn(a.key_center[size_t(row) * D + tid], qbar);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    dot += __shfl_xor_sync(kFull, dot, o);
  }
  if (lane == 0) {
    s_min[warp] = mn;
    s_max[warp] = mx;
    s_dot[warp] = dot;
  }
  __syncthreads();
  mn = s_min[0];
  mx = s_max[0];
  dot = s_dot[0];
#pragma unroll
  for (int w = 1; w < W; ++w) {
    mn = fminf(mn, s_min[w]);
    mx = fmaxf(mx, s_max[w]);
    dot += s_dot[w];
  }
  const float delta = __fdiv_rn(__fsub_rn(mx, mn), float(kRqLevels));
  int n = 0;
  if (delta > 0.0f) {
    const float t = __fdiv_rn(__fsub_rn(y, mn), delta);
    const float f = floorf(__fadd_rn(t, a.u[size_t(row) * D + tid]));
    n = f >= float(kRqLevels) ? kRqLevels : (f > 0.0f ? int(f) : 0);
  }
  uint32_t* out = a.qcode + size_t(row) * kRqRowWords;
#pragma unroll
  for (int pl = 0; pl < kRqBits; ++pl) {
    const unsigned w = __ballot_sync(kFull, (n >> pl) & 1);
    if (lane == 0) out[pl * W + warp] = w;
  }
  int sum = n;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
  if (lane == 0) s_sum[warp] = sum;
  __syncthreads();
  if (tid == 0) {
    int q = 0;
    for (int w = 0; w < W; ++w) q += s_sum[w];
    out[kRqDelta] = __float_as_uint(delta);
    out[kRqVl] = __float_as_uint(mn);
    out[kRqQsum] = uint32_t(q);
    out[kRqShift] = __float_as_uint(dot);
    out[kRqRowMax] = 0u;                         // raised by the scan
  }
}

cudaError_t launch_rq_prep(const RqPrepParams& a, cudaStream_t s) {
  if (a.d == 128) rq_prep_kernel<128><<<a.batch * a.Hkv, 128, 0, s>>>(a);
  else rq_prep_kernel<64><<<a.batch * a.Hkv, 64, 0, s>>>(a);
  return cudaGetLastError();
}

// ============================================================ scan

// A score as the select kernels read it: NaN counts as -inf, +inf as FLT_MAX; and its
// order-preserving unsigned key (a larger score, a larger key; -inf > 0).
QS_DEV float tp_clean(float x) { return x != x ? -INFINITY : fminf(x, FLT_MAX); }
QS_DEV uint32_t tp_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
QS_DEV float tp_unkey(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// float(n) for |n| < 2^22 without a conversion instruction (those share the quarter-rate
// pipe with the population counts): 1.5 * 2^23 + n is exact in float32 (its ulp is 1), so
// adding n to that value's bit pattern and subtracting it again gives n exactly.
QS_DEV float rq_int_to_float(int n) { return __int_as_float(0x4B400000 + n) - 12582912.0f; }

// Merge of log-sum-exp states: (m, l) stands for l * e^m.
QS_DEV void lse_merge(float& m, float& l, float m2, float l2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) {
    m = -INFINITY;
    l = 0.0f;
    return;
  }
  l = l * expf(m - mm) + l2 * expf(m2 - mm);
  m = mm;
}

// Persistent grid, one producer warp and four consumer warps per CTA. A unit is one
// (row = (sequence b, KV head g), page p), p fastest, so that a CTA's contiguous share of
// the units covers one or two rows: a consumer keeps the row's query code in registers
// and reloads it only when the row changes. The producer's lanes resolve 32 units' pages
// at a time and lane 0 streams each unit's (page, head) record (code bits and factors,
// 2,560 bytes at d = 128) with one bulk copy into a 12-stage shared-memory ring,
// completion counted on the stage's mbarrier; units past a row's length are skipped.
// Consumer warp c scores units c, c + 4, ...: lane l the token slots l + 32 k. The scoring
// is bound by instruction latency (20 AND/POPC pairs per token), so the CTA is kept to 64
// registers and 31 KB of shared memory: six CTAs (24 consumer warps) per SM.
constexpr int kRqConsumers = 4;
constexpr int kRqThreads = 32 * (1 + kRqConsumers);
constexpr int kRqStages = 12;

template <int D>
struct RqShape {
  static constexpr int kPageBytes = kPage * (D / 8) + kPage * 4;
  static constexpr int kSmem = kRqStages * kPageBytes + 2 * kRqStages * 8 + kRqStages * 16;
};

template <int D, int S>
__global__ void __launch_bounds__(kRqThreads, 6) rq_score_kernel(const RqScoreParams a) {
  using SH = RqShape<D>;
  constexpr int W = D / 32, PB = SH::kPageBytes;
  extern __shared__ __align__(128) uint8_t rq_smem[];
  uint8_t* slots = rq_smem;                                        // [stages][PB]
  uint64_t* full = reinterpret_cast<uint64_t*>(rq_smem + kRqStages * PB);
  uint64_t* empty = full + kRqStages;
  int4* info = reinterpret_cast<int4*>(empty + kRqStages);         // {row, page idx, L, page}
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRqStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int max_pages = a.nb_stride / (kPage / S);
  const long long U = (long long)a.batch * a.Hkv * max_pages;
  const long long u0 = U * blockIdx.x / gridDim.x, u1 = U * (blockIdx.x + 1) / gridDim.x;
  const int n_units = int(u1 - u0);

  if (warp == 0) {
    // ---------------- producer
    bool dead = false;
    for (int k0 = 0; k0 < n_units && !dead; k0 += 32) {
      int row = 0, pi = 0, L = 0, page = -1;
      if (k0 + lane < n_units) {
        const long long u = u0 + k0 + lane;
        row = int(u / max_pages);
        pi = int(u - (long long)row * max_pages);
        const int b = row / a.Hkv, g = row - b * a.Hkv;
        L = a.seq_lens[b];
        if (L > a.max_context || L < 0) {
          if (pi == 0 && g == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(b));
          L = L < 0 ? 0 : a.max_context;
        }
        const int pages = (L + kPage - 1) / kPage;
        if (pi < pages) {
          page = pi < a.max_pages_per_seq ? a.page_table[size_t(b) * a.max_pages_per_seq + pi] : -1;
          if (page < 0 || page >= a.num_pages) {
            flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(row));
            page = -1;
          }
        } else {
          page = -2;                                   // past the row's tokens: nothing
        }
      }
      const int m = min(32, n_units - k0);
      for (int j = 0; j < m; ++j) {
        const int jrow = __shfl_sync(kFull, row, j), jp = __shfl_sync(kFull, pi, j);
        const int jL = __shfl_sync(kFull, L, j), jpage = __shfl_sync(kFull, page, j);
        if (lane == 0) {
          const int k = k0 + j;
          const int s = k % kRqStages;
          if (!mbar_wait(&empty[s], (uint32_t(k / kRqStages) & 1u) ^ 1u)) {
            flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
            dead = true;
          } else {
            info[s] = make_int4(jrow, jp, jL, jpage);
            if (jpage >= 0) {
              const int g = jrow % a.Hkv;
              mbar_arrive_expect_tx(&full[s], uint32_t(PB));
              bulk_g2s(slots + s * PB, a.proxy + (size_t(jpage) * a.Hkv + g) * PB, uint32_t(PB),
                       &full[s]);
            } else {
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

  // ---------------- consumers
  const int c = warp - 1;
  int cur = -1;                                    // the row whose query code is loaded
  uint32_t plane[kRqBits][W];
  float delta = 0.0f, vl = 0.0f, shift = 0.0f;
  int Q = 0;
  for (int k = c; k < n_units; k += kRqConsumers) {
    const int s = k % kRqStages;
    if (!mbar_wait(&full[s], uint32_t(k / kRqStages) & 1u)) {
      if (lane == 0) flag_error(a.hdr, QS_ERR_DEVICE_TIMEOUT, KID_SCORE, uint32_t(k));
      break;
    }
    const int4 x = info[s];
    if (x.w >= 0) {
      const int row = x.x, pi = x.y, L = x.z;
      const uint8_t* pg = slots + s * PB;
      if (row != cur) {                            // warp-uniform
        // plain loads: word kRqRowMax of the same record is raised during this kernel
        const uint32_t* qc = a.qcode + size_t(row) * kRqRowWords;
#pragma unroll
        for (int p = 0; p < kRqBits; ++p)
#pragma unroll
          for (int w = 0; w < W; ++w) plane[p][w] = qc[p * W + w];
        delta = __uint_as_float(qc[kRqDelta]);
        vl = __uint_as_float(qc[kRqVl]);
        shift = __uint_as_float(qc[kRqShift]);
        Q = int(qc[kRqQsum]);
        cur = row;
      }
      float m[4], l[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int slot = lane + 32 * kk;
        uint32_t code[W];
        if constexpr (W == 4) {
          const uint4 v = *reinterpret_cast<const uint4*>(pg + slot * 16);
          code[0] = v.x;
          code[1] = v.y;
          code[2] = v.z;
          code[3] = v.w;
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(pg + slot * 8);
          code[0] = v.x;
          code[1] = v.y;
        }
        const float gk = reinterpret_cast<const float*>(pg + kPage * (D / 8))[slot];
        int A = 0, B = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) {
          B += __popc(code[w]);
#pragma unroll
          for (int p = 0; p < kRqBits; ++p) A += __popc(code[w] & plane[p][w]) << p;
        }
        const float est = gk * (delta * rq_int_to_float(2 * A - Q) +
                                vl * rq_int_to_float(2 * B - D)) + shift;
        const bool valid = pi * kPage + slot < L;
        m[kk] = valid ? a.scale * est : -INFINITY;
        l[kk] = valid ? 1.0f : 0.0f;
      }
      float* out = a.scores + size_t(row) * a.nb_stride + size_t(pi) * (kPage / S);
      float vmax = -INFINITY;                      // the largest score this warp writes
      if constexpr (S == 1) {
        // a block = one token: its log-sum-exp is its own scaled estimate
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          out[lane + 32 * kk] = m[kk];
          vmax = fmaxf(vmax, tp_clean(m[kk]));
        }
      } else if constexpr (S < 32) {
        // a block = S neighbouring lanes of one k
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          float mk = m[kk], lk = l[kk];
#pragma unroll
          for (int o = 1; o < S; o <<= 1) {
            const float m2 = __shfl_xor_sync(kFull, mk, o), l2 = __shfl_xor_sync(kFull, lk, o);
            lse_merge(mk, lk, m2, l2);
          }
          if ((lane & (S - 1)) == 0) {
            const float v = lk > 0.0f ? mk + logf(lk) : -INFINITY;
            out[(lane + 32 * kk) / S] = v;
            vmax = fmaxf(vmax, tp_clean(v));
          }
        }
      } else {
        // a block = S / 32 consecutive k of every lane
        constexpr int KB = S / 32;
#pragma unroll
        for (int k0 = 0; k0 < 4; k0 += KB) {
          float mk = m[k0], lk = l[k0];
#pragma unroll
          for (int kk = k0 + 1; kk < k0 + KB; ++kk) lse_merge(mk, lk, m[kk], l[kk]);
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float m2 = __shfl_xor_sync(kFull, mk, o), l2 = __shfl_xor_sync(kFull, lk, o);
            lse_merge(mk, lk, m2, l2);
          }
          if (lane == 0) {
            const float v = lk > 0.0f ? mk + logf(lk) : -INFINITY;
            out[(32 * k0) / S] = v;
            vmax = fmaxf(vmax, tp_clean(v));
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(kFull, vmax, o));
      if (lane == 0 && vmax > -INFINITY)
        atomicMax(a.qcode + size_t(row) * kRqRowWords + kRqRowMax, tp_key(vmax));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

template <int D>
static cudaError_t launch_rq_score_d(const RqScoreParams& a, cudaStream_t s) {
  using SH = RqShape<D>;
  const int max_pages = a.nb_stride / (kPage / a.S);
  const long long units = (long long)a.batch * max_pages * a.Hkv;
  long long grid = (long long)num_sms() * 6;
  if (grid > units) grid = units;
  if (grid < 1) grid = 1;
  const dim3 block(kRqThreads);
  const int smem = SH::kSmem;
#define QS_RQ(SV)                                                                          \
  {                                                                                        \
    const cudaError_t e = set_smem_limit(rq_score_kernel<D, SV>, smem);                    \
    if (e != cudaSuccess) return e;                                                        \
    rq_score_kernel<D, SV><<<unsigned(grid), block, smem, s>>>(a);                         \
    break;                                                                                 \
  }
  switch (a.S) {
    case 1: QS_RQ(1)
    case 2: QS_RQ(2)
    case 4: QS_RQ(4)
    case 8: QS_RQ(8)
    case 16: QS_RQ(16)
    case 32: QS_RQ(32)
    case 64: QS_RQ(64)
    case 128: QS_RQ(128)
    default: return cudaErrorInvalidValue;
  }
#undef QS_RQ
  return cudaGetLastError();
}

cudaError_t launch_rq_score(const RqScoreParams& a, cudaStream_t s) {
  return a.d == 128 ? launch_rq_score_d<128>(a, s) : launch_rq_score_d<64>(a, s);
}

// ============================================================ top-p selection
// CTA = one row, 1024 threads. The block scores are natural-log masses beta_j. With
// M = max beta, block j weighs w_j = e^(beta_j - M), held as an integer in units of 2^-40:
// every sum below is exact, so the result does not depend on the order of additions.
// Z = sum of all w, goal = min(Z, ceil(p Z)). The forced blocks are taken first; if their
// mass is short of the goal, the others follow in order of decreasing beta (ties to the
// lower index) until the goal is reached or the budget is full. The last beta taken is
// found by three histogram passes over the order-preserving integer key of beta (its top
// 11, next 11 and last 10 bits), each bin carrying its count and mass; blocks with exactly
// that key (equal beta, equal mass) are taken in index order, as many as still needed.
// A NaN score counts as -inf (mass 0), +inf as FLT_MAX.
constexpr int kTpThreads = 1024;
constexpr int kTpBins = 2048;
constexpr float kTpUnit = 1099511627776.0f;   // 2^40

QS_DEV unsigned long long tp_mass(float x, float M) {
  if (!(M > -INFINITY)) return 0ull;
  return __float2ull_rn(expf(x - M) * kTpUnit);
}

// One streaming pass over a row's nb scores. Sweep `it` gives thread t the blocks
// j = it + t + u kTpThreads, u < kTpUnroll: all kTpUnroll loads are issued before the first
// is used, so every thread keeps that many in flight (a pass over a token-level row is
// otherwise one dependent load after another). Every thread runs the same number of sweeps
// and calls f(j, x, in) for each of its blocks, in = j < nb, x = the cleaned score (-inf
// when !in), so whole warps stay together for warp-collective steps inside f.
constexpr int kTpUnroll = 8;
template <typename F>
QS_DEV void tp_sweep(const float* sc, int nb, F&& f) {
  for (int it = 0; it < nb; it += kTpUnroll * kTpThreads) {
    float x[kTpUnroll];
#pragma unroll
    for (int u = 0; u < kTpUnroll; ++u) {
      const int j = it + int(threadIdx.x) + u * kTpThreads;
      x[u] = j < nb ? sc[j] : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < kTpUnroll; ++u) {
      const int j = it + int(threadIdx.x) + u * kTpThreads;
      f(j, tp_clean(x[u]), j < nb);
    }
  }
}

QS_DEV float tp_block_max(float v, float* s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  if (lane == 0) s[warp] = v;
  __syncthreads();
  float r = s[0];
  for (int w = 1; w < kTpThreads / 32; ++w) r = fmaxf(r, s[w]);
  __syncthreads();
  return r;
}

// Exclusive prefix of v over the threads in order; total receives the sum of all v.
QS_DEV unsigned long long tp_scan(unsigned long long v, unsigned long long* s,
                                  unsigned long long& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned long long t = s[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += y;
    }
    s[lane] = t;
  }
  __syncthreads();
  const unsigned long long before = warp ? s[warp - 1] : 0ull;
  total = s[kTpThreads / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// The bin (of nbins, walked from the highest) at which the cumulative count reaches cap or
// the cumulative mass reaches need, with the count and mass of the bins above it; bin -1
// if neither is reached. Every thread returns the same values.
struct TpFound {
  int bin;
  uint32_t cnt_above;
  unsigned long long mass_above;
};
QS_DEV TpFound tp_find(const uint32_t* cnt, const unsigned long long* mass, int nbins,
                       uint32_t cap, unsigned long long need, unsigned long long* s_scan,
                       TpFound* s_found) {
  const int per = nbins / kTpThreads;              // 2 or 1 bins per thread
  const int hi = nbins - 1 - int(threadIdx.x) * per;
  unsigned long long c_loc = 0, m_loc = 0;
  for (int i = 0; i < per; ++i) {
    c_loc += cnt[hi - i];
    m_loc += mass[hi - i];
  }
  if (threadIdx.x == 0) {
    s_found->bin = -1;
    s_found->cnt_above = 0u;
    s_found->mass_above = 0ull;
  }
  unsigned long long tot;
  unsigned long long c = tp_scan(c_loc, s_scan, tot);
  unsigned long long m = tp_scan(m_loc, s_scan, tot);
  for (int i = 0; i < per; ++i) {
    const bool before = c >= cap || m >= need;
    c += cnt[hi - i];
    m += mass[hi - i];
    if (!before && (c >= cap || m >= need)) {
      s_found->bin = hi - i;
      s_found->cnt_above = uint32_t(c - cnt[hi - i]);
      s_found->mass_above = m - mass[hi - i];
    }
  }
  __syncthreads();
  TpFound f;
  f.bin = s_found->bin;
  f.cnt_above = s_found->cnt_above;
  f.mass_above = s_found->mass_above;
  __syncthreads();
  return f;
}

// One warp's histogram update: every lane with `active` adds one block of key bin `bin`
// and fixed-point mass w. Lanes that share a bin are combined first (one shared atomic per
// bin and warp instead of one per lane; a row's scores crowd into few bins of the top key
// bits). Masses are at most 2^40, so their 20-bit halves sum exactly in 32 bits.
QS_DEV void tp_hist_add(uint32_t* h_cnt, unsigned long long* h_mass, bool active, uint32_t bin,
                        unsigned long long w) {
  const unsigned act = __ballot_sync(kFull, active);
  if (!active) return;
  const unsigned peers = __match_any_sync(act, bin);
  const uint32_t lo = __reduce_add_sync(peers, uint32_t(w & 0xfffffull));
  const uint32_t hi = __reduce_add_sync(peers, uint32_t(w >> 20));
  if (int(threadIdx.x & 31) == __ffs(peers) - 1) {
    atomicAdd(&h_cnt[bin], uint32_t(__popc(peers)));
    atomicAdd(&h_mass[bin], ((unsigned long long)hi << 20) + lo);
  }
}

// Exclusive prefix over the 32 warps' values (v given by lane 0 of each warp); every thread
// returns its warp's prefix, total the sum. Two block barriers.
QS_DEV unsigned tp_warp_scan(unsigned v, unsigned* s, unsigned& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s[warp] = v;
  __syncthreads();
  unsigned x = s[lane], inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(kFull, inc, o);
    if (lane >= o) inc += y;
  }
  const unsigned before = __shfl_sync(kFull, inc - x, warp);
  total = __shfl_sync(kFull, inc, 31);
  __syncthreads();
  return before;
}

// CTA = one row (1,024 threads; kTpThreads / 32 = 32 warps):
//   1. M = the row's largest score; every block's mass e^(beta_j - M) as an integer in
//      units of 2^-40 (so Z, the forced mass and all cumulative sums are exact and do not
//      depend on the order of summation);
//   2. goal = min(Z, ceil(p Z)); the cut is found by three histogram passes over the
//      order-preserving key of beta (11, 11 and 10 bits), each bin carrying its count and
//      mass: the bin where the count reaches the remaining budget or the mass the
//      remaining goal, walked from the highest bin;
//   3. taken: the forced blocks, every block above the final key, and the first blocks (in
//      index order) holding the final key, as many as still needed; the output ascending.
// Loads are coalesced: the histogram passes stride the row by the CTA, and the output
// passes give warp w the contiguous span [w E, (w + 1) E) of the row, 32 blocks per step.
__global__ void __launch_bounds__(kTpThreads, 1) top_p_kernel(const TopPParams a) {
  __shared__ uint32_t h_cnt[kTpBins];
  __shared__ unsigned long long h_mass[kTpBins];
  __shared__ unsigned long long s_u[kTpThreads / 32];
  __shared__ unsigned s_w[kTpThreads / 32];
  __shared__ float s_f[kTpThreads / 32];
  __shared__ TpFound s_found;
  const int row = blockIdx.x, b = row / a.Hkv, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const float* sc = a.scores + size_t(row) * a.nb_stride;
  int32_t* out = a.sel + size_t(row) * a.budget;
  const int L = a.seq_lens[b];
  int nb = L > 0 ? (L + a.S - 1) / a.S : 0;
  if (nb > a.nb_stride) {
    if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
    nb = a.nb_stride;
  }
  const int f0 = (a.force_sink && nb > 0) ? 0 : -1;
  const int f1 = (a.force_last && nb > 0 && nb - 1 != f0) ? nb - 1 : -1;
  const int nF = (f0 >= 0) + (f1 >= 0);

  // the row's largest score
  float mx = -INFINITY;
  tp_sweep(sc, nb, [&](int, float x, bool) { mx = fmaxf(mx, x); });
  const float M = tp_block_max(mx, s_f);

  // Z, the forced blocks' mass, and the histogram of the others' top 11 key bits
  for (int i = tid; i < kTpBins; i += kTpThreads) {
    h_cnt[i] = 0u;
    h_mass[i] = 0ull;
  }
  __syncthreads();
  unsigned long long z = 0, mf = 0;
  tp_sweep(sc, nb, [&](int j, float x, bool in) {
    const unsigned long long w = in ? tp_mass(x, M) : 0ull;
    const bool forced = j == f0 || j == f1;
    z += w;
    if (forced) mf += w;
    tp_hist_add(h_cnt, h_mass, in && !forced, tp_key(x) >> 21, w);
  });
  unsigned long long Z, MF;
  tp_scan(z, s_u, Z);            // totals; the barriers inside also complete the histogram
  tp_scan(mf, s_u, MF);
  unsigned long long goal = (unsigned long long)ceil(double(a.p) * double(Z));
  if (goal > Z) goal = Z;
  uint32_t cap = uint32_t(max(0, a.budget - nF));
  unsigned long long need = goal > MF ? goal - MF : 0ull;

  // mode 0: forced blocks only; 1: every block; 2: the blocks above the key kstar, and
  // the first `ties` blocks with key kstar
  int mode = 0;
  uint32_t kstar = 0, ties = 0;
  if (need > 0 && cap > 0) {
    TpFound f = tp_find(h_cnt, h_mass, kTpBins, cap, need, s_u, &s_found);
    if (f.bin < 0) {
      mode = 1;
    } else {
      mode = 2;
      uint32_t prefix = uint32_t(f.bin);
      cap -= f.cnt_above;
      need -= f.mass_above;
      // refine: the next 11 bits, then the last 10, of the keys in the chosen bin
      for (int pass = 0; pass < 2 && mode == 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0, nbins = pass == 0 ? kTpBins : kTpBins / 2;
        const int known = pass == 0 ? 21 : 10;
        for (int i = tid; i < kTpBins; i += kTpThreads) {
          h_cnt[i] = 0u;
          h_mass[i] = 0ull;
        }
        __syncthreads();
        tp_sweep(sc, nb, [&](int j, float x, bool in) {
          in = in && j != f0 && j != f1;
          const uint32_t key = tp_key(x);
          const bool hit = in && (key >> known) == prefix;
          tp_hist_add(h_cnt, h_mass, hit, (key >> shift) & uint32_t(nbins - 1),
                      hit ? tp_mass(x, M) : 0ull);
        });
        __syncthreads();
        f = tp_find(h_cnt, h_mass, nbins, cap, need, s_u, &s_found);
        if (f.bin < 0) {
          // cannot happen (the chosen bin reaches cap or need); keep the forced blocks
          if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
          mode = 0;
        } else {
          prefix = (prefix << (pass == 0 ? 11 : 10)) | uint32_t(f.bin);
          cap -= f.cnt_above;
          need -= f.mass_above;
          if (pass == 1) {
            kstar = prefix;
            const uint32_t T = h_cnt[f.bin];
            const unsigned long long each = T ? h_mass[f.bin] / T : 0ull;
            ties = each > 0 ? uint32_t(min((unsigned long long)cap, (need + each - 1) / each)) : cap;
            ties = min(ties, T);
          }
        }
      }
    }
  }

  // output, ascending. Warp w owns blocks [w E, w E + E), E a multiple of 32; a block is
  // taken if forced, if mode 1, or (mode 2) if its key is above kstar, or if it holds
  // kstar and fewer than `ties` blocks with kstar come before it in the row.
  const int E = (nb + kTpThreads - 1) / kTpThreads * 32;
  const int j0 = warp * E, j1 = min(nb, j0 + E);
  unsigned n_sure = 0, n_tie = 0;                       // per warp (same in every lane)
  for (int jb = j0; jb < j1; jb += 32) {
    const int j = jb + lane;
    bool sure = false, tie = false;
    if (j < j1) {
      const bool forced = j == f0 || j == f1;
      if (forced || mode == 1) {
        sure = true;
      } else if (mode == 2) {
        const uint32_t key = tp_key(tp_clean(sc[j]));
        sure = key > kstar;
        tie = key == kstar;
      }
    }
    n_sure += __popc(__ballot_sync(kFull, sure));
    n_tie += __popc(__ballot_sync(kFull, tie));
  }
  unsigned tie_tot, n_tot;
  const unsigned tie_before = tp_warp_scan(n_tie, s_w, tie_tot);
  const unsigned tie_take = tie_before >= ties ? 0u : min(n_tie, ties - tie_before);
  unsigned pos = tp_warp_scan(n_sure + tie_take, s_w, n_tot);
  unsigned tie_rank = tie_before;
  for (int jb = j0; jb < j1; jb += 32) {
    const int j = jb + lane;
    bool sure = false, tie = false;
    if (j < j1) {
      const bool forced = j == f0 || j == f1;
      if (forced || mode == 1) {
        sure = true;
      } else if (mode == 2) {
        const uint32_t key = tp_key(tp_clean(sc[j]));
        sure = key > kstar;
        tie = key == kstar;
      }
    }
    const unsigned tmask = __ballot_sync(kFull, tie);
    const unsigned below = (1u << lane) - 1u;
    const bool take = sure || (tie && tie_rank + __popc(tmask & below) < ties);
    const unsigned took = __ballot_sync(kFull, take);
    if (take) {
      const unsigned at = pos + __popc(took & below);
      if (at < unsigned(a.budget)) out[at] = j;
      else flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
    }
    pos += __popc(took);
    tie_rank += __popc(tmask);
  }
  const int n = int(min(n_tot, unsigned(a.budget)));
  if (tid == 0) a.n_sel[row] = n;
  for (int i = n + tid; i < a.budget; i += kTpThreads) out[i] = -1;
}

// ------------------------------------------------------------ top-p by sorted candidates
// The same selection without 64-bit shared-memory atomics, for budgets of at most
// kTpCandMax blocks (the token-level budgets of the pages: B = 2,048), in three passes
// over the row's scores:
//   1. M, the largest score, and the smallest finite score of a non-forced block;
//   2. Z and the forced mass (per-thread 64-bit integer sums, then a block scan), and a
//      2,048-bin histogram of the finite non-forced scores linear between that minimum
//      and M (32-bit counts);
//   3. the candidates: every block in the bins from the one where the count from the top
//      reaches cap (= budget minus the forced blocks) upwards, compacted into shared
//      memory as 64-bit sort keys (key << 32 | ~index). If that bin is crowded (many equal
//      or nearly equal scores) three count-only passes over the key bits find the cap-th
//      key instead, and the candidates are the blocks above it and the first blocks (in
//      index order) holding it;
// then the candidates are bitonic-sorted, largest first (decreasing beta, ties to the
// lower index: the order in which blocks are taken), their masses summed in that order
// over the first cap of them, and the fewest whose mass with the forced blocks' reaches
// the goal are taken (all cap if none); the taken and forced blocks are marked in a bitmap
// of the row and written out in ascending order.
constexpr int kTpCandMax = 4096;

// Bin of a finite score x in the histogram linear between lo and lo + kTpBins / inv,
// clamped to [0, kTpBins - 1]: monotone in x.
QS_DEV int tp_lin_bin(float x, float lo, float inv) {
  return min(kTpBins - 1, int(fmaxf(0.0f, (x - lo) * inv)));
}
static_assert(kTpCandMax <= 4 * kTpThreads, "tp_sort holds at most 4 keys per thread");

QS_DEV void tp_count_add(uint32_t* h, bool active, uint32_t bin) {
  const unsigned act = __ballot_sync(kFull, active);
  if (!active) return;
  const unsigned peers = __match_any_sync(act, bin);
  if (int(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], uint32_t(__popc(peers)));
}

// The bin (walked from the highest of nbins) at which the cumulative count reaches cap, and
// the count of the bins above it; -1 if the counts never reach cap.
QS_DEV int tp_find_count(const uint32_t* cnt, int nbins, uint32_t cap, unsigned long long* s_scan,
                         TpFound* s_found, uint32_t& above) {
  const int per = nbins / kTpThreads;
  const int hi = nbins - 1 - int(threadIdx.x) * per;
  unsigned long long c_loc = 0;
  for (int i = 0; i < per; ++i) c_loc += cnt[hi - i];
  if (threadIdx.x == 0) {
    s_found->bin = -1;
    s_found->cnt_above = 0u;
  }
  unsigned long long tot;
  unsigned long long c = tp_scan(c_loc, s_scan, tot);
  for (int i = 0; i < per; ++i) {
    const bool before = c >= cap;
    c += cnt[hi - i];
    if (!before && c >= cap) {
      s_found->bin = hi - i;
      s_found->cnt_above = uint32_t(c - cnt[hi - i]);
    }
  }
  __syncthreads();
  const int bin = s_found->bin;
  above = s_found->cnt_above;
  __syncthreads();
  return bin;
}

// Bitonic sort of cand[0, 1024 E), largest first (the same compare-exchange network as
// sorting in shared memory). Element i = 1024 s + t is held by thread t in v[s]: a stage
// whose partner i ^ jj is in the same warp (jj < 32) exchanges by shuffles, one in the same
// thread (jj >= 1024) in registers, and only the others (32 <= jj < 1024) through cand.
// Every thread of the CTA calls it.
QS_DEV unsigned long long tp_keep(unsigned long long x, unsigned long long y, bool keep_max) {
  return (x > y) == keep_max ? x : y;
}
template <int E>
QS_DEV void tp_sort(unsigned long long* cand) {
  const int t = int(threadIdx.x);
  unsigned long long v[E];
#pragma unroll
  for (int s = 0; s < E; ++s) v[s] = cand[s * kTpThreads + t];
  for (int k = 2; k <= kTpThreads * E; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      if (jj < 32) {
#pragma unroll
        for (int s = 0; s < E; ++s) {
          const int i = s * kTpThreads + t;
          const unsigned long long o = __shfl_xor_sync(kFull, v[s], jj);
          v[s] = tp_keep(v[s], o, ((i & jj) == 0) == ((i & k) == 0));
        }
      } else if (jj < kTpThreads) {
#pragma unroll
        for (int s = 0; s < E; ++s) cand[s * kTpThreads + t] = v[s];
        __syncthreads();
#pragma unroll
        for (int s = 0; s < E; ++s) {
          const int i = s * kTpThreads + t;
          v[s] = tp_keep(v[s], cand[i ^ jj], ((i & jj) == 0) == ((i & k) == 0));
        }
        __syncthreads();
      } else {
        const int js = jj / kTpThreads;
#pragma unroll
        for (int s = 0; s < E; ++s)
#pragma unroll
          for (int s2 = s + 1; s2 < E; ++s2)
            if ((s ^ s2) == js) {                     // pair (s, s2), s the lower index
              const bool desc = ((s * kTpThreads + t) & k) == 0;
              const unsigned long long x = v[s], y = v[s2];
              v[s] = tp_keep(x, y, desc);
              v[s2] = tp_keep(x, y, !desc);
            }
      }
    }
  }
#pragma unroll
  for (int s = 0; s < E; ++s) cand[s * kTpThreads + t] = v[s];
  __syncthreads();
}

__global__ void __launch_bounds__(kTpThreads, 1) top_p_sorted_kernel(const TopPParams a) {
  extern __shared__ __align__(16) uint8_t tp_smem[];
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(tp_smem);   // [kTpCandMax]
  unsigned long long* tmp = cand + kTpCandMax;                                 // [kTpCandMax]
  unsigned long long* hmass = tmp + kTpCandMax;                                // [kTpBins]
  uint32_t* hist = reinterpret_cast<uint32_t*>(hmass + kTpBins);               // [kTpBins]
  uint32_t* bits = hist + kTpBins;                                              // [row words]
  __shared__ unsigned long long s_u[kTpThreads / 32];
  __shared__ unsigned s_w[kTpThreads / 32];
  __shared__ float s_f[kTpThreads / 32];
  __shared__ TpFound s_found;
  const int row = blockIdx.x, b = row / a.Hkv, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const float* sc = a.scores + size_t(row) * a.nb_stride;
  int32_t* out = a.sel + size_t(row) * a.budget;
  const int L = a.seq_lens[b];
  int nb = L > 0 ? (L + a.S - 1) / a.S : 0;
  if (nb > a.nb_stride) {
    if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
    nb = a.nb_stride;
  }
  const int f0 = (a.force_sink && nb > 0) ? 0 : -1;
  const int f1 = (a.force_last && nb > 0 && nb - 1 != f0) ? nb - 1 : -1;
  const int nF = (f0 >= 0) + (f1 >= 0);

  // 1. the row's largest score, and the smallest finite score of a non-forced block. When
  // the scan that wrote the scores recorded each row's largest (its order-preserving key),
  // this pass is skipped: M is that score, and the histogram below starts at M - 28
  // instead of the smallest score (a block 28 below M has mass e^-28 < 2^-40, which rounds
  // to 0; bins only need to be monotone in the score, lower scores fall into bin 0, and a
  // cut in bin 0 with too many candidates takes the key-bit passes).
  float M, lo;
  if (a.row_max) {
    const uint32_t k = a.row_max[size_t(row) * a.row_max_stride];
    M = k ? tp_unkey(k) : -INFINITY;
    lo = M > -INFINITY ? M - 28.0f : INFINITY;
  } else {
    float mx = -INFINITY, mn = INFINITY;
    tp_sweep(sc, nb, [&](int j, float x, bool) {
      mx = fmaxf(mx, x);
      if (x > -INFINITY && j != f0 && j != f1) mn = fminf(mn, x);
    });
    M = tp_block_max(mx, s_f);
    lo = -tp_block_max(-mn, s_f);
  }
  const uint32_t cap = uint32_t(max(0, min(a.budget - nF, nb - nF)));
  // 2. Z, the forced mass, the count of finite non-forced blocks and (when the finite span
  // is finite) a 2,048-bin histogram of them linear in the score between lo and M
  const float span = M - lo;
  const bool lin = cap > 0 && lo < INFINITY && span < INFINITY;
  const float inv = span > 0.0f ? float(kTpBins) / span : 0.0f;
  if (lin) {
    for (int i = tid; i < kTpBins; i += kTpThreads) hist[i] = 0u;
    __syncthreads();
  }
  unsigned long long z = 0, mf = 0;
  unsigned nfin = 0u;
  tp_sweep(sc, nb, [&](int j, float x, bool in) {
    if (!in) return;
    const unsigned long long w = tp_mass(x, M);
    z += w;
    if (j == f0 || j == f1) {
      mf += w;
    } else if (x > -INFINITY) {
      ++nfin;
      if (lin) atomicAdd(&hist[tp_lin_bin(x, lo, inv)], 1u);
    }
  });
  unsigned long long Z, MF, NFIN;
  tp_scan(z, s_u, Z);             // the barriers inside also complete the histogram
  tp_scan(mf, s_u, MF);
  tp_scan(nfin, s_u, NFIN);
  unsigned long long goal = (unsigned long long)ceil(double(a.p) * double(Z));
  if (goal > Z) goal = Z;

  // 3. the candidates: at least the cap best non-forced blocks, compacted as 64-bit sort
  // keys (key << 32 | ~index). First by a 2,048-bin histogram linear in the score between
  // the row's finite minimum and maximum (a monotone map: a higher bin never holds a lower
  // score): the bins above the one where the count reaches cap, and that bin, in one pass.
  // Blocks at -inf carry no mass and are never needed. If that bin is too crowded (many
  // equal or nearly equal scores), three count-only passes over the key bits find the
  // cap-th key and the candidates are the blocks above it plus the first blocks holding it.
  __shared__ unsigned s_nc;
  unsigned c_tot = 0u;
  bool linear_ok = false;
  if (lin) {
    // the bin where the count of finite blocks from the top reaches cap (all bins when
    // there are no more than cap finite blocks)
    uint32_t above = 0u;
    int cut = 0;
    uint32_t n_cand = uint32_t(NFIN);
    if (NFIN > cap) {
      cut = tp_find_count(hist, kTpBins, cap, s_u, &s_found, above);
      n_cand = above + hist[cut];
    }
    if (n_cand <= uint32_t(kTpCandMax)) {
      linear_ok = true;
      if (tid == 0) s_nc = 0u;
      __syncthreads();
      tp_sweep(sc, nb, [&](int j, float x, bool in) {
        const bool take = in && x > -INFINITY && j != f0 && j != f1 &&
                          tp_lin_bin(x, lo, inv) >= cut;
        const unsigned tm = __ballot_sync(kFull, take);
        if (tm == 0u) return;                          // warp-uniform
        unsigned base = 0u;
        if (lane == 0) base = atomicAdd(&s_nc, unsigned(__popc(tm)));
        base = __shfl_sync(kFull, base, 0);
        if (take)
          cand[base + __popc(tm & ((1u << lane) - 1u))] =
              ((unsigned long long)tp_key(x) << 32) | (0xffffffffu - uint32_t(j));
      });
      __syncthreads();
      c_tot = s_nc;
    }
  }
  if (cap > 0 && lo < INFINITY && !linear_ok) {      // the key-bit passes
    uint32_t kc = 0u, ties_take = 0u;
    if (cap < uint32_t(nb - nF)) {
      uint32_t prefix = 0u, need = cap;
      int known = 32;
      for (int pass = 0; pass < 3; ++pass) {
        const int width = pass < 2 ? 11 : 10, nbins = 1 << width, shift = known - width;
        for (int i = tid; i < kTpBins; i += kTpThreads) hist[i] = 0u;
        __syncthreads();
        tp_sweep(sc, nb, [&](int j, float x, bool in) {
          in = in && j != f0 && j != f1;
          const uint32_t key = in ? tp_key(x) : 0u;
          const bool hit = in && (known == 32 || (key >> known) == prefix);
          tp_count_add(hist, hit, (key >> shift) & uint32_t(nbins - 1));
        });
        __syncthreads();
        uint32_t above;
        const int bin = tp_find_count(hist, nbins < kTpThreads ? kTpThreads : nbins, need, s_u,
                                      &s_found, above);
        if (bin < 0) {                                 // cannot happen: cap < non-forced count
          if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
          break;
        }
        prefix = (prefix << width) | uint32_t(bin);
        known = shift;
        need -= above;
      }
      kc = prefix;
      ties_take = need;                                // blocks holding kc still to take
    }
    // the candidates compacted in index order: warp w owns [w E, w E + E)
    const int E = (nb + kTpThreads - 1) / kTpThreads * 32;
    const int j0 = warp * E, j1 = min(nb, j0 + E);
    unsigned n_gt = 0, n_eq = 0;
    for (int jb = j0; jb < j1; jb += 32) {
      const int j = jb + lane;
      const bool in = j < j1 && j != f0 && j != f1;
      const uint32_t key = in ? tp_key(tp_clean(sc[j])) : 0u;
      n_gt += __popc(__ballot_sync(kFull, in && key > kc));
      n_eq += __popc(__ballot_sync(kFull, in && key == kc));
    }
    unsigned eq_tot;
    const unsigned eq_before = tp_warp_scan(n_eq, s_w, eq_tot);
    const unsigned eq_take = eq_before >= ties_take ? 0u : min(n_eq, ties_take - eq_before);
    unsigned pos = tp_warp_scan(n_gt + eq_take, s_w, c_tot);
    unsigned eq_rank = eq_before;
    for (int jb = j0; jb < j1; jb += 32) {
      const int j = jb + lane;
      const bool in = j < j1 && j != f0 && j != f1;
      const uint32_t key = in ? tp_key(tp_clean(sc[j])) : 0u;
      const bool eq = in && key == kc;
      const unsigned em = __ballot_sync(kFull, eq), below = (1u << lane) - 1u;
      const bool take = (in && key > kc) || (eq && eq_rank + __popc(em & below) < ties_take);
      const unsigned tm = __ballot_sync(kFull, take);
      if (take) {
        const unsigned at = pos + __popc(tm & below);
        if (at < unsigned(kTpCandMax))
          cand[at] = ((unsigned long long)key << 32) | (0xffffffffu - uint32_t(j));
      }
      pos += __popc(tm);
      eq_rank += __popc(em);
    }
  }
  const int n_c = int(min(c_tot, unsigned(kTpCandMax)));
  const int n_top = min(n_c, int(cap));                // the cap best blocks at most
  __syncthreads();                                     // every candidate written

  // 4. The taken candidates, in the order decreasing beta, ties to the lower index: the
  // fewest whose mass with the forced blocks' reaches the goal, at most n_top. Instead of
  // sorting every candidate, a 2,048-bin histogram linear in the score over the candidates
  // (count and exact fixed-point mass per bin) finds, walking from the highest bin, the bin
  // gb where the count reaches n_top or the mass the remaining goal. Bins are monotone in
  // the score, so every candidate above gb is taken, and only gb's candidates are sorted
  // (key descending, index ascending) to take the first t_in of them.
  __shared__ unsigned s_nt;
  __shared__ int s_tin;
  int gb = kTpBins, t_in = 0;                          // no candidate taken
  uint32_t cnt_above = 0u;
  unsigned long long mass_above = 0ull;
  float cmin = 0.0f, cinv = 0.0f;
  if (n_top > 0 && MF < goal) {
    const unsigned long long need = goal - MF;
    float mx2 = -INFINITY, mn2 = INFINITY;
    for (int i = tid; i < n_c; i += kTpThreads) {
      const float x = tp_unkey(uint32_t(cand[i] >> 32));
      mx2 = fmaxf(mx2, x);
      mn2 = fminf(mn2, x);
    }
    const float cmax = tp_block_max(mx2, s_f);
    cmin = -tp_block_max(-mn2, s_f);
    cinv = cmax > cmin ? float(kTpBins) / (cmax - cmin) : 0.0f;
    for (int i = tid; i < kTpBins; i += kTpThreads) {
      hist[i] = 0u;
      hmass[i] = 0ull;
    }
    if (tid == 0) s_nt = 0u;
    __syncthreads();
    for (int i = tid; i < n_c; i += kTpThreads) {
      const float x = tp_unkey(uint32_t(cand[i] >> 32));
      const int bin = tp_lin_bin(x, cmin, cinv);
      atomicAdd(&hist[bin], 1u);
      atomicAdd(&hmass[bin], tp_mass(x, M));
    }
    __syncthreads();
    const TpFound f = tp_find(hist, hmass, kTpBins, uint32_t(n_top), need, s_u, &s_found);
    gb = f.bin;                                        // >= 0: the counts reach n_top
    cnt_above = f.cnt_above;
    mass_above = f.mass_above;
    if (gb < 0) {                                      // cannot happen; take no candidate
      if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
      gb = kTpBins;
    }
  }
  if (gb < kTpBins) {
    const unsigned long long need = goal - MF;
    // gb's candidates, then sorted
    for (int i = tid; i < n_c; i += kTpThreads) {
      const float x = tp_unkey(uint32_t(cand[i] >> 32));
      if (tp_lin_bin(x, cmin, cinv) == gb) tmp[atomicAdd(&s_nt, 1u)] = cand[i];
    }
    __syncthreads();
    const int n_t = int(s_nt);
    if (n_t <= 32) {
      if (warp == 0) {                                 // one warp: bitonic by shuffles
        unsigned long long v = lane < n_t ? tmp[lane] : 0ull;
#pragma unroll
        for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
          for (int jj = k >> 1; jj > 0; jj >>= 1) {
            const unsigned long long o = __shfl_xor_sync(kFull, v, jj);
            v = tp_keep(v, o, ((lane & jj) == 0) == ((lane & k) == 0));
          }
        tmp[lane] = v;
      }
      __syncthreads();
    } else {
      int n_pow = kTpThreads;                          // 1,024, 2,048 or 4,096 entries
      while (n_pow < n_t) n_pow <<= 1;
      for (int i = n_t + tid; i < n_pow; i += kTpThreads) tmp[i] = 0ull;   // below every key
      __syncthreads();
      if (n_pow == kTpThreads) tp_sort<1>(tmp);
      else if (n_pow == 2 * kTpThreads) tp_sort<2>(tmp);
      else tp_sort<4>(tmp);
    }
    // the first t_in of them: where the count reaches n_top or the mass the goal
    const int per = (n_t + kTpThreads - 1) / kTpThreads;     // consecutive entries per thread
    const int e0 = tid * per, e1 = min(n_t, e0 + per);
    unsigned long long loc = 0;
    for (int i = e0; i < e1; ++i) loc += tp_mass(tp_unkey(uint32_t(tmp[i] >> 32)), M);
    if (tid == 0) s_tin = n_t;
    unsigned long long tot_t;
    unsigned long long cum = mass_above + tp_scan(loc, s_u, tot_t);
    for (int i = e0; i < e1; ++i) {
      cum += tp_mass(tp_unkey(uint32_t(tmp[i] >> 32)), M);
      if (cnt_above + uint32_t(i) + 1u >= uint32_t(n_top) || cum >= need) {
        atomicMin(&s_tin, i + 1);
        break;
      }
    }
    __syncthreads();
    t_in = s_tin;
  }

  // 5. bitmap of the taken blocks, written out ascending
  const int words = (nb + 31) / 32;
  for (int i = tid; i < words; i += kTpThreads) bits[i] = 0u;
  __syncthreads();
  if (tid == 0) {
    if (f0 >= 0) atomicOr(&bits[f0 >> 5], 1u << (f0 & 31));
    if (f1 >= 0) atomicOr(&bits[f1 >> 5], 1u << (f1 & 31));
  }
  for (int i = tid; i < n_c && gb < kTpBins; i += kTpThreads) {   // the bins above gb
    if (tp_lin_bin(tp_unkey(uint32_t(cand[i] >> 32)), cmin, cinv) > gb) {
      const uint32_t j = 0xffffffffu - uint32_t(cand[i]);
      atomicOr(&bits[j >> 5], 1u << (j & 31));
    }
  }
  for (int i = tid; i < t_in; i += kTpThreads) {                  // the first t_in of gb
    const uint32_t j = 0xffffffffu - uint32_t(tmp[i]);
    atomicOr(&bits[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  const int wpt = (words + kTpThreads - 1) / kTpThreads;
  const int w0 = tid * wpt, w1 = min(words, w0 + wpt);
  unsigned long long my_n = 0;
  for (int i = w0; i < w1; ++i) my_n += __popc(bits[i]);
  unsigned long long n_tot;
  unsigned long long at = tp_scan(my_n, s_u, n_tot);
  for (int i = w0; i < w1; ++i) {
    uint32_t m = bits[i];
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1u;
      if (at < (unsigned long long)a.budget) out[at] = i * 32 + bit;
      else flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
      ++at;
    }
  }
  const int n = int(min(n_tot, (unsigned long long)a.budget));
  if (tid == 0) a.n_sel[row] = n;
  for (int i = n + tid; i < a.budget; i += kTpThreads) out[i] = -1;
}

cudaError_t launch_top_p(const TopPParams& a, cudaStream_t s) {
  if (a.budget <= kTpCandMax) {
    // candidates, histogram and the row's bitmap in dynamic shared memory
    const size_t smem = size_t(kTpCandMax) * 8 * 2 + size_t(kTpBins) * (8 + 4) +
                        size_t((a.nb_stride + 31) / 32) * 4;
    if (smem <= size_t(200) * 1024) {
      const cudaError_t e = set_smem_limit(top_p_sorted_kernel, int(200 * 1024));
      if (e != cudaSuccess) return e;
      top_p_sorted_kernel<<<a.rows, kTpThreads, smem, s>>>(a);
      return cudaGetLastError();
    }
  }
  top_p_kernel<<<a.rows, kTpThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace qs
