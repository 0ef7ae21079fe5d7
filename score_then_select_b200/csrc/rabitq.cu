// rabitq.cu - the binary-code scan and the top-p selection ("RaBitQCache", Abstract).
//
//   rq_prep_kernel:  CTA = one row (sequence b, KV head g), thread i = dimension i. The
//                    group-mean query qbar (head sum in order, divided by G), q' = qbar R[g]
//                    (j ascending, one rounding per product and per sum), v_l = min q',
//                    Delta = (max q' - v_l) / 15, codes n_i = min(15, floor((q'_i - v_l) /
//                    Delta + u_i)) (all 0 when Delta = 0), stored as 4 bit planes, with
//                    Delta, v_l, sum n_i and c . qbar. Every step is a rounded float32
//                    operation, so the codes are those of the float32 definition.
//   rq_score_kernel: one warp per (page, KV head): lane l scores token slots l + 32k,
//                    k < 4. With A = sum_p 2^p popc(b & plane_p) and B = popc(b),
//                      s = g (Delta (2A - Q) + v_l (2B - d)) + c . qbar
//                    = g sum_i (2 b_i - 1)(Delta n_i + v_l) + c . qbar (the RaBitQ estimate
//                    of q . k, Gao and Long, SIGMOD 2024, section 3), then each block's
//                    log-sum-exp of scale * s over its valid tokens (the log of its
//                    estimated attention mass up to the row's normaliser).
//   top_p_kernel:    CTA = one row; see its comment.
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
  }
}

cudaError_t launch_rq_prep(const RqPrepParams& a, cudaStream_t s) {
  if (a.d == 128) rq_prep_kernel<128><<<a.batch * a.Hkv, 128, 0, s>>>(a);
  else rq_prep_kernel<64><<<a.batch * a.Hkv, 64, 0, s>>>(a);
  return cudaGetLastError();
}

// ============================================================ scan
constexpr int kRqScanWarps = 8;

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

// Persistent grid; a unit is one (sequence b, page p, KV head g), g fastest so that a
// page's heads (contiguous in the cache) go to neighbouring warps. Warp w of the grid takes
// units w, w + W, ... and loads the next unit's codes, factors and query code before it
// scores the current one, so every warp keeps a unit's loads in flight.
struct RqUnit {
  int row, pi, L;
  bool ok;
  const uint8_t* pg;
};

template <int D>
QS_DEV RqUnit rq_unit(const RqScoreParams& a, long long u, int max_pages) {
  RqUnit x{0, 0, 0, false, nullptr};
  const long long per_b = (long long)max_pages * a.Hkv;
  const int b = int(u / per_b);
  const int rem = int(u - (long long)b * per_b);
  x.pi = rem / a.Hkv;
  const int g = rem - x.pi * a.Hkv;
  x.row = b * a.Hkv + g;
  int L = a.seq_lens[b];
  if (L > a.max_context) {
    if (x.pi == 0 && g == 0 && (threadIdx.x & 31) == 0)
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(b));
    L = a.max_context;
  }
  x.L = L;
  const int pages = L > 0 ? (L + kPage - 1) / kPage : 0;
  if (x.pi >= pages) return x;                         // past the row's tokens: nothing
  int page = -1;
  if (x.pi < a.max_pages_per_seq) page = a.page_table[size_t(b) * a.max_pages_per_seq + x.pi];
  if (page < 0 || page >= a.num_pages) {
    if ((threadIdx.x & 31) == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(x.row));
    return x;
  }
  constexpr int PB = kPage * (D / 8) + kPage * 4;
  x.pg = a.proxy + (size_t(page) * a.Hkv + g) * PB;
  x.ok = true;
  return x;
}

template <int D>
struct RqLoad {                                        // one lane's share of a unit's codes
  uint32_t code[4][D / 32];
  float gk[4];
};

template <int D>
QS_DEV void rq_load(const RqScoreParams& a, const RqUnit& x, int lane, RqLoad<D>& r) {
  constexpr int W = D / 32;
  if (!x.ok) return;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int slot = lane + 32 * k;
    if constexpr (W == 4) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(x.pg + slot * 16));
      r.code[k][0] = v.x;
      r.code[k][1] = v.y;
      r.code[k][2] = v.z;
      r.code[k][3] = v.w;
    } else {
      const uint2 v = __ldcs(reinterpret_cast<const uint2*>(x.pg + slot * 8));
      r.code[k][0] = v.x;
      r.code[k][1] = v.y;
    }
    r.gk[k] = __ldcs(reinterpret_cast<const float*>(x.pg + kPage * (D / 8)) + slot);
  }
}

template <int D, int S>
QS_DEV void rq_score_unit(const RqScoreParams& a, const RqUnit& x, const RqLoad<D>& r, int lane) {
  constexpr int W = D / 32;
  // the row's query code (a few hundred bytes per row, cached close to the SM)
  const uint32_t* qc = a.qcode + size_t(x.row) * kRqRowWords;
  uint32_t plane[kRqBits][W];
#pragma unroll
  for (int p = 0; p < kRqBits; ++p)
#pragma unroll
    for (int w = 0; w < W; ++w) plane[p][w] = __ldg(qc + p * W + w);
  const float delta = __uint_as_float(__ldg(qc + kRqDelta)), vl = __uint_as_float(__ldg(qc + kRqVl));
  const float shift = __uint_as_float(__ldg(qc + kRqShift));
  const int Q = int(__ldg(qc + kRqQsum));
  float m[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int A = 0, B = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      B += __popc(r.code[k][w]);
#pragma unroll
      for (int p = 0; p < kRqBits; ++p) A += __popc(r.code[k][w] & plane[p][w]) << p;
    }
    const float est = r.gk[k] * (delta * float(2 * A - Q) + vl * float(2 * B - D)) + shift;
    const bool valid = x.pi * kPage + lane + 32 * k < x.L;
    m[k] = valid ? a.scale * est : -INFINITY;
    l[k] = valid ? 1.0f : 0.0f;
  }
  float* out = a.scores + size_t(x.row) * a.nb_stride + size_t(x.pi) * (kPage / S);
  if constexpr (S < 32) {
    // a block = S neighbouring lanes of one k
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float mk = m[k], lk = l[k];
#pragma unroll
      for (int o = 1; o < S; o <<= 1) {
        const float m2 = __shfl_xor_sync(kFull, mk, o), l2 = __shfl_xor_sync(kFull, lk, o);
        lse_merge(mk, lk, m2, l2);
      }
      if ((lane & (S - 1)) == 0) out[(lane + 32 * k) / S] = lk > 0.0f ? mk + logf(lk) : -INFINITY;
    }
  } else {
    // a block = S / 32 consecutive k of every lane
    constexpr int KB = S / 32;
#pragma unroll
    for (int k0 = 0; k0 < 4; k0 += KB) {
      float mk = m[k0], lk = l[k0];
#pragma unroll
      for (int k = k0 + 1; k < k0 + KB; ++k) lse_merge(mk, lk, m[k], l[k]);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float m2 = __shfl_xor_sync(kFull, mk, o), l2 = __shfl_xor_sync(kFull, lk, o);
        lse_merge(mk, lk, m2, l2);
      }
      if (lane == 0) out[(32 * k0) / S] = lk > 0.0f ? mk + logf(lk) : -INFINITY;
    }
  }
}

template <int D, int S>
__global__ void __launch_bounds__(kRqScanWarps * 32) rq_score_kernel(const RqScoreParams a) {
  const int lane = threadIdx.x & 31;
  const int max_pages = a.nb_stride / (kPage / S);
  const long long units = (long long)a.batch * max_pages * a.Hkv;
  const long long stride = (long long)gridDim.x * kRqScanWarps;
  long long u = (long long)blockIdx.x * kRqScanWarps + (threadIdx.x >> 5);
  if (u >= units) return;
  RqUnit x = rq_unit<D>(a, u, max_pages);
  RqLoad<D> cur;
  rq_load<D>(a, x, lane, cur);
  while (true) {
    const long long un = u + stride;
    RqUnit xn{0, 0, 0, false, nullptr};
    RqLoad<D> nxt;
    if (un < units) {
      xn = rq_unit<D>(a, un, max_pages);
      rq_load<D>(a, xn, lane, nxt);                    // in flight while this unit is scored
    }
    if (x.ok) rq_score_unit<D, S>(a, x, cur, lane);
    if (un >= units) break;
    u = un;
    x = xn;
    cur = nxt;
  }
}

template <int D>
static cudaError_t launch_rq_score_d(const RqScoreParams& a, cudaStream_t s) {
  const int max_pages = a.nb_stride / (kPage / a.S);
  const long long warps = (long long)a.batch * max_pages * a.Hkv;
  static const int per_sm = [] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, rq_score_kernel<D, 1>,
                                                      kRqScanWarps * 32, 0) != cudaSuccess)
      n = 0;
    return n > 0 ? n : 1;
  }();
  long long grid = (long long)num_sms() * per_sm;
  const long long need = (warps + kRqScanWarps - 1) / kRqScanWarps;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  const dim3 block(kRqScanWarps * 32);
  switch (a.S) {
    case 1: rq_score_kernel<D, 1><<<unsigned(grid), block, 0, s>>>(a); break;
    case 2: rq_score_kernel<D, 2><<<unsigned(grid), block, 0, s>>>(a); break;
    case 4: rq_score_kernel<D, 4><<<unsigned(grid), block, 0, s>>>(a); break;
    case 8: rq_score_kernel<D, 8><<<unsigned(grid), block, 0, s>>>(a); break;
    case 16: rq_score_kernel<D, 16><<<unsigned(grid), block, 0, s>>>(a); break;
    case 32: rq_score_kernel<D, 32><<<unsigned(grid), block, 0, s>>>(a); break;
    case 64: rq_score_kernel<D, 64><<<unsigned(grid), block, 0, s>>>(a); break;
    case 128: rq_score_kernel<D, 128><<<unsigned(grid), block, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
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

QS_DEV float tp_clean(float x) { return x != x ? -INFINITY : fminf(x, FLT_MAX); }
QS_DEV uint32_t tp_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
QS_DEV unsigned long long tp_mass(float x, float M) {
  if (!(M > -INFINITY)) return 0ull;
  return __float2ull_rn(expf(x - M) * kTpUnit);
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
  const int nb_up = (nb + kTpThreads - 1) / kTpThreads * kTpThreads;   // whole warps per step

  // the row's largest score
  float mx = -INFINITY;
  for (int j = tid; j < nb; j += kTpThreads) mx = fmaxf(mx, tp_clean(sc[j]));
  const float M = tp_block_max(mx, s_f);

  // Z, the forced blocks' mass, and the histogram of the others' top 11 key bits
  for (int i = tid; i < kTpBins; i += kTpThreads) {
    h_cnt[i] = 0u;
    h_mass[i] = 0ull;
  }
  __syncthreads();
  unsigned long long z = 0, mf = 0;
  for (int j = tid; j < nb_up; j += kTpThreads) {
    const bool in = j < nb;
    const float x = in ? tp_clean(sc[j]) : -INFINITY;
    const unsigned long long w = in ? tp_mass(x, M) : 0ull;
    const bool forced = j == f0 || j == f1;
    z += w;
    if (forced) mf += w;
    tp_hist_add(h_cnt, h_mass, in && !forced, tp_key(x) >> 21, w);
  }
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
        for (int j = tid; j < nb_up; j += kTpThreads) {
          const bool in = j < nb && j != f0 && j != f1;
          const float x = in ? tp_clean(sc[j]) : -INFINITY;
          const uint32_t key = tp_key(x);
          const bool hit = in && (key >> known) == prefix;
          tp_hist_add(h_cnt, h_mass, hit, (key >> shift) & uint32_t(nbins - 1),
                      hit ? tp_mass(x, M) : 0ull);
        }
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
// kTpCandMax blocks (the token-level budgets of the pages: B = 2,048):
//   1. M, Z and the forced mass as above (per-thread 64-bit sums, then a block scan);
//   2. the key of the cap-th best non-forced block (cap = budget minus the forced blocks)
//      by three count-only histogram passes (11, 11 and 10 bits; 32-bit counts, lanes of a
//      warp that share a bin combined first);
//   3. the candidates: the non-forced blocks above that key and the first blocks (in index
//      order) holding it, cap at most, compacted into shared memory as 64-bit sort keys
//      (key << 32 | ~index) and bitonic-sorted, largest first: decreasing beta, ties to the
//      lower index, exactly the order in which blocks are taken;
//   4. their masses in that order, an exact prefix sum, and the number taken: the fewest
//      whose mass with the forced blocks' reaches the goal, else all of them;
//   5. the taken blocks and the forced ones marked in a bitmap of the row, written out in
//      ascending order.
constexpr int kTpCandMax = 4096;

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

__global__ void __launch_bounds__(kTpThreads, 1) top_p_sorted_kernel(const TopPParams a) {
  extern __shared__ __align__(16) uint8_t tp_smem[];
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(tp_smem);   // [kTpCandMax]
  uint32_t* hist = reinterpret_cast<uint32_t*>(cand + kTpCandMax);             // [kTpBins]
  uint32_t* bits = hist + kTpBins;                                              // [row words]
  __shared__ unsigned long long s_u[kTpThreads / 32];
  __shared__ unsigned s_w[kTpThreads / 32];
  __shared__ float s_f[kTpThreads / 32];
  __shared__ TpFound s_found;
  __shared__ int s_take;
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
  const int nb_up = (nb + kTpThreads - 1) / kTpThreads * kTpThreads;

  // 1. the row's largest score; Z and the forced mass
  float mx = -INFINITY;
  for (int j = tid; j < nb; j += kTpThreads) mx = fmaxf(mx, tp_clean(sc[j]));
  const float M = tp_block_max(mx, s_f);
  unsigned long long z = 0, mf = 0;
  for (int j = tid; j < nb; j += kTpThreads) {
    const unsigned long long w = tp_mass(tp_clean(sc[j]), M);
    z += w;
    if (j == f0 || j == f1) mf += w;
  }
  unsigned long long Z, MF;
  tp_scan(z, s_u, Z);
  tp_scan(mf, s_u, MF);
  unsigned long long goal = (unsigned long long)ceil(double(a.p) * double(Z));
  if (goal > Z) goal = Z;
  const uint32_t cap = uint32_t(max(0, min(a.budget - nF, nb - nF)));

  // 2. the key of the cap-th best non-forced block (all of them if cap covers them, none
  // if cap is 0: no key lies above 0xffffffff)
  uint32_t kc = cap == 0 ? 0xffffffffu : 0u, ties_take = 0u;
  if (cap > 0 && cap < uint32_t(nb - nF)) {
    uint32_t prefix = 0u, need = cap;
    int known = 32;
    for (int pass = 0; pass < 3; ++pass) {
      const int width = pass < 2 ? 11 : 10, nbins = 1 << width, shift = known - width;
      for (int i = tid; i < kTpBins; i += kTpThreads) hist[i] = 0u;
      __syncthreads();
      for (int j = tid; j < nb_up; j += kTpThreads) {
        const bool in = j < nb && j != f0 && j != f1;
        const uint32_t key = in ? tp_key(tp_clean(sc[j])) : 0u;
        const bool hit = in && (known == 32 || (key >> known) == prefix);
        tp_count_add(hist, hit, (key >> shift) & uint32_t(nbins - 1));
      }
      __syncthreads();
      uint32_t above;
      const int bin = tp_find_count(hist, nbins < kTpThreads ? kTpThreads : nbins, need, s_u,
                                    &s_found, above);
      if (bin < 0) {                                   // cannot happen: cap < non-forced count
        if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
        break;
      }
      prefix = (prefix << width) | uint32_t(bin);
      known = shift;
      need -= above;
    }
    kc = prefix;
    ties_take = need;                                  // blocks holding kc still to take
  }

  // 3. the candidates, compacted in index order: warp w owns [w E, w E + E)
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
  unsigned eq_tot, c_tot;
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
  const int n_c = int(min(c_tot, unsigned(kTpCandMax)));
  int n_pow = 1;
  while (n_pow < n_c) n_pow <<= 1;
  for (int i = n_c + tid; i < n_pow; i += kTpThreads) cand[i] = 0ull;   // below every block
  __syncthreads();
  // bitonic sort, largest first
  if (n_c > 1) {
    for (int k = 2; k <= n_pow; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
        for (int i = tid; i < n_pow; i += kTpThreads) {
          const int ixj = i ^ jj;
          if (ixj > i) {
            const unsigned long long x = cand[i], y = cand[ixj];
            if (((i & k) == 0) ? (x < y) : (x > y)) {
              cand[i] = y;
              cand[ixj] = x;
            }
          }
        }
        __syncthreads();
      }
    }
  }

  // 4. masses in that order; the fewest whose mass with the forced blocks reaches the goal
  const int per = (n_pow + kTpThreads - 1) / kTpThreads;     // consecutive entries per thread
  const int e0 = tid * per;
  unsigned long long loc = 0;
  for (int i = e0; i < min(n_c, e0 + per); ++i)
    loc += tp_mass(tp_clean(sc[0xffffffffu - uint32_t(cand[i])]), M);
  if (tid == 0) s_take = n_c;
  unsigned long long tot_c;
  unsigned long long cum = MF + tp_scan(loc, s_u, tot_c);
  if (MF >= goal) {
    if (tid == 0) s_take = 0;
  } else {
    for (int i = e0; i < min(n_c, e0 + per); ++i) {
      cum += tp_mass(tp_clean(sc[0xffffffffu - uint32_t(cand[i])]), M);
      if (cum >= goal) {
        atomicMin(&s_take, i + 1);
        break;
      }
    }
  }
  __syncthreads();
  const int n_take = s_take;

  // 5. bitmap of the taken blocks, written out ascending
  const int words = (nb + 31) / 32;
  for (int i = tid; i < words; i += kTpThreads) bits[i] = 0u;
  __syncthreads();
  if (tid == 0) {
    if (f0 >= 0) atomicOr(&bits[f0 >> 5], 1u << (f0 & 31));
    if (f1 >= 0) atomicOr(&bits[f1 >> 5], 1u << (f1 & 31));
  }
  for (int i = tid; i < n_take; i += kTpThreads) {
    const uint32_t j = 0xffffffffu - uint32_t(cand[i]);
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
    const size_t smem = size_t(kTpCandMax) * 8 + size_t(kTpBins) * 4 +
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
