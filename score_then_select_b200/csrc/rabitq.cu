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
  for (int j = 0; j < D; ++j) y = __fadd_rn(y, __fmul_rn(s_qbar[j], Rg[size_t(j) * D + tid]));

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
constexpr int kRqPagesPerCta = 8;

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

// CTA = (8 pages, sequence b); warp = one (page, KV head) at a time, all of a page's heads
// (contiguous in the cache) handled by neighbouring warps.
template <int D, int S>
__global__ void __launch_bounds__(kRqScanWarps * 32) rq_score_kernel(const RqScoreParams a) {
  constexpr int W = D / 32;                            // code words per token
  constexpr int PB = kPage * (D / 8) + kPage * 4;      // bytes per (page, KV head)
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int L = a.seq_lens[b];
  if (L > a.max_context) {
    if (threadIdx.x == 0 && blockIdx.x == 0)
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(b));
    L = a.max_context;
  }
  const int pages = L > 0 ? (L + kPage - 1) / kPage : 0;
  const int max_pages = a.nb_stride / (kPage / S);
  const int p0 = blockIdx.x * kRqPagesPerCta;
  for (int it = warp; it < kRqPagesPerCta * a.Hkv; it += kRqScanWarps) {
    const int pi = p0 + it / a.Hkv, g = it % a.Hkv;
    if (pi >= pages || pi >= max_pages) continue;
    const int row = b * a.Hkv + g;
    int page = -1;
    if (pi < a.max_pages_per_seq) page = a.page_table[size_t(b) * a.max_pages_per_seq + pi];
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(row));
      continue;
    }
    const uint8_t* pg = a.proxy + (size_t(page) * a.Hkv + g) * PB;
    // the page's codes and factors first, then the row's query code
    uint32_t code[4][W];
    float gk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int slot = lane + 32 * k;
      if constexpr (W == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(pg + slot * 16);
        code[k][0] = v.x;
        code[k][1] = v.y;
        code[k][2] = v.z;
        code[k][3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(pg + slot * 8);
        code[k][0] = v.x;
        code[k][1] = v.y;
      }
      gk[k] = reinterpret_cast<const float*>(pg + kPage * (D / 8))[slot];
    }
    const uint32_t* qc = a.qcode + size_t(row) * kRqRowWords;
    uint32_t plane[kRqBits][W];
#pragma unroll
    for (int p = 0; p < kRqBits; ++p)
#pragma unroll
      for (int w = 0; w < W; ++w) plane[p][w] = qc[p * W + w];
    const float delta = __uint_as_float(qc[kRqDelta]), vl = __uint_as_float(qc[kRqVl]);
    const float shift = __uint_as_float(qc[kRqShift]);
    const int Q = int(qc[kRqQsum]);

    float m[4], l[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int A = 0, B = 0;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        B += __popc(code[k][w]);
#pragma unroll
        for (int p = 0; p < kRqBits; ++p) A += __popc(code[k][w] & plane[p][w]) << p;
      }
      const float est = gk[k] * (delta * float(2 * A - Q) + vl * float(2 * B - D)) + shift;
      const bool valid = pi * kPage + lane + 32 * k < L;
      m[k] = valid ? a.scale * est : -INFINITY;
      l[k] = valid ? 1.0f : 0.0f;
    }
    float* out = a.scores + size_t(row) * a.nb_stride + size_t(pi) * (kPage / S);
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
}

template <int D>
static cudaError_t launch_rq_score_d(const RqScoreParams& a, cudaStream_t s) {
  const int max_pages = a.nb_stride / (kPage / a.S);
  const dim3 grid((max_pages + kRqPagesPerCta - 1) / kRqPagesPerCta, a.batch);
  const dim3 block(kRqScanWarps * 32);
  switch (a.S) {
    case 1: rq_score_kernel<D, 1><<<grid, block, 0, s>>>(a); break;
    case 2: rq_score_kernel<D, 2><<<grid, block, 0, s>>>(a); break;
    case 4: rq_score_kernel<D, 4><<<grid, block, 0, s>>>(a); break;
    case 8: rq_score_kernel<D, 8><<<grid, block, 0, s>>>(a); break;
    case 16: rq_score_kernel<D, 16><<<grid, block, 0, s>>>(a); break;
    case 32: rq_score_kernel<D, 32><<<grid, block, 0, s>>>(a); break;
    case 64: rq_score_kernel<D, 64><<<grid, block, 0, s>>>(a); break;
    case 128: rq_score_kernel<D, 128><<<grid, block, 0, s>>>(a); break;
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

// Is block j taken? tie_rank counts the blocks with key kstar met so far.
QS_DEV bool tp_taken(const float* sc, int j, int f0, int f1, int mode, uint32_t kstar,
                     uint32_t ties, unsigned long long& tie_rank) {
  if (j == f0 || j == f1 || mode == 1) return true;
  if (mode == 0) return false;
  const uint32_t key = tp_key(tp_clean(sc[j]));
  if (key > kstar) return true;
  if (key == kstar) return tie_rank++ < ties;
  return false;
}

__global__ void __launch_bounds__(kTpThreads, 1) top_p_kernel(const TopPParams a) {
  __shared__ uint32_t h_cnt[kTpBins];
  __shared__ unsigned long long h_mass[kTpBins];
  __shared__ unsigned long long s_u[kTpThreads / 32];
  __shared__ float s_f[kTpThreads / 32];
  __shared__ TpFound s_found;
  const int row = blockIdx.x, b = row / a.Hkv, tid = threadIdx.x;
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
  for (int j = tid; j < nb; j += kTpThreads) mx = fmaxf(mx, tp_clean(sc[j]));
  const float M = tp_block_max(mx, s_f);

  // Z, the forced blocks' mass, and the histogram of the others' top 11 key bits
  for (int i = tid; i < kTpBins; i += kTpThreads) {
    h_cnt[i] = 0u;
    h_mass[i] = 0ull;
  }
  __syncthreads();
  unsigned long long z = 0, mf = 0;
  for (int j = tid; j < nb; j += kTpThreads) {
    const float x = tp_clean(sc[j]);
    const unsigned long long w = tp_mass(x, M);
    z += w;
    if (j == f0 || j == f1) {
      mf += w;
    } else {
      const uint32_t bin = tp_key(x) >> 21;
      atomicAdd(&h_cnt[bin], 1u);
      atomicAdd(&h_mass[bin], w);
    }
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
        for (int j = tid; j < nb; j += kTpThreads) {
          if (j == f0 || j == f1) continue;
          const float x = tp_clean(sc[j]);
          const uint32_t key = tp_key(x);
          if ((key >> known) != prefix) continue;
          const uint32_t bin = (key >> shift) & uint32_t(nbins - 1);
          atomicAdd(&h_cnt[bin], 1u);
          atomicAdd(&h_mass[bin], tp_mass(x, M));
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

  // output, ascending: thread t owns blocks [t C, t C + C)
  const int C = (nb + kTpThreads - 1) / kTpThreads;
  const int j0 = min(nb, tid * C), j1 = min(nb, j0 + C);
  unsigned long long my_ties = 0;
  if (mode == 2)
    for (int j = j0; j < j1; ++j)
      my_ties += (j != f0 && j != f1 && tp_key(tp_clean(sc[j])) == kstar);
  unsigned long long tie_tot;
  const unsigned long long tie0 = tp_scan(my_ties, s_u, tie_tot);
  unsigned long long my_n = 0, tr = tie0;
  for (int j = j0; j < j1; ++j) my_n += tp_taken(sc, j, f0, f1, mode, kstar, ties, tr);
  unsigned long long n_tot;
  unsigned long long pos = tp_scan(my_n, s_u, n_tot);
  tr = tie0;
  for (int j = j0; j < j1; ++j) {
    if (!tp_taken(sc, j, f0, f1, mode, kstar, ties, tr)) continue;
    if (pos < (unsigned long long)a.budget) out[pos] = j;
    else flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
    ++pos;
  }
  const int n = int(min(n_tot, (unsigned long long)a.budget));
  if (tid == 0) a.n_sel[row] = n;
  for (int i = n + tid; i < a.budget; i += kTpThreads) out[i] = -1;
}

cudaError_t launch_top_p(const TopPParams& a, cudaStream_t s) {
  top_p_kernel<<<a.rows, kTpThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace qs
