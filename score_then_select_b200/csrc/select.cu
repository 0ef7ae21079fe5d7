// select.cu - per-row top-k block selection.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1 and
// Table 15: each KV head selects its own top-B positions, shared by its query heads.
// "Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention", Full text:
// blocks kept at full precision are always attended.
//
// Result (deterministic): if nb <= k every block; otherwise the forced set F (sink, last,
// kept) plus the k - |F| best other blocks by score, equal scores ordered by lower index;
// ascending.
//
// Algorithm, one CTA per row. Warp w owns the contiguous blocks w * 32 * ITEMS ..
// (w + 1) * 32 * ITEMS - 1; lane l holds its blocks l, l + 32, ... in registers, so loads
// coalesce and index order is (warp, item, lane):
//   1. the score loads are issued first; forced blocks are marked by their owners (the
//      kept blocks are the n_keep complete blocks with the largest block error, found by
//      two block-wide arg-max reductions);
//   2. one pass of a 2048-bin histogram that is linear in the score between the active
//      minimum and maximum (a monotone map, so every block in a higher bin scores higher)
//      selects every bin above the threshold bin and leaves only the threshold bin active;
//      the bins stay packed in registers for the classification;
//   3. the few blocks left in the threshold bin are ranked pairwise (score descending,
//      index ascending) and kept by their owners if ranked within the need; only if many
//      are left (many equal or nearly equal scores) does an exact MSB-first radix select
//      (4 x 8-bit digits) over order-preserving uint32 keys narrow them to one key value;
//   4. the remaining slots go to the lowest-indexed blocks holding that key;
//   5. the ascending indices are written with one ballot per item and a prefix over warps.
// The count left in the threshold bin is read from the histogram, so no extra block-wide
// reduction is needed between passes.
#include <cfloat>
#include <cooperative_groups.h>

#include "qs_device.cuh"

namespace qs {

constexpr int kLinBins = 2048;
constexpr int kRankCap = 1024;     // candidates ranked pairwise after the histogram pass

// float -> uint32 whose unsigned order is the float order (NaN ranks as -FLT_MAX, -0 == +0)
QS_DEV uint32_t order_key(float v) {
  if (v != v) v = -FLT_MAX;
  if (v == 0.0f) v = 0.0f;
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NT>
struct BlockOps {
  static constexpr int NW = NT / 32;
  int* s_i;      // [NW + 1]
  float* s_f;    // [2 * NW + 2]

  // exclusive prefix sum over threads; total via *total
  QS_DEV int exclusive_sum(int v, int* total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_i[w] = x;
    __syncthreads();
    if (w == 0) {
      int t = lane < NW ? s_i[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, t, o);
        if (lane >= o) t += y;
      }
      if (lane < NW) s_i[lane] = t;              // inclusive warp totals
      if (lane == NW - 1) s_i[NW] = t;
    }
    __syncthreads();
    const int before = (w == 0 ? 0 : s_i[w - 1]) + x - v;
    *total = s_i[NW];
    __syncthreads();
    return before;
  }
  QS_DEV int sum(int v) {
    int t;
    exclusive_sum(v, &t);
    return t;
  }
  QS_DEV void minmax(float& lo, float& hi) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    lo = warp_min(lo);
    hi = warp_max(hi);
    if (lane == 0) { s_f[w] = lo; s_f[NW + w] = hi; }
    __syncthreads();
    if (w == 0) {                                  // warp 0 combines the warps' results
      float a = lane < NW ? s_f[lane] : FLT_MAX, b = lane < NW ? s_f[NW + lane] : -FLT_MAX;
      a = warp_min(a);
      b = warp_max(b);
      if (lane == 0) { s_f[2 * NW] = a; s_f[2 * NW + 1] = b; }
    }
    __syncthreads();
    lo = s_f[2 * NW];
    hi = s_f[2 * NW + 1];
  }
  // arg-max of (value, -index) over the CTA; returns the index (or -1 if none valid)
  QS_DEV int argmax(float v, int idx) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    unsigned long long key = idx < 0 ? 0ull
                                     : ((unsigned long long)order_key(v) << 32) |
                                           (0xffffffffu - uint32_t(idx));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(kFull, key, o);
      key = y > key ? y : key;
    }
    __shared__ unsigned long long s_k[NW];
    if (lane == 0) s_k[w] = key;
    __syncthreads();
    unsigned long long best = 0ull;
    for (int i = 0; i < NW; ++i) best = s_k[i] > best ? s_k[i] : best;
    __syncthreads();
    return best == 0ull ? -1 : int(0xffffffffu - uint32_t(best & 0xffffffffull));
  }
};

// Threshold bin search over a histogram: the largest bin b with (#active in bins >= b)
// >= need. Writes the count strictly above b.
template <int NT>
QS_DEV void find_threshold_bin(const int* hist, int nbins, int need, int* s_bin, int* s_above,
                               BlockOps<NT>& ops) {
  // suffix sums: process bins from the top; thread t owns a contiguous range of bins
  constexpr int MAXPER = (kLinBins + NT - 1) / NT;
  const int per = (nbins + NT - 1) / NT;
  // thread t owns bins [nbins - (t+1)*per, nbins - t*per) (top bins for low t)
  const int hi_b = nbins - int(threadIdx.x) * per;
  const int lo_b = max(hi_b - per, 0);
  int local = 0;
  for (int bn = lo_b; bn < hi_b; ++bn) local += hist[bn];
  int total;
  const int above_me = ops.exclusive_sum(local, &total);  // count in bins above my range
  if (above_me < need && above_me + local >= need) {
    int acc = above_me;
    for (int bn = hi_b - 1; bn >= lo_b; --bn) {
      if (acc + hist[bn] >= need) {
        *s_bin = bn;
        *s_above = acc;
        break;
      }
      acc += hist[bn];
    }
  }
  (void)MAXPER;
  __syncthreads();
}

// NaN ranks lowest (fmaxf returns the other operand); +-inf are clamped to +-FLT_MAX
QS_DEV float sanitize(float x) { return fminf(fmaxf(x, -FLT_MAX), FLT_MAX); }

// Exclusive prefix of one value per warp (lane 0's `v`) over the CTA's warps, and the total;
// every lane of warp w receives the sum over warps 0 .. w-1.
template <int NW>
QS_DEV int warp_exclusive(int v, int* s_w, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) s_w[w] = v;
  __syncthreads();
  int x = lane < NW ? s_w[lane] : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  const int before = __shfl_sync(kFull, x, w) - __shfl_sync(kFull, lane < NW ? s_w[lane] : 0, w);
  *total = __shfl_sync(kFull, x, NW - 1);
  __syncthreads();
  return before;
}

// Transpose of a 32 x 32 bit matrix held one row per lane (bit c of lane r = M[r][c]): lane
// c receives column c (bit r = M[r][c]). Five rounds swap the off-diagonal j x j blocks.
QS_DEV uint32_t transpose32(uint32_t x, int lane) {
  const uint32_t hi[5] = {0xFFFF0000u, 0xFF00FF00u, 0xF0F0F0F0u, 0xCCCCCCCCu, 0xAAAAAAAAu};
#pragma unroll
  for (int t = 0; t < 5; ++t) {
    const int j = 16 >> t;
    const uint32_t y = __shfl_xor_sync(kFull, x, j);
    // the row with bit j set keeps its right half and takes its partner's right half into
    // its left half; the other keeps its left half and takes the partner's left half
    x = (lane & j) ? ((x & hi[t]) | ((y & hi[t]) >> j)) : ((x & ~hi[t]) | ((y & ~hi[t]) << j));
  }
  return x;
}

// CL > 1: a cluster of CL CTAs shares one row (CTA rank c holds blocks c * CAP ..
// (c + 1) * CAP - 1); the minimum and maximum, the histograms, the candidate list and the
// output offsets are combined through distributed shared memory between cluster barriers.
template <int NT, int ITEMS, int CL>
__global__ void __launch_bounds__(NT) select_kernel(const SelectParams a) {
  namespace cg = cooperative_groups;
  constexpr int NW = NT / 32;
  constexpr int CAP = NT * ITEMS;                 // blocks one CTA can hold
  constexpr int SPAN = 32 * ITEMS;                // blocks of one warp (contiguous)
  __shared__ int s_i[NW + 1];
  __shared__ float s_f[2 * NW + 2];
  __shared__ int hist[kLinBins];
  __shared__ int hsum[CL > 1 ? kLinBins : 1];     // cluster-wide histogram
  __shared__ float list_v[kRankCap];
  __shared__ int list_j[kRankCap];
  __shared__ int s_bin, s_above, s_cnt, s_forced[4], s_nforced;
  __shared__ int s_ctot;
  __shared__ float s_mm[2];
  __shared__ uint32_t s_out[NW * 64];
  BlockOps<NT> ops{s_i, s_f};

  pdl_wait();      // the scores come from the kernel before
  pdl_trigger();
  int crank = 0;
  if constexpr (CL > 1) crank = int(cg::this_cluster().block_rank());
  auto csync = [&]() {
    if constexpr (CL > 1) cg::this_cluster().sync();
  };
  // exclusive prefix of one value per CTA over the cluster's ranks, and the total
  auto cluster_prefix = [&](int v, int* total) {
    if constexpr (CL > 1) {
      if (threadIdx.x == 0) s_ctot = v;
      csync();
      int before = 0, all = 0;
      for (int r = 0; r < CL; ++r) {
        const int x = *cg::this_cluster().map_shared_rank(&s_ctot, r);
        all += x;
        if (r < crank) before += x;
      }
      csync();
      *total = all;
      return before;
    } else {
      *total = v;
      return 0;
    }
  };
  // replaces the CTA's histogram of `nbins` bins by the cluster-wide sum (in hsum)
  auto cluster_hist = [&](int nbins) -> const int* {
    if constexpr (CL > 1) {
      csync();
      for (int i = threadIdx.x; i < nbins; i += NT) {
        int x = 0;
        for (int r = 0; r < CL; ++r) x += cg::this_cluster().map_shared_rank(hist, r)[i];
        hsum[i] = x;
      }
      csync();
      return hsum;
    } else {
      return hist;
    }
  };
  const int row = blockIdx.x / CL;
  const int b = row / a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // item i of this thread is block j = rank * CAP + warp * SPAN + i * 32 + lane: each warp
  // owns a contiguous range (index order = rank, warp, item, lane) and its loads coalesce
  const int jbase = crank * CAP;
  const int jw = jbase + warp * SPAN + lane;
  const float* sc = a.scores + size_t(row) * a.nb_stride;
  const int nb_cap = a.nb_stride < CL * CAP ? a.nb_stride : CL * CAP;
  // the loads are issued before the row length arrives: every entry of the row's stride is
  // readable, and blocks at or past nb are masked out below
  float v[ITEMS];
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) v[i] = (jw + i * 32 < nb_cap) ? sc[jw + i * 32] : -FLT_MAX;
  int L = a.seq_lens[b];
  int nb = int((static_cast<long long>(L) + a.S - 1) / a.S);
  if (L < 0 || nb > nb_cap) {
    if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
    nb = L < 0 ? 0 : nb_cap;
    if (L < 0) L = 0;
  }
  int32_t* sel = a.sel + size_t(row) * a.budget;
  const int k = a.budget;
  const int n_out = nb < k ? nb : k;
  if (tid == 0 && crank == 0) a.n_sel[row] = n_out;

  if (nb <= k) {  // the budget covers every block (the same branch in every CTA of a cluster)
    if (crank == 0)
      for (int i = tid; i < k; i += NT) sel[i] = i < nb ? i : -1;
    return;
  }

  // ---------------- forced blocks: sink, last, and the kept (largest-error) blocks
  if (a.n_keep > 0 && a.block_err != nullptr) {
    const float* err = a.block_err + size_t(row) * a.nb_stride;
    const int ncomplete = min(L / a.S, nb);
    int kept0 = -1;
    for (int r = 0; r < a.n_keep; ++r) {
      float bv = -INFINITY;
      int bi = -1;
      for (int j = tid; j < ncomplete; j += NT) {
        const float e = err[j];
        if (j != kept0 && (bi < 0 || order_key(e) > order_key(bv))) {
          bv = e;
          bi = j;
        }
      }
      const int best = ops.argmax(bv, bi);
      if (tid == 0) s_forced[2 + r] = best;
      kept0 = best;
      __syncthreads();
    }
  }
  if (tid == 0) {
    s_forced[0] = a.force_sink ? 0 : -1;
    s_forced[1] = a.force_last ? nb - 1 : -1;
    if (!(a.n_keep > 0 && a.block_err != nullptr) || a.n_keep < 1) s_forced[2] = -1;
    if (!(a.n_keep > 0 && a.block_err != nullptr) || a.n_keep < 2) s_forced[3] = -1;
    int n = 0;
    for (int i = 0; i < 4; ++i) {
      const int f = s_forced[i];
      bool dup = f < 0;
      for (int q = 0; q < i && !dup; ++q) dup = (s_forced[q] == f);
      if (dup) s_forced[i] = -1; else ++n;
    }
    s_nforced = n;
  }
  uint32_t active = 0u, chosen = 0u;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    if (jw + i * 32 < nb) active |= 1u << i;
    v[i] = sanitize(v[i]);
  }
  __syncthreads();
  // each forced block moves from active to chosen in the thread that owns it
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int f = s_forced[q] - jbase;
    if (f >= 0 && f < CAP && f / SPAN == warp && (f & 31) == lane) {
      const int i = (f % SPAN) >> 5;
      chosen |= 1u << i;
      active &= ~(1u << i);
    }
  }
  int need = k - s_nforced;
  int n_active = nb - s_nforced;                     // known exactly: no reduction needed

  // ---------------- linear-bin pass: everything above the threshold bin is chosen
  if (need > 0 && n_active > need) {
    float lo = FLT_MAX, hi = -FLT_MAX;
#pragma unroll
    for (int i = 0; i < ITEMS; ++i)
      if (active >> i & 1u) { lo = fminf(lo, v[i]); hi = fmaxf(hi, v[i]); }
    ops.minmax(lo, hi);
    if constexpr (CL > 1) {
      if (tid == 0) { s_mm[0] = lo; s_mm[1] = hi; }
      csync();
      for (int r = 0; r < CL; ++r) {
        const float* m = cg::this_cluster().map_shared_rank(s_mm, r);
        lo = fminf(lo, m[0]);
        hi = fmaxf(hi, m[1]);
      }
      csync();
    }
    if (hi > lo) {
      for (int i = tid; i < kLinBins; i += NT) hist[i] = 0;
      __syncthreads();
      // bin = nearest integer to fma(x, scale, -lo * scale), clamped to the last bin: a
      // correctly rounded FMA with a positive scale, rounding to an integer (adding
      // 1.5 * 2^23) and a clamp are each monotone, so a higher bin always holds higher
      // scores. An overflowing range saturates and only coarsens the bins.
      const float scale = float(kLinBins - 1) / (hi - lo);
      const float off = -lo * scale;
      uint32_t bins[(ITEMS + 1) / 2];                // two 16-bit bins per word
#pragma unroll
      for (int i = 0; i < ITEMS; ++i) {
        int bn = __float_as_int(__fadd_rn(__fmaf_rn(v[i], scale, off), 12582912.0f)) - 0x4B400000;
        bn = bn < 0 ? 0 : (bn >= kLinBins ? kLinBins - 1 : bn);
        if (i % 2 == 0) bins[i / 2] = uint32_t(bn); else bins[i / 2] |= uint32_t(bn) << 16;
        if (active >> i & 1u) atomicAdd(&hist[bn], 1);
      }
      __syncthreads();
      const int* H = cluster_hist(kLinBins);
      find_threshold_bin<NT>(H, kLinBins, need, &s_bin, &s_above, ops);
      const uint32_t bstar = uint32_t(s_bin);
      const int above = s_above;
      const int cnt = H[bstar];
#pragma unroll
      for (int i = 0; i < ITEMS; ++i) {
        const uint32_t bn = (bins[i / 2] >> (16 * (i % 2))) & 0xFFFFu;
        if (!(active >> i & 1u)) continue;
        if (bn > bstar) { chosen |= 1u << i; active &= ~(1u << i); }
        else if (bn < bstar) active &= ~(1u << i);
      }
      need -= above;
      n_active = cnt;
      __syncthreads();
    }
  }

  // ---------------- few candidates left (the usual case): rank them all pairwise under the
  // order (higher score, then lower index); each candidate's owner keeps it if its rank is
  // below `need`
  if (need > 0 && n_active > need && n_active <= kRankCap) {
    if (tid == 0) s_cnt = 0;
    __syncthreads();
    // one shared-memory atomic per warp reserves the warp's slots
    const int my = __popc(active);
    int incl = my;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    int base = 0;
    if (lane == 31 && incl > 0) base = atomicAdd(&s_cnt, incl);
    int slot = __shfl_sync(kFull, base, 31) + incl - my;
    // (scores are re-read from the row's buffer: the registers now hold the packed bins;
    // loops over this thread's few candidates, not over all items, keep the code small)
    for (uint32_t bits = active; bits != 0u; bits &= bits - 1u) {
      const int jc = jw + (__ffs(bits) - 1) * 32;
      list_v[slot] = sanitize(sc[jc]);
      list_j[slot] = jc;
      ++slot;
    }
    __syncthreads();
    csync();                                         // every CTA's list is complete
    for (uint32_t bits = active; bits != 0u; bits &= bits - 1u) {
      const int i = __ffs(bits) - 1;
      const int jc = jw + i * 32;
      const float vc = sanitize(sc[jc]);
      int rank = 0;
      for (int r = 0; r < CL; ++r) {
        const float* lv = list_v;
        const int* lj = list_j;
        int n = s_cnt;
        if constexpr (CL > 1) {
          lv = cg::this_cluster().map_shared_rank(list_v, r);
          lj = cg::this_cluster().map_shared_rank(list_j, r);
          n = *cg::this_cluster().map_shared_rank(&s_cnt, r);
        }
        for (int o = 0; o < n; ++o) {
          const float vo = lv[o];
          rank += (vo > vc) || (vo == vc && lj[o] < jc);
        }
      }
      if (rank < need) chosen |= 1u << i;
    }
    csync();                                         // no CTA still reads the lists
    need = 0;
    active = 0u;
  }

  // ---------------- exact radix select on order keys over what is left (many equal or
  // nearly equal scores)
  for (int shift = 24; shift >= 0 && need > 0 && n_active > need; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < ITEMS; ++i)
      if (active >> i & 1u) atomicAdd(&hist[(order_key(sanitize(sc[jw + i * 32])) >> shift) & 255u], 1);
    __syncthreads();
    const int* H = cluster_hist(256);
    find_threshold_bin<NT>(H, 256, need, &s_bin, &s_above, ops);
    const uint32_t dstar = uint32_t(s_bin);
    const int above = s_above;
    const int cnt = H[dstar];
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
      if (!(active >> i & 1u)) continue;
      const uint32_t dg = (order_key(sanitize(sc[jw + i * 32])) >> shift) & 255u;
      if (dg > dstar) { chosen |= 1u << i; active &= ~(1u << i); }
      else if (dg < dstar) active &= ~(1u << i);
    }
    need -= above;
    n_active = cnt;
    __syncthreads();
  }

  // ---------------- remaining slots: the lowest-indexed actives (they share one key)
  if (need > 0) {
    int wcnt = 0;
#pragma unroll 1
    for (int i = 0; i < ITEMS; ++i) wcnt += __popc(__ballot_sync(kFull, active >> i & 1u));
    int tot, ctot;
    int before = warp_exclusive<NW>(wcnt, s_i, &tot);
    before += cluster_prefix(tot, &ctot);
#pragma unroll 1
    for (int i = 0; i < ITEMS; ++i) {
      const uint32_t m = __ballot_sync(kFull, active >> i & 1u);
      if ((active >> i & 1u) && before + __popc(m & ((1u << lane) - 1u)) < need) chosen |= 1u << i;
      before += __popc(m);
    }
  }

  // ---------------- ascending output: warp ranges in order, items in order, lanes in order.
  // Transposing the warp's 32 x 32 bit matrix (lane = row, item = column) gives lane i the
  // mask of lanes that chose item i; a scan of their counts over the lanes places every item.
  uint32_t tr = transpose32(chosen, lane);
  const int cnt_i = __popc(tr);
  int incl = cnt_i;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t* s_tr = s_out + warp * 64;                  // [lane masks of item i, items before i]
  s_tr[lane] = tr;
  s_tr[32 + lane] = uint32_t(incl - cnt_i);
  int tot_cta, tot;
  int pos = warp_exclusive<NW>(__shfl_sync(kFull, incl, 31), s_i, &tot_cta);  // syncs the CTA
  pos += cluster_prefix(tot_cta, &tot);
  for (uint32_t bits = chosen; bits != 0u; bits &= bits - 1u) {
    const int i = __ffs(bits) - 1;
    const int p = pos + int(s_tr[32 + i]) + __popc(s_tr[i] & ((1u << lane) - 1u));
    if (p < k) sel[p] = jw + i * 32;
  }
  if (tot != n_out && tid == 0 && crank == 0)
    flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
  if (crank == 0)
    for (int i = tot + tid; i < k; i += NT) sel[i] = -1;
}

template <int NT, int ITEMS, int CL>
static cudaError_t launch_select_t(const SelectParams& a, cudaStream_t s, bool pdl) {
  if constexpr (CL == 1) {
    return launch_k(select_kernel<NT, ITEMS, 1>, dim3(a.rows), dim3(NT), 0, s, pdl, a);
  } else {
    // a cluster of CL CTAs per row
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL * a.rows);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, select_kernel<NT, ITEMS, CL>, a);
  }
}

// CTA shape of the selection of more than 4,096 blocks per row: 1024 threads x 32 blocks, one
// CTA per row up to 32,768 blocks, a cluster of 4 beyond. Measured alternatives (token
// level, batch 16): 512 x 32 in clusters of 2 / 8 took 23.9 / 121.8 us against 19.2 / 83.8
// us at 32K / 128K, and 256 x 32 in clusters of 4 took 37.0 us at 32K (cluster barriers
// cost more than the extra CTAs per SM gain).
constexpr int kSelNT = 1024, kSelItems = 32, kSelCap = kSelNT * kSelItems;

cudaError_t launch_select(const Plan& p, const SelectParams& a, cudaStream_t s, bool pdl) {
  const int nbs = a.nb_stride;
  if (nbs <= 256 * 4) return launch_select_t<256, 4, 1>(a, s, pdl);
  if (nbs <= 256 * 16) return launch_select_t<256, 16, 1>(a, s, pdl);
  if (nbs <= 32768) return launch_select_t<kSelNT, kSelItems, 32768 / kSelCap>(a, s, pdl);
  if (nbs <= 131072) return launch_select_t<kSelNT, kSelItems, 131072 / kSelCap>(a, s, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace qs
