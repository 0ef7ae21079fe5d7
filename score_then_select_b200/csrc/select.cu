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
// Algorithm, one CTA per row; thread t owns blocks t, t + NT, t + 2 NT, ... in registers
// (coalesced loads); shared-memory bitmaps restore index order at the end:
//   1. forced blocks are marked (the kept blocks are the n_keep complete blocks with the
//      largest block error, found by two block-wide arg-max reductions);
//   2. one pass of a 2048-bin histogram that is linear in the score between the active
//      minimum and maximum (a monotone map, so every block in a higher bin scores higher)
//      selects every bin above the threshold bin and leaves only the threshold bin active;
//   3. the few blocks left in the threshold bin are ranked pairwise (score descending,
//      index ascending) and the first ones taken; only if many are left (many equal or
//      nearly equal scores) does an exact MSB-first radix select (4 x 8-bit digits) over
//      order-preserving uint32 keys narrow them to one key value;
//   4. the remaining slots go to the lowest-indexed blocks holding that key (a scan over
//      the bitmap of remaining candidates);
//   5. a scan over the bitmap of chosen blocks writes the ascending indices.
// The count left in the threshold bin is read from the histogram, so no extra block-wide
// reduction is needed between passes.
#include <cfloat>

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
  float* s_f;    // [2 * NW]

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
    lo = s_f[0];
    hi = s_f[NW];
    for (int i = 1; i < NW; ++i) { lo = fminf(lo, s_f[i]); hi = fmaxf(hi, s_f[NW + i]); }
    __syncthreads();
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

template <int NT, int ITEMS>
__global__ void __launch_bounds__(NT) select_kernel(const SelectParams a) {
  constexpr int NW = NT / 32;
  constexpr int CAP = NT * ITEMS;                 // blocks one CTA can hold
  constexpr int NWORDS = CAP / 32;                // bitmap words
  constexpr int WPT = (NWORDS + NT - 1) / NT;     // bitmap words per thread (contiguous)
  __shared__ int s_i[NW + 1];
  __shared__ float s_f[2 * NW];
  __shared__ int hist[kLinBins];
  __shared__ uint32_t chosen_bits[NWORDS], active_bits[NWORDS];
  __shared__ float list_v[kRankCap];
  __shared__ int list_j[kRankCap];
  __shared__ int s_bin, s_above, s_cnt, s_forced[4], s_nforced;
  BlockOps<NT> ops{s_i, s_f};

  pdl_wait();      // the scores come from the kernel before
  pdl_trigger();
  const int row = blockIdx.x;
  const int b = row / a.Hkv;
  const int tid = threadIdx.x;
  int L = a.seq_lens[b];
  const int nb_cap = a.nb_stride < CAP ? a.nb_stride : CAP;
  int nb = (L + a.S - 1) / a.S;
  if (L < 0 || nb > nb_cap) {
    if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
    nb = L < 0 ? 0 : nb_cap;
    if (L < 0) L = 0;
  }
  int32_t* sel = a.sel + size_t(row) * a.budget;
  const int k = a.budget;
  const int n_out = nb < k ? nb : k;
  if (tid == 0) a.n_sel[row] = n_out;

  if (nb <= k) {  // the budget covers every block
    for (int i = tid; i < k; i += NT) sel[i] = i < nb ? i : -1;
    return;
  }

  // item i of this thread is block j = i * NT + tid (coalesced loads)
  const float* sc = a.scores + size_t(row) * a.nb_stride;
  float v[ITEMS];
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const int j = i * NT + tid;
    v[i] = j < nb ? sc[j] : -FLT_MAX;
  }
  for (int w = tid; w < NWORDS; w += NT) chosen_bits[w] = active_bits[w] = 0u;

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
  __syncthreads();
  int need = k - s_nforced;
  uint32_t active = 0u, chosen = 0u;
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const int j = i * NT + tid;
    if (j < nb) {
      bool f = false;
#pragma unroll
      for (int q = 0; q < 4; ++q) f |= (s_forced[q] == j);
      if (f) chosen |= 1u << i; else active |= 1u << i;
      float x = v[i];
      if (x != x) x = -FLT_MAX;                      // NaN ranks lowest
      v[i] = fminf(fmaxf(x, -FLT_MAX), FLT_MAX);
    }
  }
  int n_active = nb - s_nforced;                     // known exactly: no reduction needed

  // ---------------- linear-bin pass: everything above the threshold bin is chosen
  if (need > 0 && n_active > need) {
    float lo = FLT_MAX, hi = -FLT_MAX;
#pragma unroll
    for (int i = 0; i < ITEMS; ++i)
      if (active >> i & 1u) { lo = fminf(lo, v[i]); hi = fmaxf(hi, v[i]); }
    ops.minmax(lo, hi);
    if (hi > lo) {
      for (int i = tid; i < kLinBins; i += NT) hist[i] = 0;
      __syncthreads();
      // bin = trunc((x - lo) * scale): a rounded subtraction, a rounded product by a
      // positive constant and a truncation are each monotone, so a higher bin always holds
      // higher scores (recomputed below rather than kept, to stay within the 64 registers
      // of a 1024-thread CTA); an overflowing range saturates and only coarsens the bins
      const float scale = float(kLinBins) / (hi - lo);
      auto bin_of = [&](float x) {
        const int bn = __float2int_rz((x - lo) * scale);
        return bn < 0 ? 0 : (bn >= kLinBins ? kLinBins - 1 : bn);
      };
#pragma unroll
      for (int i = 0; i < ITEMS; ++i)
        if (active >> i & 1u) atomicAdd(&hist[bin_of(v[i])], 1);
      __syncthreads();
      find_threshold_bin<NT>(hist, kLinBins, need, &s_bin, &s_above, ops);
      const int bstar = s_bin;
      const int above = s_above;
      const int cnt = hist[bstar];
#pragma unroll
      for (int i = 0; i < ITEMS; ++i) {
        if (!(active >> i & 1u)) continue;
        const int bn = bin_of(v[i]);
        if (bn > bstar) { chosen |= 1u << i; active &= ~(1u << i); }
        else if (bn < bstar) active &= ~(1u << i);
      }
      need -= above;
      n_active = cnt;
      __syncthreads();
    }
  }

  // ---------------- few candidates left (the usual case): rank them all pairwise under the
  // order (higher score, then lower index) and keep the first `need`
  if (need > 0 && n_active > need && n_active <= kRankCap) {
    if (tid == 0) s_cnt = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
      if (active >> i & 1u) {
        const int slot = atomicAdd(&s_cnt, 1);
        list_v[slot] = v[i];
        list_j[slot] = i * NT + tid;
      }
    }
    __syncthreads();
    const int n = s_cnt;
    for (int c = tid; c < n; c += NT) {
      const float vc = list_v[c];
      const int jc = list_j[c];
      int rank = 0;
      for (int o = 0; o < n; ++o) {
        const float vo = list_v[o];
        rank += (vo > vc) || (vo == vc && list_j[o] < jc);
      }
      if (rank < need) atomicOr(&chosen_bits[jc >> 5], 1u << (jc & 31));
    }
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
      if (active >> i & 1u) atomicAdd(&hist[(order_key(v[i]) >> shift) & 255u], 1);
    __syncthreads();
    find_threshold_bin<NT>(hist, 256, need, &s_bin, &s_above, ops);
    const uint32_t dstar = uint32_t(s_bin);
    const int above = s_above;
    const int cnt = hist[dstar];
#pragma unroll
    for (int i = 0; i < ITEMS; ++i) {
      if (!(active >> i & 1u)) continue;
      const uint32_t dg = (order_key(v[i]) >> shift) & 255u;
      if (dg > dstar) { chosen |= 1u << i; active &= ~(1u << i); }
      else if (dg < dstar) active &= ~(1u << i);
    }
    need -= above;
    n_active = cnt;
    __syncthreads();
  }

  // ---------------- index order: chosen blocks, plus the `need` lowest-indexed actives
#pragma unroll
  for (int i = 0; i < ITEMS; ++i) {
    const int j = i * NT + tid;
    if (chosen >> i & 1u) atomicOr(&chosen_bits[j >> 5], 1u << (j & 31));
    if (need > 0 && (active >> i & 1u)) atomicOr(&active_bits[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  const int w0 = tid * WPT;
  if (need > 0) {
    // remaining actives share one key (or exactly fill the need): lowest indices first
    int cnt = 0;
#pragma unroll
    for (int w = 0; w < WPT; ++w)
      if (w0 + w < NWORDS) cnt += __popc(active_bits[w0 + w]);
    int tot;
    int before = ops.exclusive_sum(cnt, &tot);
#pragma unroll
    for (int w = 0; w < WPT; ++w) {
      if (w0 + w >= NWORDS) break;
      uint32_t bits = active_bits[w0 + w];
      while (bits != 0u && before < need) {
        const uint32_t low = bits & (~bits + 1u);
        chosen_bits[w0 + w] |= low;
        bits ^= low;
        ++before;
      }
    }
    __syncthreads();
  }
  int cnt = 0;
#pragma unroll
  for (int w = 0; w < WPT; ++w)
    if (w0 + w < NWORDS) cnt += __popc(chosen_bits[w0 + w]);
  int tot;
  int pos = ops.exclusive_sum(cnt, &tot);
#pragma unroll
  for (int w = 0; w < WPT; ++w) {
    if (w0 + w >= NWORDS) break;
    uint32_t bits = chosen_bits[w0 + w];
    while (bits != 0u) {
      const int bit = __ffs(bits) - 1;
      if (pos < k) sel[pos] = (w0 + w) * 32 + bit;
      ++pos;
      bits &= bits - 1u;
    }
  }
  if (tot != n_out && tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
  for (int i = tot + tid; i < k; i += NT) sel[i] = -1;
}

cudaError_t launch_select(const Plan& p, const SelectParams& a, cudaStream_t s, bool pdl) {
  const int nbs = a.nb_stride;
  if (nbs <= 256 * 4) return launch_k(select_kernel<256, 4>, dim3(a.rows), dim3(256), 0, s, pdl, a);
  if (nbs <= 256 * 16) return launch_k(select_kernel<256, 16>, dim3(a.rows), dim3(256), 0, s, pdl, a);
  if (nbs <= 1024 * 32) return launch_k(select_kernel<1024, 32>, dim3(a.rows), dim3(1024), 0, s, pdl, a);
  return cudaErrorInvalidValue;
}

}  // namespace qs
