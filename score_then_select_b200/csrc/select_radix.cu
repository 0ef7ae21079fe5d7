// select_radix.cu - top-k block selection by histogram (radix) passes, one CTA per row.
//
// The same result as select.cu ("Joint Subspace Sparse Attention for Efficient
// Long-Context Decoding", Figure 1 and Table 15: each KV head's top blocks; "Jet-QSparse",
// Full text: kept blocks always attended): if nb <= k every block; otherwise the forced
// set F (sink, last, the n_keep complete blocks with the largest error) plus the k - |F|
// best other blocks, equal scores to the lower index, ascending. Scores are ranked after
// NaN and -inf become -FLT_MAX, +inf becomes FLT_MAX and -0 becomes +0.
//
// Instead of ranking candidates pairwise, the cut is found on the order-preserving 32-bit
// key of each score by three counting passes (its top 11, next 11 and last 10 bits): each
// pass histograms the keys that share the bits found so far and finds the bin where the
// count from the top reaches the remaining need. Blocks above the final key are taken, and
// the blocks holding it in index order, as many as are still needed. Every pass reads the
// row's scores from global memory (L2-resident after the scan), so the cost is a few
// streaming passes and no pairwise work.
#include <cfloat>

#include "qs_device.cuh"

namespace qs {

constexpr int kRxThreads = 1024;
constexpr int kRxBins = 2048;

QS_DEV uint32_t rx_key(float x) {
  x = fminf(fmaxf(x, -FLT_MAX), FLT_MAX);           // NaN, -inf -> -FLT_MAX; +inf -> FLT_MAX
  if (x == 0.0f) x = 0.0f;                           // -0 ranks with +0
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix of v over the CTA's threads in order; total receives the sum.
QS_DEV int rx_scan(int v, int* s, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = s[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += y;
    }
    s[lane] = t;
  }
  __syncthreads();
  const int before = warp ? s[warp - 1] : 0;
  total = s[kRxThreads / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// The bin (walked from the highest) where the count from the top reaches `need`, and the
// count above it; every thread returns the same values. The histogram always reaches it.
QS_DEV int rx_find(const int* hist, int nbins, int need, int* s_scan, int* s_found,
                   int& above) {
  const int per = nbins / kRxThreads;
  const int hi = nbins - 1 - int(threadIdx.x) * per;
  int loc = 0;
  for (int i = 0; i < per; ++i) loc += hist[hi - i];
  if (threadIdx.x == 0) {
    s_found[0] = -1;
    s_found[1] = 0;
  }
  int tot;
  int c = rx_scan(loc, s_scan, tot);
  for (int i = 0; i < per; ++i) {
    const int prev = c;
    c += hist[hi - i];
    if (prev < need && c >= need) {
      s_found[0] = hi - i;
      s_found[1] = prev;
    }
  }
  __syncthreads();
  const int bin = s_found[0];
  above = s_found[1];
  __syncthreads();
  return bin;
}

// Block-wide arg-max of the error over the complete blocks j < n, skipping `skip`: the
// larger key, then the lower index; -1 if none.
QS_DEV int rx_argmax(const float* err, int n, int skip, uint32_t* s_k, int* s_j) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t bk = 0u;
  int bj = -1;
  for (int j = threadIdx.x; j < n; j += kRxThreads) {
    const uint32_t k = rx_key(err[j]);
    if (j != skip && (bj < 0 || k > bk)) {
      bk = k;
      bj = j;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t k = __shfl_xor_sync(kFull, bk, o);
    const int j = __shfl_xor_sync(kFull, bj, o);
    if (j >= 0 && (bj < 0 || k > bk || (k == bk && j < bj))) {
      bk = k;
      bj = j;
    }
  }
  if (lane == 0) {
    s_k[warp] = bk;
    s_j[warp] = bj;
  }
  __syncthreads();
  uint32_t rk = s_k[0];
  int rj = s_j[0];
  for (int w = 1; w < kRxThreads / 32; ++w)
    if (s_j[w] >= 0 && (rj < 0 || s_k[w] > rk || (s_k[w] == rk && s_j[w] < rj))) {
      rk = s_k[w];
      rj = s_j[w];
    }
  __syncthreads();
  return rj;
}

__global__ void __launch_bounds__(kRxThreads, 1) select_radix_kernel(const SelectParams a) {
  __shared__ int hist[kRxBins];
  __shared__ int s_scan[kRxThreads / 32];
  __shared__ int s_found[2];
  __shared__ uint32_t s_k[kRxThreads / 32];
  __shared__ int s_j[kRxThreads / 32];
  const int row = blockIdx.x, b = row / a.Hkv, tid = threadIdx.x;
  const float* sc = a.scores + size_t(row) * a.nb_stride;
  int32_t* sel = a.sel + size_t(row) * a.budget;
  const int k = a.budget;
  int L = a.seq_lens[b];
  int nb = int((static_cast<long long>(L) + a.S - 1) / a.S);
  if (L < 0 || nb > a.nb_stride) {
    if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
    nb = L < 0 ? 0 : a.nb_stride;
    if (L < 0) L = 0;
  }
  if (tid == 0) a.n_sel[row] = nb < k ? nb : k;
  if (nb <= k) {
    for (int i = tid; i < k; i += kRxThreads) sel[i] = i < nb ? i : -1;
    return;
  }
  // forced blocks: sink, last, kept
  int f[4] = {a.force_sink ? 0 : -1, a.force_last ? nb - 1 : -1, -1, -1};
  if (a.n_keep > 0 && a.block_err != nullptr) {
    const float* err = a.block_err + size_t(row) * a.nb_stride;
    const int complete = min(L / a.S, nb);
    f[2] = rx_argmax(err, complete, -1, s_k, s_j);
    if (a.n_keep > 1) f[3] = rx_argmax(err, complete, f[2], s_k, s_j);
  }
  int nf = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bool dup = f[i] < 0;
#pragma unroll
    for (int q = 0; q < i; ++q) dup = dup || f[q] == f[i];
    if (dup) f[i] = -1;
    else ++nf;
  }
  const int f0 = f[0], f1 = f[1], f2 = f[2], f3 = f[3];
#define RX_FORCED(j) ((j) == f0 || (j) == f1 || (j) == f2 || (j) == f3)
  int need = k - nf;
  const bool rest = need > 0;                       // else the forced blocks fill the budget
  // three counting passes over the non-forced keys
  uint32_t prefix = 0u;
  int known = 32;                                   // bits of the key not yet fixed
  for (int pass = 0; pass < 3 && need > 0; ++pass) {
    const int width = pass < 2 ? 11 : 10, nbins = 1 << width;
    const int shift = known - width;
    for (int i = tid; i < kRxBins; i += kRxThreads) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < nb; j += kRxThreads) {
      if (RX_FORCED(j)) continue;
      const uint32_t key = rx_key(sc[j]);
      if (known < 32 && (key >> known) != prefix) continue;
      atomicAdd(&hist[(key >> shift) & uint32_t(nbins - 1)], 1);
    }
    __syncthreads();
    int above;
    const int bin = rx_find(hist, nbins < kRxThreads ? kRxThreads : nbins, need, s_scan, s_found,
                            above);
    prefix = (prefix << width) | uint32_t(bin);
    known = shift;
    need -= above;
  }
  const uint32_t kstar = prefix;                    // all 32 bits fixed
  // output: forced, keys above kstar, and the first `need` blocks holding kstar
  const int C = (nb + kRxThreads - 1) / kRxThreads;
  const int j0 = min(nb, tid * C), j1 = min(nb, j0 + C);
  int my_ties = 0;
  for (int j = j0; j < j1; ++j) my_ties += (rest && !RX_FORCED(j) && rx_key(sc[j]) == kstar);
  int tot;
  const int tie0 = rx_scan(my_ties, s_scan, tot);
  int my_n = 0, tr = tie0;
  for (int j = j0; j < j1; ++j) {
    if (RX_FORCED(j)) { ++my_n; continue; }
    if (!rest) continue;
    const uint32_t key = rx_key(sc[j]);
    if (key > kstar || (key == kstar && tr++ < need)) ++my_n;
  }
  int pos = rx_scan(my_n, s_scan, tot);
  tr = tie0;
  for (int j = j0; j < j1; ++j) {
    bool take = RX_FORCED(j);
    if (!take && rest) {
      const uint32_t key = rx_key(sc[j]);
      take = key > kstar || (key == kstar && tr++ < need);
    }
    if (!take) continue;
    if (pos < k) sel[pos] = j;
    else flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SELECT, uint32_t(row));
    ++pos;
  }
#undef RX_FORCED
}

cudaError_t launch_select_radix(const SelectParams& a, cudaStream_t s) {
  select_radix_kernel<<<a.rows, kRxThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace qs
