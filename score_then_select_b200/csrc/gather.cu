// gather.cu - the first half of gather-then-attend: copy every row's selected blocks out of
// the paged cache into a compact buffer that dense attention then reads.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 2 (b) and
// Figure 6 (a): the pages measure this two-step variant (materialise the selected keys and
// values contiguously, then run ordinary attention over them) against attention that reads
// the selected positions in place. It is built here as that comparison, not as the path.
//
// Compact layout: gathered slot i * S + u of row (b, g) holds token sel[i] * S + u of the
// row, at page b * dst_pages_per_seq + slot / 128, row slot % 128 of a cache-shaped buffer
// [batch * dst_pages_per_seq][Hkv][128][d]. Only the row's last block can be cut by the
// sequence length, and it is the last selected block when selected, so the valid tokens
// form a prefix of row_lens[row] slots; the slots after it are left unwritten.
//
// One CTA per (row, 16 x kUnroll slots at d = 128): thread = one 16-byte chunk of a token
// row of K and of V; each thread first resolves kUnroll slots (selection entry, then page
// table), then issues all of its loads, then all of its stores.
#include "qs_device.cuh"

namespace qs {

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 8;

template <int D>
__global__ void __launch_bounds__(kGatherThreads) gather_kv_kernel(const GatherParams a) {
  constexpr int CH = D / 8;                       // 16-byte chunks of a token row
  constexpr int TPP = kGatherThreads / CH;        // token rows per pass of the CTA
  constexpr int U = kGatherUnroll;
  const int row = blockIdx.x, b = row / a.Hkv, g = row - b * a.Hkv;
  const int n = a.n_sel[row], L = a.seq_lens[b];
  const int S = 1 << a.log2_S;
  if (n < 0 || n > a.budget || L < 0) {
    if (blockIdx.y == 0 && threadIdx.x == 0) {
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_GATHER, uint32_t(row));
      a.row_lens[row] = 0;
    }
    return;
  }
  const long long nb = (static_cast<long long>(L) + S - 1) >> a.log2_S;
  if (blockIdx.y == 0 && threadIdx.x == 0) {
    // valid gathered tokens: full blocks, except a selected last block cut by L
    long long len = 0;
    if (n > 0) {
      const int last = a.sel[size_t(row) * a.budget + n - 1];
      const long long cut = static_cast<long long>(L) - static_cast<long long>(last) * S;
      len = static_cast<long long>(n - 1) * S + (cut < 0 ? 0 : (cut < S ? cut : S));
    }
    a.row_lens[row] = int(len);
  }
  const int nslots = n << a.log2_S;
  const int slot0 = blockIdx.y * (TPP * U);
  if (slot0 >= nslots) return;
  const int c = threadIdx.x % CH, tl = threadIdx.x / CH;

  int blk[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int slot = slot0 + u * TPP + tl;
    blk[u] = slot < nslots ? a.sel[size_t(row) * a.budget + (slot >> a.log2_S)] : -2;
  }
  int pg[U], tok[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int slot = slot0 + u * TPP + tl;
    pg[u] = -1;
    tok[u] = 0;
    if (blk[u] == -2) continue;
    if (blk[u] < 0 || blk[u] >= nb) {
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_GATHER, uint32_t(row));
      continue;
    }
    const long long t = (static_cast<long long>(blk[u]) << a.log2_S) + (slot & (S - 1));
    if (t >= L) continue;                         // the cut part of the last block
    tok[u] = int(t);
    const int pi = tok[u] >> 7;                   // kPage = 128
    pg[u] = pi < a.max_pages_per_seq ? a.page_table[size_t(b) * a.max_pages_per_seq + pi] : -1;
    if (pg[u] < 0 || pg[u] >= a.num_pages) {      // a valid token needs a mapped page
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_GATHER, uint32_t(row));
      pg[u] = -1;
    }
  }
  uint4 kx[U], vx[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (pg[u] < 0) continue;
    const size_t src = ((size_t(pg[u]) * a.Hkv + g) * kPage + (tok[u] & (kPage - 1))) * D + c * 8;
    kx[u] = __ldcs(reinterpret_cast<const uint4*>(a.k + src));
    vx[u] = __ldcs(reinterpret_cast<const uint4*>(a.v + src));
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (pg[u] < 0) continue;
    const int slot = slot0 + u * TPP + tl;
    const size_t dst =
        ((size_t(b * a.dst_pages_per_seq + (slot >> 7)) * a.Hkv + g) * kPage + (slot & (kPage - 1))) * D +
        c * 8;
    *reinterpret_cast<uint4*>(a.k_dst + dst) = kx[u];
    *reinterpret_cast<uint4*>(a.v_dst + dst) = vx[u];
  }
}

cudaError_t launch_gather_kv(const Plan& p, const GatherParams& a, cudaStream_t s) {
  const int per_cta = (kGatherThreads / (p.d / 8)) * kGatherUnroll;
  const int slices = (p.budget * p.S + per_cta - 1) / per_cta;
  const dim3 grid(a.rows, slices);
  if (p.d == 128) return launch_k(gather_kv_kernel<128>, grid, dim3(kGatherThreads), 0, s, false, a);
  if (p.d == 64) return launch_k(gather_kv_kernel<64>, grid, dim3(kGatherThreads), 0, s, false, a);
  return cudaErrorInvalidValue;
}

}  // namespace qs
