// score_centroid.cu - centroid scoring of contiguous blocks.
//
// "Coarse Semantic Blocks ...", Abstract: each block is scored by its centroid against the
// query. Here the centroid is the mean of the block's stored keys (the cache holds FP32
// sums, append.cu) and the block score is the group-mean query dotted with it:
//   beta_j = qbar . sum_j / count_j,   qbar = mean of the group's query heads (FP32),
// which is the mean of the block's exact group-mean scores. The scan reads d * 4 bytes per
// block instead of r * 2 bytes per token.
//
// CTA = (32 blocks of one sequence), warp w = KV heads w, w + 8, ... (the page's sums of all
// heads are contiguous, so the CTA reads each page as one region); each lane holds 4
// (d = 128) or 2 (d = 64) entries of qbar and of each centroid; a warp resolves 8 pages at
// once, issues the 8 centroid loads, then reduces each block with shuffles. Measured at
// 128K (S 128, 64 MB of sums): 26.8 us for the standalone call; 8 blocks per CTA (35.3 us)
// and all 32 pages resolved at once with double-buffered loads (37.9 us, 117 registers)
// were slower.
// Blocks past ceil(seq_len / S) that share a page with valid tokens are written -inf.
#include "qs_device.cuh"

namespace qs {

constexpr int kCentBlocksPerCta = 32;

template <int D>
__global__ void __launch_bounds__(256) score_centroid_kernel(const ScoreParams a) {
  constexpr int E = D / 32;                       // entries per lane
  pdl_wait();      // the sums and seq_lens come from the kernel before
  pdl_trigger();
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_context) {
    if (threadIdx.x == 0 && blockIdx.x == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(b));
    L = L < 0 ? 0 : a.max_context;
  }
  const int S = a.S, bpp = kPage / S;
  const int nb = (L + S - 1) / S;
  const int nb_pages = (L + kPage - 1) / kPage * bpp;   // blocks of the pages in use
  const int j0 = blockIdx.x * kCentBlocksPerCta;
  if (j0 >= nb_pages) return;
  const int j_end = min(j0 + kCentBlocksPerCta, nb_pages);
  const float* sums = reinterpret_cast<const float*>(a.proxy);
  const int Hq = a.Hkv * a.G;
  // warp w takes KV heads w, w + 8, ...: the CTA's warps read the heads of the same pages
  // together, so each page's sums (all heads, contiguous) are read as one region
  for (int g = warp; g < a.Hkv; g += 8) {
    const int row = b * a.Hkv + g;
    // qbar: the mean of the group's heads, ascending head order, FP32
    float qv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float sq = 0.0f;
      for (int h = 0; h < a.G; ++h)
        sq += bf16_to_f32(a.q[(size_t(b) * Hq + size_t(g) * a.G + h) * D + lane * E + e]);
      qv[e] = sq / float(a.G);
    }
    float* out = a.scores + size_t(row) * a.nb_stride;
    // 8 consecutive blocks at a time: lane u < 8 resolves block jw + u's page, then all 8
    // centroid loads are issued before any is reduced
    for (int jw = j0; jw < j_end; jw += 8) {
      int page = -1;
      if (lane < 8 && jw + lane < nb) {
        const int pi = ((jw + lane) * S) >> 7;
        page = pi < a.max_pages_per_seq ? a.page_table[size_t(b) * a.max_pages_per_seq + pi] : -1;
        if (page < 0 || page >= a.num_pages) {
          flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SCORE, uint32_t(row));
          page = -1;
        }
      }
      float v[8][E];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int pg = __shfl_sync(kFull, page, u);
        const int j = jw + u;
#pragma unroll
        for (int e = 0; e < E; ++e) v[u][e] = 0.0f;
        if (pg >= 0) {
          const float* c = sums + ((size_t(pg) * a.Hkv + g) * bpp + (j % bpp)) * D + lane * E;
          if constexpr (E == 4) {
            const float4 x = *reinterpret_cast<const float4*>(c);
            v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
          } else {
            const float2 x = *reinterpret_cast<const float2*>(c);
            v[u][0] = x.x; v[u][1] = x.y;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float dot = 0.0f;
#pragma unroll
        for (int e = E - 1; e >= 0; --e) dot = fmaf(qv[e], v[u][e], dot);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(kFull, dot, o);
        const int j = jw + u;
        const int pg = __shfl_sync(kFull, page, u);
        if (lane == 0 && j < j_end)
          out[j] = (j < nb && pg >= 0) ? __fdiv_rn(dot, float(min(S, L - j * S))) : -INFINITY;
      }
    }
  }
}

cudaError_t launch_score_centroid(const Plan& p, const ScoreParams& a, cudaStream_t s, bool pdl) {
  const dim3 grid((a.nb_stride + kCentBlocksPerCta - 1) / kCentBlocksPerCta, a.batch);
  if (p.d == 128) return launch_k(score_centroid_kernel<128>, grid, dim3(256), 0, s, pdl, a);
  if (p.d == 64) return launch_k(score_centroid_kernel<64>, grid, dim3(256), 0, s, pdl, a);
  return cudaErrorInvalidValue;
}

}  // namespace qs
