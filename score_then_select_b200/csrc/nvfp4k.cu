// nvfp4k.cu - the attended keys of the NVFP4 storage variant, gathered for attention.
//
// "Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention" (Full
// text): the persistent cache keeps the keys in NVFP4, and at most two blocks per sequence
// at BF16 (those with the largest quantisation error). Reading: a token in a kept block is
// attended with its stored BF16 key; any other token with its NVFP4 code dequantised and
// un-centred, e * sigma * g_k + mu, each product and sum a rounded float32 operation, then
// rounded to nearest-even BF16 for the attention's BF16 operands.
//
// This kernel writes those keys (and the values) of every row's selected blocks into the
// compact buffer of gather-then-attend (gather.cu), which dense attention then reads. The
// kept blocks are recomputed per CTA from the per-block errors: the n_keep complete blocks
// with the largest error (a NaN error ranking as -FLT_MAX), ties to the lower index, as the
// select kernel takes them.
//
// One CTA per (row, 128 slots = one selected block, since the NVFP4 path has S = 128):
// thread = one 16-byte chunk (8 elements) of a token row.
#include <cfloat>
#include <cuda_bf16.h>

#include "qs_device.cuh"
#include "nvfp4k.h"

namespace qs {

constexpr int kNkThreads = 256;
constexpr int kNkUnroll = 8;

// E2M1 code -> value: magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}, bit 3 the sign.
QS_DEV float nk_e2m1(uint32_t c) {
  const uint32_t m = c & 7u;
  const float mag = m < 4u ? 0.5f * float(m) : float(2u << ((m - 4u) >> 1)) * (1.0f + 0.5f * float(m & 1u));
  return (c & 8u) ? -mag : mag;
}
// UE4M3 code -> value: bias 7, 3 mantissa bits, subnormals m * 2^-9.
QS_DEV float nk_ue4m3(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  if (e == 0u) return float(m) * 0.001953125f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// The better of two (error, block) candidates: larger error, then lower index.
QS_DEV bool nk_better(float v1, int j1, float v2, int j2) {
  return v1 > v2 || (v1 == v2 && j1 < j2);
}

// Block-wide arg-max over the row's complete blocks, skipping `skip`; -1 if none.
QS_DEV int nk_argmax(const float* err, int n_complete, int skip, float* s_v, int* s_j) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float bv = -INFINITY;
  int bj = -1;
  for (int j = threadIdx.x; j < n_complete; j += blockDim.x) {
    const float e = err[j];
    const float v = e != e ? -FLT_MAX : e;              // NaN ranks as -FLT_MAX
    if (j != skip && (bj < 0 || nk_better(v, j, bv, bj))) {
      bv = v;
      bj = j;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v = __shfl_xor_sync(kFull, bv, o);
    const int j = __shfl_xor_sync(kFull, bj, o);
    if (j >= 0 && (bj < 0 || nk_better(v, j, bv, bj))) {
      bv = v;
      bj = j;
    }
  }
  if (lane == 0) {
    s_v[warp] = bv;
    s_j[warp] = bj;
  }
  __syncthreads();
  float rv = s_v[0];
  int rj = s_j[0];
  for (int w = 1; w < int(blockDim.x) / 32; ++w)
    if (s_j[w] >= 0 && (rj < 0 || nk_better(s_v[w], s_j[w], rv, rj))) {
      rv = s_v[w];
      rj = s_j[w];
    }
  __syncthreads();
  return rj;
}

__global__ void __launch_bounds__(kNkThreads) gather_kv_nvfp4k_kernel(const GatherNvParams p) {
  constexpr int D = 128, CH = D / 8, TPP = kNkThreads / CH, U = kNkUnroll;
  __shared__ float s_v[kNkThreads / 32];
  __shared__ int s_j[kNkThreads / 32];
  const GatherParams& a = p.base;
  const int row = blockIdx.x, b = row / a.Hkv, g = row - b * a.Hkv;
  const int n = a.n_sel[row], L = a.seq_lens[b];
  if (n < 0 || n > a.budget || L < 0) {
    if (blockIdx.y == 0 && threadIdx.x == 0) {
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_GATHER, uint32_t(row));
      a.row_lens[row] = 0;
    }
    return;
  }
  const int nb = (L + kPage - 1) / kPage;
  if (blockIdx.y == 0 && threadIdx.x == 0) {
    long long len = 0;
    if (n > 0) {
      const int last = a.sel[size_t(row) * a.budget + n - 1];
      const long long cut = static_cast<long long>(L) - static_cast<long long>(last) * kPage;
      len = static_cast<long long>(n - 1) * kPage + (cut < 0 ? 0 : (cut < kPage ? cut : kPage));
    }
    a.row_lens[row] = int(len);
  }
  const int nslots = n * kPage;
  const int slot0 = blockIdx.y * (TPP * U);
  if (slot0 >= nslots) return;
  // the row's kept blocks
  int k1 = -1, k2 = -1;
  if (p.n_keep > 0 && p.block_err) {
    const float* err = p.block_err + size_t(row) * p.nb_stride;
    const int complete = min(L / kPage, p.nb_stride);
    k1 = nk_argmax(err, complete, -1, s_v, s_j);
    if (p.n_keep > 1 && k1 >= 0) k2 = nk_argmax(err, complete, k1, s_v, s_j);
  }
  const int c = threadIdx.x % CH, tl = threadIdx.x / CH;
  const float gk = *p.key_gscale;
  const float* mu = p.key_center + size_t(row) * D + c * 8;
  int blk[U], pg[U], tok[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int slot = slot0 + u * TPP + tl;
    blk[u] = slot < nslots ? a.sel[size_t(row) * a.budget + slot / kPage] : -2;
  }
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
    const int t = blk[u] * kPage + slot % kPage;
    if (t >= L) continue;
    tok[u] = t;
    const int pi = t / kPage;
    pg[u] = pi < a.max_pages_per_seq ? a.page_table[size_t(b) * a.max_pages_per_seq + pi] : -1;
    if (pg[u] < 0 || pg[u] >= a.num_pages) {
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_GATHER, uint32_t(row));
      pg[u] = -1;
    }
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (pg[u] < 0) continue;
    const int slot = slot0 + u * TPP + tl, s_in = tok[u] % kPage;
    const size_t src = ((size_t(pg[u]) * a.Hkv + g) * kPage + s_in) * D + c * 8;
    uint4 kx;
    if (blk[u] == k1 || blk[u] == k2) {
      kx = *reinterpret_cast<const uint4*>(a.k + src);          // a kept block: BF16
    } else {
      const size_t ph = size_t(pg[u]) * a.Hkv + g;
      const int gr = c >> 1;                                    // the 16-element group
      const uint32_t code = *reinterpret_cast<const uint32_t*>(
          p.codes + ph * kNvfp4PageCodeBytes + nvfp4_code_off(s_in, gr) + (c & 1) * 4);
      const float sig = nk_ue4m3(p.scales[ph * kNvfp4PageScaleBytes + nvfp4_scale_off(s_in, gr)]);
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = __fadd_rn(__fmul_rn(nk_e2m1((code >> (8 * e)) & 15u) * sig, gk), mu[2 * e]);
        const float hi = __fadd_rn(__fmul_rn(nk_e2m1((code >> (8 * e + 4)) & 15u) * sig, gk),
                                   mu[2 * e + 1]);
        w[e] = uint32_t(f32_to_bf16_rn(lo)) | (uint32_t(f32_to_bf16_rn(hi)) << 16);
      }
      kx = make_uint4(w[0], w[1], w[2], w[3]);
    }
    const uint4 vx = *reinterpret_cast<const uint4*>(a.v + src);
    const size_t dst =
        ((size_t(b * a.dst_pages_per_seq + slot / kPage) * a.Hkv + g) * kPage + slot % kPage) * D + c * 8;
    *reinterpret_cast<uint4*>(a.k_dst + dst) = kx;
    *reinterpret_cast<uint4*>(a.v_dst + dst) = vx;
  }
}

// CTA = one row: its n_keep kept blocks (the complete blocks with the largest error, ranked
// as the select kernel ranks them), written for the attention over the NVFP4 keys.
__global__ void __launch_bounds__(128) kept_blocks_kernel(const KeptParams p) {
  __shared__ float s_v[4];
  __shared__ int s_j[4];
  pdl_wait();                  // the errors (and the step before) come from earlier kernels
  pdl_trigger();
  const int row = blockIdx.x, b = row / p.Hkv;
  const int L = max(0, p.seq_lens[b]);
  const float* err = p.block_err + size_t(row) * p.nb_stride;
  const int complete = min(L / kPage, p.nb_stride);
  int k1 = -1, k2 = -1;
  if (p.n_keep > 0) k1 = nk_argmax(err, complete, -1, s_v, s_j);
  if (p.n_keep > 1 && k1 >= 0) k2 = nk_argmax(err, complete, k1, s_v, s_j);
  if (threadIdx.x == 0) {
    p.kept[2 * row] = k1;
    p.kept[2 * row + 1] = k2;
  }
}

cudaError_t launch_kept_blocks(const KeptParams& p, cudaStream_t s, bool pdl) {
  return launch_k(kept_blocks_kernel, dim3(p.rows), dim3(128), 0, s, pdl, p);
}

cudaError_t launch_gather_kv_nvfp4k(const Plan& pl, const GatherNvParams& p, cudaStream_t s) {
  const int per_cta = (kNkThreads / 16) * kNkUnroll;            // 128 slots
  const int slices = (pl.budget * kPage + per_cta - 1) / per_cta;
  gather_kv_nvfp4k_kernel<<<dim3(p.base.rows, slices), kNkThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace qs
