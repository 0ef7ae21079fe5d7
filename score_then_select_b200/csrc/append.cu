// append.cu - cache writers fused with the KV append, and the scoring-prep kernels.
//
// Rank-r writer ("Joint Subspace Sparse Attention for Efficient Long-Context Decoding",
// Figure 1): the projected-key cache entry of a new token is k . P[g], evaluated in float32
// in ascending index order with one rounding per product and per sum (no fused
// multiply-add), then stored as float32, or rounded to nearest-even BF16 or FP8 E4M3
// (saturating at +-448; Figure 10 keeps the scoring cache at FP8 or BF16).
//
// Centroid writer ("Coarse Semantic Blocks ...", Abstract): each block's FP32 key sum,
// continued in token order.
//
// Binary-code writer ("RaBitQCache", Abstract): the sign bits of the rotated centred key
// and its factor |o|^2 / |y|_1 (the RaBitQ code).
//
// NVFP4 writer ("Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse
// Attention", Full text): the persistent scoring cache is packed straight from the BF16
// keys after calibrated centring: x = float(k) - mu (float32), then per 16 elements
// a = max|x|, sf = a / (6 g_k), sigma = UE4M3(sf), e_i = E2M1(x_i / (sigma g_k)), every
// step a correctly rounded float32 operation, every conversion nearest-even and
// saturating. Blocks completed by the append get their squared quantisation error, which
// decides the blocks kept at full precision.
#include "qs_device.cuh"
#include "rabitq.h"
#include "semantic.h"

namespace qs {

// ============================================================ NVFP4 element / scale codecs
// E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}: count the rounding thresholds passed; a
// value exactly on a midpoint goes to the neighbour with the even code (strict '>' where
// the lower code is even, '>=' where the upper code is even); beyond 6 saturates to 6.
QS_DEV uint32_t e2m1_encode(float t) {
  const uint32_t sign = (__float_as_uint(t) >> 31) << 3;
  const float a = fabsf(t);
  const uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                     (a >= 3.5f) + (a > 5.0f);
  return sign | c;
}
QS_DEV float e2m1_decode(uint32_t c) {
  const uint32_t m = c & 7u;
  // magnitudes: m < 4 -> m/2 ; m >= 4 -> {2, 3, 4, 6}
  float v = (m < 4u) ? 0.5f * float(m) : (m == 7u ? 6.0f : float(m - 2u));
  return (c & 8u) ? -v : v;
}
QS_DEV float ue4m3_decode(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  if (e == 0u) return float(m) * 0.001953125f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Pack one group of 16 float32 values; returns the scale code and writes 8 code bytes.
QS_DEV uint32_t nvfp4_pack16(const float (&x)[16], float g, uint32_t (&packed)[2]) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  const float sf = __fdiv_rn(a, __fmul_rn(6.0f, g));
  const uint32_t sc = ue4m3_encode(sf);
  const float sv = ue4m3_decode(sc);
  packed[0] = packed[1] = 0u;
  if (sv > 0.0f) {
    const float den = __fmul_rn(sv, g);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t c = e2m1_encode(__fdiv_rn(x[i], den));
      packed[i >> 3] |= c << (4 * (i & 7));
    }
  }
  return sc;
}

// ============================================================ shared helpers
// Resolve the cache slot of token t of sequence b; false (and an error flag) if invalid.
QS_DEV bool cache_slot(const int32_t* page_table, int b, int t, int mpps, int num_pages,
                       int max_context, uint32_t* hdr, uint32_t kid, int& page, int& slot) {
  const int pi = t / kPage;
  if (t < 0 || t >= max_context || pi >= mpps) {
    flag_error(hdr, QS_ERR_DEVICE_BOUNDS, kid, uint32_t(b));
    return false;
  }
  page = page_table[size_t(b) * mpps + pi];
  if (page < 0 || page >= num_pages) {
    flag_error(hdr, QS_ERR_DEVICE_BOUNDS, kid, uint32_t(b));
    return false;
  }
  slot = t % kPage;
  return true;
}

// Scoring prep of one row: qbar = (sum of the group's query heads) / G, q~ = qbar . P[g].
// Uses smem scratch of d floats; P read from global (it is small and L2-resident).
QS_DEV void row_prep(const uint16_t* q, const float* Pg, float* qt_row, float* qbar_s, int b,
                     int g, int Hkv, int G, int d, int r) {
  const int Hq = Hkv * G;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float s = 0.0f;
    for (int h = 0; h < G; ++h) s += bf16_to_f32(q[(size_t(b) * Hq + g * G + h) * d + i]);
    qbar_s[i] = s / float(G);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < r; j += blockDim.x) {
    float acc = 0.0f;
    for (int i = 0; i < d; ++i) acc = fmaf(qbar_s[i], Pg[i * r + j], acc);
    qt_row[j] = acc;
  }
}

// Advance seq_lens once every CTA of the append grid has read them ("last CTA" pattern).
QS_DEV void finish_append(const AppendParams& a) {
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned total = gridDim.x * gridDim.y;
    const unsigned prev = atomicAdd(a.hdr + kCtrAppend, 1u);
    s_last = (prev == total - 1u);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int b = threadIdx.x; b < a.batch; b += blockDim.x) {
    int n = a.n_new ? a.n_new[b] : 1;
    if (n < 0 || n > a.max_new) n = 0;
    a.seq_lens[b] += n;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    a.hdr[kCtrAppend] = 0u;
    __threadfence();
  }
}

// ============================================================ rank-r writer
// CTA = one row (b, g) x TT tokens. Thread (tg, og) computes a 4-token x 4-output
// micro-tile, so each k_i / P_ij loaded from shared memory feeds 4 products.
template <typename PT, int R, int D>
__global__ void __launch_bounds__(64 * R / 16)
append_rankr_kernel(const AppendParams a) {
  constexpr int TT = 64;
  constexpr int NT = TT * R / 16;
  constexpr int OG = R / 4;          // output groups of 4
  extern __shared__ __align__(16) float smem[];
  float* Ps = smem;                  // [D][R]
  float* kT = smem + D * R;          // [D][TT] keys as float, token-minor
  __shared__ int s_page[TT], s_slot[TT];

  const int row = blockIdx.y;
  const int b = row / a.Hkv, g = row % a.Hkv;
  int n_b = a.n_new ? a.n_new[b] : 1;
  if (n_b < 0 || n_b > a.max_new) {
    if (threadIdx.x == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_APPEND, uint32_t(b));
    n_b = 0;
  }
  const int old = a.seq_lens[b];
  const int t0 = blockIdx.x * TT;
  const int cnt = min(TT, n_b - t0);
  const bool prep = (a.q != nullptr) && blockIdx.x == 0;

  if (cnt > 0 || prep) {
    const float* Pg = a.P + size_t(g) * D * R;
    for (int i = threadIdx.x; i < D * R / 4; i += NT)
      reinterpret_cast<float4*>(Ps)[i] = reinterpret_cast<const float4*>(Pg)[i];
  }
  if (cnt > 0) {
    if (threadIdx.x < TT) {
      int page = -1, slot = 0;
      if (int(threadIdx.x) < cnt)
        cache_slot(a.page_table, b, old + t0 + threadIdx.x, a.max_pages_per_seq, a.num_pages,
                   a.max_context, a.hdr, KID_APPEND, page, slot);
      s_page[threadIdx.x] = page;
      s_slot[threadIdx.x] = slot;
    }
    // keys -> smem (transposed, float) and K/V rows -> cache, 16 bytes per thread-step
    constexpr int CH = D / 8;  // 16-byte chunks per row
    for (int it = threadIdx.x; it < TT * CH; it += NT) {
      const int n = it / CH, c = it % CH;
      if (n < cnt) {
        const size_t src = ((size_t(b) * a.Hkv + g) * a.max_new + t0 + n) * D + c * 8;
        const uint4 kv = *reinterpret_cast<const uint4*>(a.k_new + src);
        const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kT[(c * 8 + 2 * e) * TT + n] = bf16_lo(w[e]);
          kT[(c * 8 + 2 * e + 1) * TT + n] = bf16_hi(w[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) kT[(c * 8 + e) * TT + n] = 0.0f;
      }
    }
    __syncthreads();
    for (int it = threadIdx.x; it < cnt * CH; it += NT) {
      const int n = it / CH, c = it % CH;
      const int page = s_page[n];
      if (page < 0) continue;
      const size_t src = ((size_t(b) * a.Hkv + g) * a.max_new + t0 + n) * D + c * 8;
      const size_t dst = ((size_t(page) * a.Hkv + g) * kPage + s_slot[n]) * D + c * 8;
      *reinterpret_cast<uint4*>(a.k + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
      *reinterpret_cast<uint4*>(a.v + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
    }
    // projected keys: ascending i, separate float32 roundings for product and sum
    const int tg = threadIdx.x / OG, og = threadIdx.x % OG;
    float acc[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[x][y] = 0.0f;
#pragma unroll 4
    for (int i = 0; i < D; ++i) {
      const float4 kk = *reinterpret_cast<const float4*>(kT + i * TT + tg * 4);
      const float4 pp = *reinterpret_cast<const float4*>(Ps + i * R + og * 4);
      const float kx[4] = {kk.x, kk.y, kk.z, kk.w};
      const float px[4] = {pp.x, pp.y, pp.z, pp.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = __fadd_rn(acc[x][y], __fmul_rn(kx[x], px[y]));
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int n = tg * 4 + x;
      if (n >= cnt) continue;
      const int page = s_page[n];
      if (page < 0) continue;
      const size_t base = ((size_t(page) * a.Hkv + g) * kPage + s_slot[n]) * R + og * 4;
      if constexpr (sizeof(PT) == 4) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.proxy) + base) =
            make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
      } else if constexpr (sizeof(PT) == 1) {
        *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(a.proxy) + base) =
            e4m3_encode(acc[x][0]) | (e4m3_encode(acc[x][1]) << 8) |
            (e4m3_encode(acc[x][2]) << 16) | (e4m3_encode(acc[x][3]) << 24);
      } else {
        const uint32_t lo = uint32_t(f32_to_bf16_rn(acc[x][0])) |
                            (uint32_t(f32_to_bf16_rn(acc[x][1])) << 16);
        const uint32_t hi = uint32_t(f32_to_bf16_rn(acc[x][2])) |
                            (uint32_t(f32_to_bf16_rn(acc[x][3])) << 16);
        *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.proxy) + base) =
            make_uint2(lo, hi);
      }
    }
  }
  if (prep) {
    __syncthreads();
    float* qbar = kT;  // reuse (the keys are no longer needed)
    const int Hq = a.Hkv * a.G;
    for (int i = threadIdx.x; i < D; i += NT) {
      float s = 0.0f;
      for (int h = 0; h < a.G; ++h) s += bf16_to_f32(a.q[(size_t(b) * Hq + g * a.G + h) * D + i]);
      qbar[i] = s / float(a.G);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < R; j += NT) {
      float acc = 0.0f;
      for (int i = 0; i < D; ++i) acc = fmaf(qbar[i], Ps[i * R + j], acc);
      a.qt[size_t(row) * R + j] = acc;
    }
  }
  finish_append(a);
}

// ============================================================ rank-r writer, one new token
// The decode step appends one token per row: CTA = one row. Thread j < R computes
// projected entry j with the same ascending, separately rounded float32 evaluation as the
// bulk writer (so both writers produce identical bits); with a query given, threads
// R..2R-1 compute the row's q~ (the fused scoring prep).
template <typename PT, int R, int D>
__global__ void __launch_bounds__(128) append_one_rankr_kernel(const AppendParams a) {
  __shared__ __align__(16) float Ps[D * R];
  __shared__ float kf[D], qbar[D];
  __shared__ int s_page, s_slot;
  pdl_trigger();
  const int row = blockIdx.x;
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int tid = threadIdx.x;
  int n_b = a.n_new ? a.n_new[b] : 1;
  if (n_b < 0 || n_b > 1) {
    if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_APPEND, uint32_t(b));
    n_b = 0;
  }
  // every global load of the prologue is issued before any is consumed
  const float* Pg = a.P + size_t(g) * D * R;
  constexpr int NP4 = D * R / 4 / 128;               // float4 loads of P per thread
  float4 pv[NP4];
#pragma unroll
  for (int j = 0; j < NP4; ++j) pv[j] = reinterpret_cast<const float4*>(Pg)[j * 128 + tid];
  const size_t src = size_t(row) * a.max_new * D;  // token 0 of this row in k_new / v_new
  const bool has_k = n_b == 1 && tid < D;
  const uint16_t kraw = has_k ? a.k_new[src + tid] : uint16_t(0);
  const bool prep = a.q != nullptr && tid < D;
  uint16_t qraw[kMaxGroup];
  {
    const int Hq = a.Hkv * a.G;
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
      qraw[h] = (prep && h < a.G) ? a.q[(size_t(b) * Hq + g * a.G + h) * D + tid] : uint16_t(0);
  }
  if (tid == 0) {
    int page = -1, slot = 0;
    if (n_b == 1)
      cache_slot(a.page_table, b, a.seq_lens[b], a.max_pages_per_seq, a.num_pages,
                 a.max_context, a.hdr, KID_APPEND, page, slot);
    s_page = page;
    s_slot = slot;
  }
#pragma unroll
  for (int j = 0; j < NP4; ++j) reinterpret_cast<float4*>(Ps)[j * 128 + tid] = pv[j];
  if (has_k) kf[tid] = bf16_to_f32(kraw);
  if (prep) {
    float s = 0.0f;
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
      if (h < a.G) s += bf16_to_f32(qraw[h]);
    qbar[tid] = s / float(a.G);
  }
  __syncthreads();
  const int page = s_page;
  if (n_b == 1 && page >= 0) {
    const size_t dst = ((size_t(page) * a.Hkv + g) * kPage + s_slot) * D;
    constexpr int CH = D / 8;
    if (tid < CH)
      reinterpret_cast<uint4*>(a.k + dst)[tid] = reinterpret_cast<const uint4*>(a.k_new + src)[tid];
    else if (tid < 2 * CH)
      reinterpret_cast<uint4*>(a.v + dst)[tid - CH] =
          reinterpret_cast<const uint4*>(a.v_new + src)[tid - CH];
    if (tid < R) {
      float acc = 0.0f;
#pragma unroll 8
      for (int i = 0; i < D; ++i) acc = __fadd_rn(acc, __fmul_rn(kf[i], Ps[i * R + tid]));
      const size_t pdst = ((size_t(page) * a.Hkv + g) * kPage + s_slot) * R + tid;
      if constexpr (sizeof(PT) == 4)
        reinterpret_cast<float*>(a.proxy)[pdst] = acc;
      else if constexpr (sizeof(PT) == 1)
        reinterpret_cast<uint8_t*>(a.proxy)[pdst] = uint8_t(e4m3_encode(acc));
      else
        reinterpret_cast<uint16_t*>(a.proxy)[pdst] = f32_to_bf16_rn(acc);
    }
  }
  if (a.q != nullptr && tid >= 64 && tid < 64 + R) {
    const int j = tid - 64;
    float acc = 0.0f;
#pragma unroll 8
    for (int i = 0; i < D; ++i) acc = fmaf(qbar[i], Ps[i * R + j], acc);
    a.qt[size_t(row) * R + j] = acc;
  }
  finish_append(a);
}

// ============================================================ centroid writer
// "Coarse Semantic Blocks ...", Abstract: blocks are scored by their centroids. The cache
// holds each block's FP32 key sum; the scan divides by the block's valid count.
// CTA = (row, one block touched by this call): thread i < d carries dimension i of the
// block's sum through the call's tokens in order (restarting at the block's first token,
// continuing a sum left by an earlier call otherwise); all threads copy the tokens' K and V
// rows into their page slots.
template <int D>
__global__ void __launch_bounds__(128) append_centroid_kernel(const AppendParams a) {
  pdl_trigger();   // the scan may launch now; it waits for this grid before reading
  const int row = blockIdx.y;
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int tid = threadIdx.x;
  int n_b = a.n_new ? a.n_new[b] : 1;
  if (n_b < 0 || n_b > a.max_new) {
    if (tid == 0 && blockIdx.x == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_APPEND, uint32_t(b));
    n_b = 0;
  }
  const int old = a.seq_lens[b], S = a.S;
  const int j = (old >= 0 ? old / S : 0) + int(blockIdx.x);     // this CTA's block
  const int t_lo = max(old, j * S), t_hi = min(old + n_b, (j + 1) * S);
  if (old >= 0 && t_lo < t_hi) {
    const int pi = (j * S) >> 7;                                  // kPage = 128
    int page = -1;
    if (pi < a.max_pages_per_seq) page = a.page_table[size_t(b) * a.max_pages_per_seq + pi];
    if (page < 0 || page >= a.num_pages || t_hi > a.max_context) {
      if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_APPEND, uint32_t(row));
    } else {
      const size_t src0 = size_t(row) * a.max_new * D;           // token 0 of this row's k_new
      // K and V rows of the block's new tokens -> their page slots (16 bytes per step)
      constexpr int CH = D / 8;
      for (int e = tid; e < (t_hi - t_lo) * CH; e += blockDim.x) {
        const int t = t_lo + e / CH, c = e % CH;
        const size_t src = src0 + size_t(t - old) * D + c * 8;
        const size_t dst = ((size_t(page) * a.Hkv + g) * kPage + (t & (kPage - 1))) * D + c * 8;
        *reinterpret_cast<uint4*>(a.k + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
        *reinterpret_cast<uint4*>(a.v + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
      }
      // the block's key sum, dimension tid, in token order
      float* sum = reinterpret_cast<float*>(a.proxy) +
                   ((size_t(page) * a.Hkv + g) * (kPage / S) + ((j * S) & (kPage - 1)) / S) * D;
      if (tid < D) {
        float acc = t_lo == j * S ? 0.0f : sum[tid];
        for (int t = t_lo; t < t_hi; ++t) {
          const float x = bf16_to_f32(a.k_new[src0 + size_t(t - old) * D + tid]);
          acc = t == j * S ? x : __fadd_rn(acc, x);
        }
        sum[tid] = acc;
      }
    }
  }
  finish_append(a);
}

// ============================================================ NVFP4 writer
// CTA = one row x 64 tokens; thread = (token, 16-element group).
__global__ void __launch_bounds__(128) append_nvfp4_kernel(const AppendParams a) {
  constexpr int TT = 64, D = 128, GR = D / 16;
  __shared__ int s_page[TT], s_slot[TT];
  __shared__ float s_mu[D];
  pdl_trigger();   // the block-error kernel may launch now; it waits for this grid
  const int row = blockIdx.y;
  const int b = row / a.Hkv, g = row % a.Hkv;
  int n_b = a.n_new ? a.n_new[b] : 1;
  if (n_b < 0 || n_b > a.max_new) {
    if (threadIdx.x == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_APPEND, uint32_t(b));
    n_b = 0;
  }
  const int old = a.seq_lens[b];
  const int t0 = blockIdx.x * TT;
  const int cnt = min(TT, n_b - t0);
  if (cnt > 0) {
    const float gk = *a.key_gscale;
    for (int i = threadIdx.x; i < D; i += blockDim.x) s_mu[i] = a.key_center[size_t(row) * D + i];
    if (threadIdx.x < TT) {
      int page = -1, slot = 0;
      if (int(threadIdx.x) < cnt)
        cache_slot(a.page_table, b, old + t0 + threadIdx.x, a.max_pages_per_seq, a.num_pages,
                   a.max_context, a.hdr, KID_APPEND, page, slot);
      s_page[threadIdx.x] = page;
      s_slot[threadIdx.x] = slot;
    }
    __syncthreads();
    // K/V rows to the cache
    constexpr int CH = D / 8;
    for (int it = threadIdx.x; it < cnt * CH; it += blockDim.x) {
      const int n = it / CH, c = it % CH;
      const int page = s_page[n];
      if (page < 0) continue;
      const size_t src = ((size_t(b) * a.Hkv + g) * a.max_new + t0 + n) * D + c * 8;
      const size_t dst = ((size_t(page) * a.Hkv + g) * kPage + s_slot[n]) * D + c * 8;
      *reinterpret_cast<uint4*>(a.k + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
      *reinterpret_cast<uint4*>(a.v + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
    }
    // centre and pack
    for (int it = threadIdx.x; it < cnt * GR; it += blockDim.x) {
      const int n = it / GR, gr = it % GR;
      const int page = s_page[n];
      if (page < 0) continue;
      const size_t src = ((size_t(b) * a.Hkv + g) * a.max_new + t0 + n) * D + gr * 16;
      const uint4 k0 = *reinterpret_cast<const uint4*>(a.k_new + src);
      const uint4 k1 = *reinterpret_cast<const uint4*>(a.k_new + src + 8);
      const uint32_t w[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
      float x[16];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[2 * e] = __fsub_rn(bf16_lo(w[e]), s_mu[gr * 16 + 2 * e]);
        x[2 * e + 1] = __fsub_rn(bf16_hi(w[e]), s_mu[gr * 16 + 2 * e + 1]);
      }
      uint32_t packed[2];
      const uint32_t sc = nvfp4_pack16(x, gk, packed);
      // page-head layouts read directly by the FP4 tensor-core scan (see include/qs.h)
      const size_t ph = size_t(page) * a.Hkv + g;
      const int slot = s_slot[n];
      *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(a.proxy) + ph * kNvfp4PageCodeBytes +
                                nvfp4_code_off(slot, gr)) = make_uint2(packed[0], packed[1]);
      a.proxy_scale[ph * kNvfp4PageScaleBytes + nvfp4_scale_off(slot, gr)] = uint8_t(sc);
    }
  }
  finish_append(a);
}

// ============================================================ binary-code writer
// "RaBitQCache", Abstract, with the RaBitQ code (Gao and Long, SIGMOD 2024, section 3):
// o = float(k) - c (float32), y = o R[g] with each y_i summed over j ascending (one
// rounding per product and per sum), bits b_i = [y_i > 0] packed 32 to a word by a warp
// ballot (little-endian words, so bit i lands in byte i / 8 at position i % 8), and
// g = fp32(sum_j o_j^2) / fp32(sum_i |y_i|) with both sums taken left to right (g = 0 when
// the second is 0). CTA = one row x TT tokens (16 for bulk appends, 1 for a decode step's
// single token), thread i = dimension i (blockDim = D): each R[g][j][i] is loaded once per
// CTA (16 loads in flight) and applied to the TT tokens.
template <int D, int TT>
__global__ void __launch_bounds__(D) append_rabitq_kernel(const AppendParams a) {
  constexpr int PB = kPage * (D / 8) + kPage * 4;      // bytes per (page, KV head)
  __shared__ float s_o[TT][D];
  __shared__ float s_ay[TT][D];
  __shared__ int s_page[TT], s_slot[TT];
  const int row = blockIdx.y;
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int n_b = a.n_new ? a.n_new[b] : 1;
  if (n_b < 0 || n_b > a.max_new) {
    if (tid == 0 && blockIdx.x == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_APPEND, uint32_t(b));
    n_b = 0;
  }
  const int old = a.seq_lens[b];
  const int t0 = blockIdx.x * TT;
  const int cnt = min(TT, n_b - t0);
  if (cnt > 0) {
    if (tid < TT) {
      int page = -1, slot = 0;
      if (tid < cnt)
        cache_slot(a.page_table, b, old + t0 + tid, a.max_pages_per_seq, a.num_pages,
                   a.max_context, a.hdr, KID_APPEND, page, slot);
      s_page[tid] = page;
      s_slot[tid] = slot;
    }
    const float c_i = a.key_center[size_t(row) * D + tid];
    const size_t src0 = (size_t(row) * a.max_new + t0) * D;
    for (int n = 0; n < TT; ++n)
      s_o[n][tid] = n < cnt ? __fsub_rn(bf16_to_f32(a.k_new[src0 + size_t(n) * D + tid]), c_i)
                            : 0.0f;
    __syncthreads();
    // K and V rows of the chunk's tokens -> their page slots (16 bytes per step)
    constexpr int CH = D / 8;
    for (int it = tid; it < cnt * CH; it += D) {
      const int n = it / CH, c = it % CH;
      const int page = s_page[n];
      if (page < 0) continue;
      const size_t src = src0 + size_t(n) * D + c * 8;
      const size_t dst = ((size_t(page) * a.Hkv + g) * kPage + s_slot[n]) * D + c * 8;
      *reinterpret_cast<uint4*>(a.k + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
      *reinterpret_cast<uint4*>(a.v + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
    }
    // y_i of every token of the chunk, j ascending
    const float* Rg = a.P + size_t(g) * D * D;
    float acc[TT];
#pragma unroll
    for (int n = 0; n < TT; ++n) acc[n] = 0.0f;
    for (int j0 = 0; j0 < D; j0 += 16) {             // 16 loads of R in flight at a time
      float r[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) r[u] = __ldg(Rg + size_t(j0 + u) * D + tid);
#pragma unroll
      for (int u = 0; u < 16; ++u)
#pragma unroll
        for (int n = 0; n < TT; ++n) acc[n] = __fadd_rn(acc[n], __fmul_rn(s_o[n][j0 + u], r[u]));
    }
    uint8_t* base = static_cast<uint8_t*>(a.proxy);
#pragma unroll
    for (int n = 0; n < TT; ++n) {
      const unsigned word = __ballot_sync(kFull, acc[n] > 0.0f);
      s_ay[n][tid] = fabsf(acc[n]);
      if (n < cnt && lane == 0 && s_page[n] >= 0) {
        uint8_t* pg = base + (size_t(s_page[n]) * a.Hkv + g) * PB;
        reinterpret_cast<uint32_t*>(pg + s_slot[n] * (D / 8))[warp] = word;
      }
    }
    __syncthreads();
    // the factor g of each token: one thread per token, both sums in index order
    if (tid < cnt && s_page[tid] >= 0) {
      float n2 = 0.0f, l1 = 0.0f;
      for (int j = 0; j < D; ++j) n2 = __fadd_rn(n2, __fmul_rn(s_o[tid][j], s_o[tid][j]));
      for (int i = 0; i < D; ++i) l1 = __fadd_rn(l1, s_ay[tid][i]);
      uint8_t* pg = base + (size_t(s_page[tid]) * a.Hkv + g) * PB;
      reinterpret_cast<float*>(pg + kPage * (D / 8))[s_slot[tid]] =
          l1 > 0.0f ? __fdiv_rn(n2, l1) : 0.0f;
    }
  }
  finish_append(a);
}

// ============================================================ K/V only
// The semantic-block index covers the prompt; tokens decoded after it have no scoring
// entry (they are always attended), so their append copies K and V only.
// CTA = one row x 64 tokens.
__global__ void __launch_bounds__(128) append_kv_kernel(const AppendParams a) {
  constexpr int TT = 64;
  __shared__ int s_page[TT], s_slot[TT];
  const int row = blockIdx.y;
  const int b = row / a.Hkv, g = row % a.Hkv;
  int n_b = a.n_new ? a.n_new[b] : 1;
  if (n_b < 0 || n_b > a.max_new) {
    if (threadIdx.x == 0 && blockIdx.x == 0)
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_APPEND, uint32_t(b));
    n_b = 0;
  }
  const int old = a.seq_lens[b];
  const int t0 = blockIdx.x * TT;
  const int cnt = min(TT, n_b - t0);
  if (cnt > 0) {
    if (threadIdx.x < TT) {
      int page = -1, slot = 0;
      if (int(threadIdx.x) < cnt)
        cache_slot(a.page_table, b, old + t0 + threadIdx.x, a.max_pages_per_seq, a.num_pages,
                   a.max_context, a.hdr, KID_APPEND, page, slot);
      s_page[threadIdx.x] = page;
      s_slot[threadIdx.x] = slot;
    }
    __syncthreads();
    const int CH = a.d / 8;
    for (int it = threadIdx.x; it < cnt * CH; it += blockDim.x) {
      const int n = it / CH, c = it % CH;
      const int page = s_page[n];
      if (page < 0) continue;
      const size_t src = ((size_t(row) * a.max_new) + t0 + n) * a.d + c * 8;
      const size_t dst = ((size_t(page) * a.Hkv + g) * kPage + s_slot[n]) * a.d + c * 8;
      *reinterpret_cast<uint4*>(a.k + dst) = *reinterpret_cast<const uint4*>(a.k_new + src);
      *reinterpret_cast<uint4*>(a.v + dst) = *reinterpret_cast<const uint4*>(a.v_new + src);
    }
  }
  finish_append(a);
}

// ============================================================ NVFP4 block error
// CTA = one (row, block) pair that this append may have completed; 256 threads, each
// owning (token, 16-element group) items i = tid + 256 m. An item's error is summed over
// its 16 elements in order, a thread's items in order, then warps by butterfly and the
// 8 warp sums in order: a fixed, deterministic float32 reduction.
__global__ void __launch_bounds__(256) block_err_kernel(const BlockErrParams a) {
  constexpr int D = 128, GR = D / 16;
  __shared__ float s_mu[D];
  __shared__ float s_red[8];
  pdl_wait();      // the cache and seq_lens come from the append kernel before
  pdl_trigger();
  const int row = blockIdx.y;
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int n_b = a.n_new ? a.n_new[b] : 1;
  const int new_len = a.seq_lens[b];
  const int old = new_len - n_b;
  const int j = old / a.S + blockIdx.x;
  if (n_b <= 0 || old < 0 || (j + 1) * a.S > new_len || j >= a.nb_stride) return;  // not completed here
  const float gk = *a.key_gscale;
  if (threadIdx.x < D) s_mu[threadIdx.x] = a.key_center[size_t(row) * D + threadIdx.x];
  __syncthreads();
  float err = 0.0f;
  for (int i = threadIdx.x; i < a.S * GR; i += 256) {
    const int tt = i / GR, gr = i % GR;
    const int t = j * a.S + tt;
    const int pi = t / kPage;
    if (pi >= a.max_pages_per_seq) { flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_BLOCKERR, b); continue; }
    const int page = a.page_table[size_t(b) * a.max_pages_per_seq + pi];
    if (page < 0 || page >= a.num_pages) { flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_BLOCKERR, b); continue; }
    const uint16_t* kr = a.k + ((size_t(page) * a.Hkv + g) * kPage + t % kPage) * D + gr * 16;
    const uint4 k0 = *reinterpret_cast<const uint4*>(kr);
    const uint4 k1 = *reinterpret_cast<const uint4*>(kr + 8);
    const uint32_t w[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
    float x[16];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      x[2 * e] = __fsub_rn(bf16_lo(w[e]), s_mu[gr * 16 + 2 * e]);
      x[2 * e + 1] = __fsub_rn(bf16_hi(w[e]), s_mu[gr * 16 + 2 * e + 1]);
    }
    uint32_t packed[2];
    const float sv = ue4m3_decode(nvfp4_pack16(x, gk, packed));
    float e_it = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float dq = __fmul_rn(__fmul_rn(e2m1_decode((packed[e >> 3] >> (4 * (e & 7))) & 15u), sv), gk);
      const float df = __fsub_rn(x[e], dq);
      e_it = __fadd_rn(e_it, __fmul_rn(df, df));
    }
    err = __fadd_rn(err, e_it);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) err = __fadd_rn(err, __shfl_xor_sync(kFull, err, m));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = err;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.0f;
    for (int w = 0; w < 8; ++w) tot = __fadd_rn(tot, s_red[w]);
    a.block_err[size_t(row) * a.nb_stride + j] = tot;
  }
}

// ============================================================ scoring prep
__global__ void __launch_bounds__(128) prep_rankr_kernel(const PrepParams a) {
  extern __shared__ __align__(16) float Ps[];      // P[g]: [d][r]
  __shared__ float qbar[256];
  pdl_trigger();   // the scan may launch now; it waits for this grid before reading q~
  const int row = blockIdx.x, tid = threadIdx.x;
  const int b = row / a.Hkv, g = row % a.Hkv;
  // every global load is issued before any is consumed: P[g] (at most 32 KiB) as float4
  // and the group's query elements of dimension tid
  constexpr int kMaxP4 = 128 * 64 / 4 / 128;       // float4 loads per thread (d = 128, r = 64)
  const int n4 = a.d * a.r / 4;
  const float4* Pg4 = reinterpret_cast<const float4*>(a.P + size_t(g) * a.d * a.r);
  float4 pv[kMaxP4];
#pragma unroll
  for (int j = 0; j < kMaxP4; ++j)
    if (j * 128 + tid < n4) pv[j] = Pg4[j * 128 + tid];
  const int Hq = a.Hkv * a.G;
  const bool has_q = tid < a.d;
  uint16_t qraw[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h)
    qraw[h] = (has_q && h < a.G) ? a.q[(size_t(b) * Hq + g * a.G + h) * a.d + tid] : uint16_t(0);
#pragma unroll
  for (int j = 0; j < kMaxP4; ++j)
    if (j * 128 + tid < n4) reinterpret_cast<float4*>(Ps)[j * 128 + tid] = pv[j];
  if (has_q) {
    float s = 0.0f;
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h)
      if (h < a.G) s += bf16_to_f32(qraw[h]);
    qbar[tid] = s / float(a.G);
  }
  __syncthreads();
  // q~_j = sum_i qbar_i P_ij, ascending i (the decode append's fused prep does the same)
  for (int j = tid; j < a.r; j += 128) {
    float acc = 0.0f;
#pragma unroll 8
    for (int i = 0; i < a.d; ++i) acc = fmaf(qbar[i], Ps[i * a.r + j], acc);
    a.qt[size_t(row) * a.r + j] = acc;
  }
}

// NVFP4 query packing: CTA = one row (sequence, KV head). g_q = max|q| / 2688 over the
// whole q tensor (every CTA computes the same maximum from L2-resident q; CTA 0 stores
// it), then the group's heads are packed like the keys (without centring) into the row's
// query tile: [4 chunks][8 heads][16 B] B-operand codes (heads past the group zero)
// followed by their scales in the tensor-core scale-factor order.
__global__ void __launch_bounds__(256) qpack_kernel(const QPackParams a) {
  __shared__ float s_red[8];
  __shared__ float s_g;
  pdl_trigger();   // the scan may launch now; it waits for this grid before reading the tiles
  const int tid = threadIdx.x, row = blockIdx.x;
  float m = 0.0f;
  const uint4* q4 = reinterpret_cast<const uint4*>(a.q);
  const int n4 = a.n / 8;
  for (int i0 = 0; i0 < n4; i0 += 256 * 4) {
    uint4 w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = i0 + j * 256 + tid;
      w[j] = i < n4 ? q4[i] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t x[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf16_lo(x[e])), fabsf(bf16_hi(x[e]))));
    }
  }
  m = warp_max(m);
  if ((tid & 31) == 0) s_red[tid >> 5] = m;
  uint4* tile4 = reinterpret_cast<uint4*>(a.tiles + size_t(row) * kQTileBytes);
  for (int i = tid; i < kQTileBytes / 16; i += 256) tile4[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (tid == 0) {
    float v = s_red[0];
    for (int w = 1; w < 8; ++w) v = fmaxf(v, s_red[w]);
    s_g = __fdiv_rn(v, 2688.0f);
    if (row == 0) *a.gscale = s_g;
  }
  __syncthreads();
  const float gq = s_g;
  constexpr int GR = 8;  // 16-element groups per head (d = 128)
  if (tid < a.G * GR) {
    const int gr = tid % GR, n = tid / GR;
    const int b = row / a.Hkv, g = row % a.Hkv;
    const uint16_t* qh = a.q + (size_t(b) * a.Hkv * a.G + g * a.G + n) * 128 + gr * 16;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = bf16_to_f32(qh[i]);
    uint32_t packed[2];
    const uint32_t sc = nvfp4_pack16(x, gq, packed);
    uint8_t* tile = a.tiles + size_t(row) * kQTileBytes;
    *reinterpret_cast<uint2*>(tile + qtile_code_off(n, gr)) = make_uint2(packed[0], packed[1]);
    tile[qtile_scale_off(n, gr)] = uint8_t(sc);
  }
  // Packing reads only q, so it runs alongside the kernel before; waiting for that kernel
  // before exiting keeps "this grid done" implying "every earlier grid done" for the scan.
  pdl_wait();
}

// ============================================================ launchers
template <typename PT, int R, int D>
static cudaError_t launch_rankr(const Plan& p, const AppendParams& a, cudaStream_t s) {
  constexpr int NT = 64 * R / 16;
  const size_t smem = size_t(D) * R * 4 + size_t(D) * 64 * 4;
  auto k = append_rankr_kernel<PT, R, D>;
  const cudaError_t attr = set_smem_limit(k, int(smem));
  if (attr != cudaSuccess) return attr;
  dim3 grid((a.max_new + 63) / 64, a.batch * a.Hkv);
  k<<<grid, NT, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(const Plan& p, const AppendParams& a, cudaStream_t s) {
  if (p.kind == PK_SEMANTIC) {
    append_kv_kernel<<<dim3((a.max_new + 63) / 64, a.batch * a.Hkv), 128, 0, s>>>(a);
    return cudaGetLastError();
  }
  if (p.kind == PK_RABITQ) {
    if (a.max_new == 1) {
      const dim3 grid(1, a.batch * a.Hkv);
      if (p.d == 128) append_rabitq_kernel<128, 1><<<grid, 128, 0, s>>>(a);
      else append_rabitq_kernel<64, 1><<<grid, 64, 0, s>>>(a);
    } else {
      const dim3 grid((a.max_new + 15) / 16, a.batch * a.Hkv);
      if (p.d == 128) append_rabitq_kernel<128, 16><<<grid, 128, 0, s>>>(a);
      else append_rabitq_kernel<64, 16><<<grid, 64, 0, s>>>(a);
    }
    return cudaGetLastError();
  }
  if (p.kind == PK_CENTROID) {
    // blocks a call can touch: ceil(max_new / S) + 1 (the first may be partly filled)
    const dim3 grid((a.max_new + p.S - 1) / p.S + 1, a.batch * a.Hkv);
    if (p.d == 128) append_centroid_kernel<128><<<grid, 128, 0, s>>>(a);
    else append_centroid_kernel<64><<<grid, 128, 0, s>>>(a);
    return cudaGetLastError();
  }
  if (p.kind == PK_NVFP4) {
    dim3 grid((a.max_new + 63) / 64, a.batch * a.Hkv);
    append_nvfp4_kernel<<<grid, 128, 0, s>>>(a);
    return cudaGetLastError();
  }
  const bool f32 = p.proxy_dtype == QS_F32;
  const bool fp8 = p.proxy_dtype == QS_E4M3;
  if (a.max_new == 1) {
#define QS_ONE(PT, R, D) \
  { append_one_rankr_kernel<PT, R, D><<<a.batch * a.Hkv, 128, 0, s>>>(a); return cudaGetLastError(); }
    if (fp8) {
      if (p.d == 64 && p.r == 32) QS_ONE(uint8_t, 32, 64)
      if (p.d == 128 && p.r == 32) QS_ONE(uint8_t, 32, 128)
      if (p.d == 128 && p.r == 64) QS_ONE(uint8_t, 64, 128)
      return cudaErrorInvalidValue;
    }
    if (p.d == 64) {
      if (f32 && p.r == 16) QS_ONE(float, 16, 64)
      if (!f32 && p.r == 32) QS_ONE(uint16_t, 32, 64)
    } else {
      if (f32 && p.r == 16) QS_ONE(float, 16, 128)
      if (f32 && p.r == 32) QS_ONE(float, 32, 128)
      if (!f32 && p.r == 32) QS_ONE(uint16_t, 32, 128)
      if (!f32 && p.r == 64) QS_ONE(uint16_t, 64, 128)
    }
#undef QS_ONE
    return cudaErrorInvalidValue;
  }
  if (fp8) {
    if (p.d == 64 && p.r == 32) return launch_rankr<uint8_t, 32, 64>(p, a, s);
    if (p.d == 128 && p.r == 32) return launch_rankr<uint8_t, 32, 128>(p, a, s);
    if (p.d == 128 && p.r == 64) return launch_rankr<uint8_t, 64, 128>(p, a, s);
    return cudaErrorInvalidValue;
  }
  if (p.d == 64) {
    if (f32 && p.r == 16) return launch_rankr<float, 16, 64>(p, a, s);
    if (!f32 && p.r == 32) return launch_rankr<uint16_t, 32, 64>(p, a, s);
  } else {
    if (f32 && p.r == 16) return launch_rankr<float, 16, 128>(p, a, s);
    if (f32 && p.r == 32) return launch_rankr<float, 32, 128>(p, a, s);
    if (!f32 && p.r == 32) return launch_rankr<uint16_t, 32, 128>(p, a, s);
    if (!f32 && p.r == 64) return launch_rankr<uint16_t, 64, 128>(p, a, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_block_err(const Plan& p, const BlockErrParams& a, cudaStream_t s) {
  return launch_k(block_err_kernel, dim3(a.max_blocks_per_call, a.batch * a.Hkv), dim3(256), 0, s,
                  true, a);
}

cudaError_t launch_prep(const Plan& p, const PrepParams& a, cudaStream_t s) {
  const size_t smem = size_t(a.d) * a.r * sizeof(float);      // <= 32 KiB
  prep_rankr_kernel<<<a.batch * a.Hkv, 128, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_qpack(const Plan& p, const QPackParams& a, cudaStream_t s, bool pdl) {
  return launch_k(qpack_kernel, dim3(a.rows), dim3(256), 0, s, pdl, a);
}

}  // namespace qs
