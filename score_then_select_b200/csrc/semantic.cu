// semantic.cu - the semantic-block index (float32 k-means over the prompt's keys) and its
// decode side ("Coarse Semantic Blocks for Efficient Training-Free Sparse Attention",
// Abstract; the readings are in semantic.h).
//
// Index build, per row (sequence b, KV head g), L0 = the prompt length, C = ceil(L0 / S):
//   sem_seed_kernel:   c_j = key at floor(j * L0 / C).
//   then `iters` times:
//   sem_assign_kernel: CTA = (row, page of 128 keys), thread = key; the page's keys sit
//                      transposed in shared memory (conflict-free per-thread columns), the
//                      centroids stream through in chunks of 32; distances summed over the
//                      dimensions in order with one rounding per operation.
//   sem_csr_kernel:    CTA = row: member counts, offsets (exclusive scan), then a stable
//                      fill: 1,024 keys at a time, warps in order, each warp's equal-cluster
//                      lanes found with match.any, so members stay in token order.
//   sem_update_kernel: thread = (cluster, dimension): the members' sum in token order, then
//                      one division by the count (an empty cluster keeps its centroid).
// Decode:
//   sem_score_kernel:  CTA = (row, 32 clusters), qbar formed once in shared memory, a warp
//                      per 4 clusters: beta_j = qbar . c_j (float32).
//   (the existing select kernel picks the top clusters over C_b candidates)
//   sem_expand_kernel: CTA = row: the selected clusters' members, then the tokens after the
//                      prompt, as the row's token list for the token-level attention.
#include <cfloat>

#include "qs_device.cuh"
#include "semantic.h"

namespace qs {

constexpr int kSemTile = 128;        // keys per assignment CTA (one page)
constexpr int kSemChunk = 32;        // centroids per shared-memory chunk
constexpr int kSemThreads = 1024;    // CSR and expansion CTAs

QS_DEV int sem_clusters(int L0, int S) { return L0 > 0 ? (L0 + S - 1) / S : 0; }

// The prompt length of sequence b, clamped to the index's capacity.
QS_DEV int sem_prompt(const int32_t* prompt_lens, int b, int l_max) {
  const int L0 = prompt_lens[b];
  return L0 < 0 ? 0 : (L0 > l_max ? l_max : L0);
}

// Pointer to key t of row (b, g) in the paged cache, or nullptr (and an error flag).
QS_DEV const uint16_t* sem_key(const SemIndexParams& a, int b, int g, int t) {
  const int pi = t / kPage;
  int page = -1;
  if (pi < a.max_pages_per_seq) page = a.page_table[size_t(b) * a.max_pages_per_seq + pi];
  if (page < 0 || page >= a.num_pages) {
    flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SEMANTIC, uint32_t(b));
    return nullptr;
  }
  return a.k + ((size_t(page) * a.Hkv + g) * kPage + (t % kPage)) * a.d;
}

// Exclusive prefix of v over the CTA's threads in order (blockDim = kSemThreads); total
// receives the sum of all v.
QS_DEV int sem_scan(int v, int* s, int& total) {
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
  total = s[kSemThreads / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// ============================================================ index build
__global__ void __launch_bounds__(256) sem_seed_kernel(const SemIndexParams a) {
  const int row = blockIdx.x, b = row / a.Hkv, g = row % a.Hkv;
  const int L0 = sem_prompt(a.prompt_lens, b, a.l_max);
  const int C = min(sem_clusters(L0, a.S), a.c_max);
  float* cent = a.cent + size_t(row) * a.c_max * a.d;
  for (int e = threadIdx.x; e < C * a.d; e += blockDim.x) {
    const int j = e / a.d, i = e % a.d;
    const int t = int((long long)j * L0 / C);
    const uint16_t* kp = sem_key(a, b, g, t);
    cent[size_t(j) * a.d + i] = kp ? bf16_to_f32(kp[i]) : 0.0f;
  }
}

template <int D>
__global__ void __launch_bounds__(kSemTile) sem_assign_kernel(const SemIndexParams a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* xs = reinterpret_cast<float*>(smem_raw);                  // [D][kSemTile]
  float* cs = xs + D * kSemTile;                                    // [kSemChunk][D]
  const int row = blockIdx.y, b = row / a.Hkv, g = row % a.Hkv, tid = threadIdx.x;
  const int L0 = sem_prompt(a.prompt_lens, b, a.l_max);
  const int C = min(sem_clusters(L0, a.S), a.c_max);
  const int t0 = blockIdx.x * kSemTile;
  if (t0 >= L0) return;
  const uint16_t* kp = sem_key(a, b, g, t0);                        // the page's first key
  if (!kp) return;
  // the page's keys, transposed: xs[i][t]
  for (int e = tid; e < kSemTile * D; e += kSemTile) {
    const int t = e / D, i = e % D;
    xs[i * kSemTile + t] = t0 + t < L0 ? bf16_to_f32(kp[size_t(t) * D + i]) : 0.0f;
  }
  const float* cent = a.cent + size_t(row) * a.c_max * D;
  float best = INFINITY;
  int arg = 0;
  for (int c0 = 0; c0 < C; c0 += kSemChunk) {
    const int n = min(kSemChunk, C - c0);
    __syncthreads();
    for (int e = tid; e < n * D; e += kSemTile) cs[e] = cent[size_t(c0) * D + e];
    __syncthreads();
    for (int jj = 0; jj < n; ++jj) {
      float dist = 0.0f;
#pragma unroll 8
      for (int i = 0; i < D; ++i) {
        const float diff = __fsub_rn(xs[i * kSemTile + tid], cs[jj * D + i]);
        dist = __fadd_rn(dist, __fmul_rn(diff, diff));
      }
      if (dist < best) {
        best = dist;
        arg = c0 + jj;
      }
    }
  }
  if (t0 + tid < L0) a.assign[size_t(row) * a.l_max + t0 + tid] = arg;
}

__global__ void __launch_bounds__(kSemThreads) sem_csr_kernel(const SemIndexParams a) {
  __shared__ int s_scan[kSemThreads / 32];
  const int row = blockIdx.x, b = row / a.Hkv, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int L0 = sem_prompt(a.prompt_lens, b, a.l_max);
  const int C = min(sem_clusters(L0, a.S), a.c_max);
  const int32_t* asg = a.assign + size_t(row) * a.l_max;
  int32_t* cur = a.cursor + size_t(row) * a.c_max;
  int32_t* off = a.offsets + size_t(row) * (a.c_max + 1);
  int32_t* mem = a.members + size_t(row) * a.l_max;
  // member counts
  for (int j = tid; j < C; j += kSemThreads) cur[j] = 0;
  __syncthreads();
  for (int t = tid; t < L0; t += kSemThreads) {
    const int j = asg[t];
    if (j >= 0 && j < C) atomicAdd(&cur[j], 1);
    else flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SEMANTIC, uint32_t(row));
  }
  __syncthreads();
  // offsets: exclusive prefix of the counts
  int running = 0;
  for (int base = 0; base < C; base += kSemThreads) {
    const int j = base + tid;
    const int v = j < C ? cur[j] : 0;
    int total;
    const int ex = sem_scan(v, s_scan, total);
    if (j < C) off[j] = running + ex;
    running += total;
  }
  if (tid == 0) off[C] = running;
  __syncthreads();
  for (int j = tid; j < C; j += kSemThreads) cur[j] = 0;
  // stable fill: keys in order, 1,024 at a time; warps take turns
  for (int base = 0; base < L0; base += kSemThreads) {
    const int t = base + tid;
    int j = t < L0 ? asg[t] : -1;
    if (j >= C) j = -1;
    const unsigned grp = __match_any_sync(kFull, j);
    const int rank = __popc(grp & ((1u << lane) - 1u));
    const int leader = __ffs(grp) - 1;
    for (int w = 0; w < kSemThreads / 32; ++w) {
      __syncthreads();
      if (warp == w) {                     // the whole warp: each lane reads its group leader
        int pos = 0;
        if (j >= 0 && lane == leader) {
          pos = cur[j];
          cur[j] = pos + __popc(grp);
        }
        pos = __shfl_sync(kFull, pos, leader);
        if (j >= 0) mem[off[j] + pos + rank] = t;
      }
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256) sem_update_kernel(const SemIndexParams a) {
  const int row = blockIdx.y, b = row / a.Hkv, g = row % a.Hkv;
  const int L0 = sem_prompt(a.prompt_lens, b, a.l_max);
  const int C = min(sem_clusters(L0, a.S), a.c_max);
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = e / a.d, i = e % a.d;
  if (j >= C) return;
  const int32_t* off = a.offsets + size_t(row) * (a.c_max + 1);
  const int32_t* mem = a.members + size_t(row) * a.l_max;
  const int lo = off[j], hi = off[j + 1];
  if (hi <= lo) return;                                  // empty: the centroid stays
  float s = 0.0f;
  for (int m = lo; m < hi; ++m) {
    const uint16_t* kp = sem_key(a, b, g, mem[m]);
    s = __fadd_rn(s, kp ? bf16_to_f32(kp[i]) : 0.0f);
  }
  a.cent[(size_t(row) * a.c_max + j) * a.d + i] = __fdiv_rn(s, float(hi - lo));
}

cudaError_t launch_sem_index(const SemIndexParams& a, int iters, cudaStream_t s) {
  const int rows = a.batch * a.Hkv;
  sem_seed_kernel<<<rows, 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t(a.d) * kSemTile + size_t(kSemChunk) * a.d) * sizeof(float);
  auto assign = a.d == 128 ? sem_assign_kernel<128> : sem_assign_kernel<64>;
  if ((e = set_smem_limit(assign, int(smem))) != cudaSuccess) return e;
  const dim3 agrid((a.l_max + kSemTile - 1) / kSemTile, rows);
  const dim3 ugrid((a.c_max * a.d + 255) / 256, rows);
  for (int it = 0; it < (iters < 1 ? 1 : iters); ++it) {
    assign<<<agrid, kSemTile, smem, s>>>(a);
    sem_csr_kernel<<<rows, kSemThreads, 0, s>>>(a);
    sem_update_kernel<<<ugrid, 256, 0, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ============================================================ decode
constexpr int kSemScoreWarps = 8;
constexpr int kSemScorePerWarp = 4;                        // clusters per warp

// CTA = (row, 32 clusters): beta_j = qbar . c_j (float32); -inf past the row's clusters.
// qbar (the group's head sum in order, divided by G) is formed once per CTA in shared
// memory; warp w scores clusters 4w .. 4w + 3 of the CTA's 32, lane l summing dimensions
// l + 32 m in order and the lanes combined by shuffles. Also writes each sequence's
// cluster count, which the select kernel takes as its number of candidates.
template <int D>
__global__ void __launch_bounds__(kSemScoreWarps * 32) sem_score_kernel(const SemSelectParams a) {
  constexpr int PER = D / 32;
  constexpr int CPB = kSemScoreWarps * kSemScorePerWarp;
  __shared__ float s_qbar[D];
  const int row = blockIdx.y, b = row / a.Hkv, g = row % a.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L0 = sem_prompt(a.prompt_lens, b, a.l_max);
  const int C = min(sem_clusters(L0, a.S), a.c_max);
  if (blockIdx.x == 0 && g == 0 && threadIdx.x == 0) a.n_clusters[b] = C;
  const int Hq = a.Hkv * a.G;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    float s = 0.0f;
    for (int h = 0; h < a.G; ++h)
      s += bf16_to_f32(a.q[(size_t(b) * Hq + size_t(g) * a.G + h) * D + i]);
    s_qbar[i] = s / float(a.G);
  }
  __syncthreads();
  float* out = a.scores + size_t(row) * a.c_max;
  const int j0 = blockIdx.x * CPB + warp * kSemScorePerWarp;
  float cv[kSemScorePerWarp][PER];
#pragma unroll
  for (int u = 0; u < kSemScorePerWarp; ++u) {
    const int j = j0 + u;
    const float* c = a.cent + (size_t(row) * a.c_max + (j < C ? j : 0)) * D;
#pragma unroll
    for (int m = 0; m < PER; ++m) cv[u][m] = j < C ? __ldg(c + lane + 32 * m) : 0.0f;
  }
#pragma unroll
  for (int u = 0; u < kSemScorePerWarp; ++u) {
    const int j = j0 + u;
    if (j >= a.c_max) break;                       // warp-uniform
    float dot = 0.0f;
#pragma unroll
    for (int m = 0; m < PER; ++m) dot = fmaf(cv[u][m], s_qbar[lane + 32 * m], dot);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(kFull, dot, o);
    if (lane == 0) out[j] = j < C ? dot : -INFINITY;
  }
}

// CTA (row, 0): the members of the selected clusters (each cluster's in token order, the
// clusters in the order selected), then the tokens after the prompt, L0 <= t < seq_len.
// A scan over the selected clusters' sizes gives each cluster's place in the list; warp w
// then copies clusters w, w + 32, ..., its lanes striding over the cluster's members.
// CTAs (row, 1 .. kSemPadParts): the rest of the row's list, up to max_tokens, padded with
// -1 in kSemPadParts slices by 16-byte stores; each finds the list's length n itself from
// the selected clusters' sizes.
constexpr int kSemPadParts = 7;
__global__ void __launch_bounds__(kSemThreads) sem_expand_kernel(const SemSelectParams a) {
  __shared__ int s_scan[kSemThreads / 32];
  __shared__ int s_lo[kSemThreads], s_sz[kSemThreads], s_dst[kSemThreads];
  const int row = blockIdx.x, b = row / a.Hkv, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int L0 = sem_prompt(a.prompt_lens, b, a.l_max);
  const int C = min(sem_clusters(L0, a.S), a.c_max);
  int L = a.seq_lens[b];
  if (L < L0) L = L0;
  const int32_t* off = a.offsets + size_t(row) * (a.c_max + 1);
  const int32_t* mem = a.members + size_t(row) * a.l_max;
  const int32_t* cs = a.csel + size_t(row) * a.budget;
  int32_t* out = a.tokens + size_t(row) * a.max_tokens;
  int ncs = a.n_csel[row];
  if (ncs < 0 || ncs > a.budget) {
    if (tid == 0 && blockIdx.y == 0)
      flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SEMANTIC, uint32_t(row));
    ncs = 0;
  }
  if (blockIdx.y > 0) {
    // the list's length, as CTA (row, 0) forms it
    int sz = 0;
    for (int i = tid; i < ncs; i += kSemThreads) {
      const int c = cs[i];
      if (c >= 0 && c < C) sz += off[c + 1] - off[c];
    }
    int total;
    sem_scan(sz, s_scan, total);
    const int n = min(a.max_tokens, total + (L - L0));
    // 4-byte stores up to a 16-byte boundary and after the last whole vector (slice 0),
    // 16-byte stores in between, split into kSemPadParts slices
    int i0 = n;
    while (i0 < a.max_tokens && (reinterpret_cast<uintptr_t>(out + i0) & 15u) != 0u) ++i0;
    const int nv = (a.max_tokens - i0) / 4;
    const int p = int(blockIdx.y) - 1, P = int(gridDim.y) - 1;
    const int v0 = int((long long)nv * p / P), v1 = int((long long)nv * (p + 1) / P);
    int4* out4 = reinterpret_cast<int4*>(out + i0);
    for (int i = v0 + tid; i < v1; i += kSemThreads) out4[i] = make_int4(-1, -1, -1, -1);
    if (p == 0) {
      if (tid < i0 - n) out[n + tid] = -1;
      for (int i = i0 + 4 * nv + tid; i < a.max_tokens; i += kSemThreads) out[i] = -1;
    }
    return;
  }
  int running = 0;
  bool over = false;
  for (int base = 0; base < ncs; base += kSemThreads) {
    const int i = base + tid;
    const int c = i < ncs ? cs[i] : -1;
    const bool ok = c >= 0 && c < C;
    if (i < ncs && !ok) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SEMANTIC, uint32_t(row));
    const int lo = ok ? off[c] : 0, sz = ok ? off[c + 1] - lo : 0;
    int total;
    const int dst = running + sem_scan(sz, s_scan, total);
    s_lo[tid] = lo;
    s_sz[tid] = sz;
    s_dst[tid] = dst;
    __syncthreads();
    const int nc = min(kSemThreads, ncs - base);
    for (int k = warp; k < nc; k += kSemThreads / 32) {
      const int klo = s_lo[k], ksz = s_sz[k], kdst = s_dst[k];
      for (int m = lane; m < ksz; m += 32) {
        if (kdst + m < a.max_tokens) out[kdst + m] = mem[klo + m];
        else over = true;
      }
    }
    __syncthreads();                               // before the next batch's table
    running += total;
  }
  for (int t = L0 + tid; t < L; t += kSemThreads) {
    const int pos = running + (t - L0);
    if (pos < a.max_tokens) out[pos] = t;
    else over = true;
  }
  if (over) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_SEMANTIC, uint32_t(row));
  int n = running + (L - L0);
  if (n > a.max_tokens) n = a.max_tokens;
  if (tid == 0) a.n_tokens[row] = n;
}

cudaError_t launch_sem_score(const SemSelectParams& a, cudaStream_t s) {
  constexpr int CPB = kSemScoreWarps * kSemScorePerWarp;
  const dim3 grid((a.c_max + CPB - 1) / CPB, a.batch * a.Hkv);
  if (a.d == 128) sem_score_kernel<128><<<grid, kSemScoreWarps * 32, 0, s>>>(a);
  else sem_score_kernel<64><<<grid, kSemScoreWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_sem_expand(const SemSelectParams& a, cudaStream_t s) {
  sem_expand_kernel<<<dim3(a.batch * a.Hkv, 1 + kSemPadParts), kSemThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace qs
