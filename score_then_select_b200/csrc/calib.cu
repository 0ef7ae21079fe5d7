// calib.cu - the shared scoring basis P of each KV head from calibration queries and keys.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Abstract and
// Table 9: the subspace is learned by minimising a tractable bound on the token-score
// preservation error, whose solution is spectral, and the pages compare raw with
// unit-trace-normalised group-mean moments. Reading (the bound is not on the pages):
//   M = C_q / tr(C_q) + C_k / tr(C_k),  C_q = mean over positions of qbar qbar^T (qbar =
//   mean of the group's query heads), C_k = mean of k k^T;  P = top-r eigenvectors of M,
//   eigenvalue descending, each column signed so that its largest-magnitude entry (lowest
//   index on ties) is positive.
// Calibration runs once, before decoding; it is not part of the decode step.
//
//   moments_kernel: CTA = (KV head, 32 x 32 tile of C_q and C_k); FP64 sums over the
//                   positions, staged 32 positions at a time through shared memory.
//   basis_kernel:   CTA = one KV head; cyclic Jacobi eigenvalue iteration on M (FP64 in
//                   shared memory) with the eigenvectors accumulated in FP32. Each round
//                   rotates d/2 disjoint index pairs (round-robin ordering, so the rotations
//                   of a round commute and run in parallel); sweeps stop when the
//                   off-diagonal mass is below 1e-26 of the total (at most 40 sweeps).
#include "qs_device.cuh"

namespace qs {

constexpr int kCalTile = 32;
constexpr int kCalChunk = 32;          // positions per shared-memory stage
constexpr int kCalThreads = 256;
constexpr int kBasisThreads = 1024;
constexpr int kMaxSweeps = 40;

__global__ void __launch_bounds__(kCalThreads) moments_kernel(const CalibParams a) {
  __shared__ double qi[kCalChunk][kCalTile], qj[kCalChunk][kCalTile];
  __shared__ double ki[kCalChunk][kCalTile], kj[kCalChunk][kCalTile];
  const int g = blockIdx.x, i0 = blockIdx.y * kCalTile, j0 = blockIdx.z * kCalTile;
  const int tid = threadIdx.x;
  const int Hq = a.Hkv * a.G;
  // this thread's 4 entries of the tile: row ti, columns tj, tj + 8, tj + 16, tj + 24
  const int ti = tid / 8, tj = tid % 8;
  double sq[4] = {0.0, 0.0, 0.0, 0.0}, sk[4] = {0.0, 0.0, 0.0, 0.0};
  for (int t0 = 0; t0 < a.n; t0 += kCalChunk) {
    __syncthreads();
    for (int e = tid; e < kCalChunk * kCalTile * 2; e += kCalThreads) {
      const int side = e / (kCalChunk * kCalTile);       // 0: columns i, 1: columns j
      const int rem = e % (kCalChunk * kCalTile);
      const int t = rem / kCalTile, c = rem % kCalTile;
      const int col = (side ? j0 : i0) + c;
      double qv = 0.0, kv = 0.0;
      if (t0 + t < a.n) {
        const size_t pos = size_t(t0 + t);
        for (int h = 0; h < a.G; ++h)
          qv += double(bf16_to_f32(a.q[(pos * Hq + size_t(g) * a.G + h) * a.d + col]));
        qv /= double(a.G);
        kv = double(bf16_to_f32(a.k[(pos * a.Hkv + g) * a.d + col]));
      }
      (side ? qj : qi)[t][c] = qv;
      (side ? kj : ki)[t][c] = kv;
    }
    __syncthreads();
    for (int t = 0; t < kCalChunk; ++t) {
      const double x = qi[t][ti], y = ki[t][ti];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        sq[u] = fma(x, qj[t][tj + 8 * u], sq[u]);
        sk[u] = fma(y, kj[t][tj + 8 * u], sk[u]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const size_t o = (size_t(g) * a.d + i0 + ti) * a.d + j0 + tj + 8 * u;
    a.mq[o] = sq[u];
    a.mk[o] = sk[u];
  }
}

__global__ void __launch_bounds__(kBasisThreads) basis_kernel(const CalibParams a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int d = a.d, half = d / 2, g = blockIdx.x, tid = threadIdx.x;
  double* A = reinterpret_cast<double*>(smem_raw);                 // [d][d]
  float* V = reinterpret_cast<float*>(A + d * d);                   // [d][d]
  double* cs = reinterpret_cast<double*>(V + d * d);               // [half][2] cos, sin
  int* pq = reinterpret_cast<int*>(cs + 2 * half);                 // [half][2]
  double* red = reinterpret_cast<double*>(pq + 2 * half);          // [64] reduction
  int* rank = reinterpret_cast<int*>(red + 64);                    // [d]
  __shared__ double s_tr[2];
  __shared__ int s_done;

  const double* mq = a.mq + size_t(g) * d * d;
  const double* mk = a.mk + size_t(g) * d * d;
  if (tid < 2) {
    const double* m = tid == 0 ? mq : mk;
    double t = 0.0;
    for (int i = 0; i < d; ++i) t += m[i * d + i];
    s_tr[tid] = t;
  }
  __syncthreads();
  // the positions' count cancels in each normalised term
  const double iq = s_tr[0] > 0.0 ? 1.0 / s_tr[0] : 0.0, ik = s_tr[1] > 0.0 ? 1.0 / s_tr[1] : 0.0;
  for (int e = tid; e < d * d; e += kBasisThreads) {
    A[e] = mq[e] * iq + mk[e] * ik;
    V[e] = (e / d == e % d) ? 1.0f : 0.0f;
  }
  __syncthreads();

  for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
    for (int round = 0; round < d - 1; ++round) {
      // round-robin pairs: position 0 holds index 0, position i > 0 holds
      // 1 + (i - 1 + round) mod (d - 1); position i meets position d - 1 - i
      if (tid < half) {
        auto at = [&](int pos) { return pos == 0 ? 0 : 1 + (pos - 1 + round) % (d - 1); };
        int p = at(tid), q = at(d - 1 - tid);
        if (p > q) { const int t = p; p = q; q = t; }
        const double apq = A[p * d + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          // Golub & Van Loan, symmetric Schur decomposition of a 2 x 2 block
          const double theta = (A[q * d + q] - A[p * d + p]) / (2.0 * apq);
          const double t = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(1.0 + theta * theta));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        cs[2 * tid] = c;
        cs[2 * tid + 1] = s;
        pq[2 * tid] = p;
        pq[2 * tid + 1] = q;
      }
      __syncthreads();
      // rows p, q of every pair: A <- J^T A
      for (int e = tid; e < half * d; e += kBasisThreads) {
        const int pr = e / d, col = e % d;
        const int p = pq[2 * pr], q = pq[2 * pr + 1];
        const double c = cs[2 * pr], s = cs[2 * pr + 1];
        const double ap = A[p * d + col], aq = A[q * d + col];
        A[p * d + col] = c * ap - s * aq;
        A[q * d + col] = s * ap + c * aq;
      }
      __syncthreads();
      // columns p, q of every pair: A <- A J, V <- V J
      for (int e = tid; e < half * d; e += kBasisThreads) {
        const int pr = e / d, row = e % d;
        const int p = pq[2 * pr], q = pq[2 * pr + 1];
        const double c = cs[2 * pr], s = cs[2 * pr + 1];
        const double ap = A[row * d + p], aq = A[row * d + q];
        A[row * d + p] = c * ap - s * aq;
        A[row * d + q] = s * ap + c * aq;
        const float fc = float(c), fs = float(s);
        const float vp = V[row * d + p], vq = V[row * d + q];
        V[row * d + p] = fc * vp - fs * vq;
        V[row * d + q] = fs * vp + fc * vq;
      }
      __syncthreads();
    }
    // convergence: off-diagonal mass against the total
    double off = 0.0, tot = 0.0;
    for (int e = tid; e < d * d; e += kBasisThreads) {
      const double x = A[e] * A[e];
      tot += x;
      if (e / d != e % d) off += x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(kFull, off, o);
      tot += __shfl_xor_sync(kFull, tot, o);
    }
    if ((tid & 31) == 0) {
      red[tid >> 5] = off;
      red[32 + (tid >> 5)] = tot;
    }
    __syncthreads();
    if (tid == 0) {
      double o2 = 0.0, t2 = 0.0;
      for (int w = 0; w < kBasisThreads / 32; ++w) {
        o2 += red[w];
        t2 += red[32 + w];
      }
      s_done = (o2 <= 1e-26 * t2) ? 1 : 0;
    }
    __syncthreads();
    if (s_done) break;
  }

  // eigenvalues: the diagonal; rank = number of larger ones (lower index first on ties)
  if (tid < d) {
    const double li = A[tid * d + tid];
    int rk = 0;
    for (int j = 0; j < d; ++j) {
      const double lj = A[j * d + j];
      rk += (lj > li) || (lj == li && j < tid);
    }
    rank[tid] = rk;
  }
  __syncthreads();
  // columns of rank < r: signed so that the largest-magnitude entry is positive
  if (tid < d && rank[tid] < a.r) {
    const int c = tid, rk = rank[tid];
    int best = 0;
    float bv = -1.0f;
    for (int i = 0; i < d; ++i) {
      const float x = fabsf(V[i * d + c]);
      if (x > bv) { bv = x; best = i; }
    }
    const float sgn = V[best * d + c] < 0.0f ? -1.0f : 1.0f;
    float* Pg = a.P + size_t(g) * d * a.r;
    for (int i = 0; i < d; ++i) Pg[size_t(i) * a.r + rk] = sgn * V[i * d + c];
    if (a.eig) a.eig[size_t(g) * a.r + rk] = float(A[c * d + c]);
  }
}

size_t calib_ws_bytes(int Hkv, int d) { return size_t(kHdrWords) * 4 + 2 * size_t(Hkv) * d * d * 8; }

cudaError_t launch_calibrate(const CalibParams& a, cudaStream_t s) {
  const dim3 grid(a.Hkv, a.d / kCalTile, a.d / kCalTile);
  moments_kernel<<<grid, kCalThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int d = a.d;
  auto bytes = [](int dd) {
    return size_t(dd) * dd * 8 + size_t(dd) * dd * 4 + size_t(dd / 2) * 2 * 8 +
           size_t(dd / 2) * 2 * 4 + 64 * 8 + size_t(dd) * 4;
  };
  const size_t smem = bytes(d);                     // 194.5 KiB at d = 128
  const cudaError_t attr = set_smem_limit(basis_kernel, int(bytes(128)));
  if (attr != cudaSuccess) return attr;
  basis_kernel<<<a.Hkv, kBasisThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace qs
