// attn_gather.cu - split-K sparse attention with its LSE combine, for selections of short
// runs (block size < 8, e.g. token-level selection) and for shapes with too little work per
// CTA for the tile pipeline of attn.cu (one CTA per (row, split), no separate merge launch).
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1 and
// Abstract: gather-free indexed attention reads the original full-dimensional keys and
// values of the selected positions straight from the standard GQA paged cache, with a
// distinct selection per KV head shared by that head's query heads.
// "Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention", Full
// text: value aggregation in FP16 with FP32 accumulation over contiguous block tiles.
//
// A split is a slice of a row's selected token slots (the plan's tokens per split); the
// row's splits that hold slots are taken by the row's CTAs in turn (CTA x: splits x,
// x + gridDim.x, ...). A split is streamed in 64-token tiles (K and V, 16-byte cp.async
// into an XOR-swizzled 3-stage ring); each of the 4 warps owns 16 tokens of a tile and
// keeps its own online-softmax state. The first two tiles' pages are resolved and their
// loads started before the rest of the split's pages are resolved. Each split writes one
// partial; the CTA completing the row's last split merges them.
//
// Tensor-core mapping and online softmax: attn_warp_tile (attn_core.cuh).
#include "attn_core.cuh"

namespace qs {

constexpr int kGTileT = 64;
constexpr int kGStages = 3;
constexpr int kGMaxTokensPerSplit = 2048;
constexpr int kGEntCap = kGMaxTokensPerSplit / 16 + 8;   // staged entries (blocks >= 16 tokens)

template <int D>
struct GatherSmem {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kTileBytes = kGTileT * kRowBytes;          // one of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kRingBytes = kGStages * kStageBytes;
  static constexpr int kRowsOff = kRingBytes;                    // int32 [kGMaxTokensPerSplit]
  static constexpr int kTotal = kRowsOff + kGMaxTokensPerSplit * 4;
};

// byte offset of (token row r, 16-byte chunk c) inside a swizzled tile
template <int D>
QS_DEV uint32_t gswz(int r, int c) {
  return uint32_t(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

template <int D>
QS_DEV void gather_merge_row(const AttnParams& a, int row, int nsp, uint8_t* smem);

template <int D, bool V_F16, bool AGG_F16>
__global__ void __launch_bounds__(128, 2) attn_gather_kernel(const AttnParams a) {
  using SM = GatherSmem<D>;
  constexpr int KS = D / 16;       // k-steps over the head dimension
  constexpr int CH = D / 8;        // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem[];
  int* s_rows = reinterpret_cast<int*>(smem + SM::kRowsOff);

  pdl_wait();      // the selection comes from the kernel before
  const int row = blockIdx.y;
  const int b = row / a.Hkv, g = row % a.Hkv;
  const int Hq = a.Hkv * a.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  int n = a.n_sel[row];
  int L = a.seq_lens[b];
  if (n < 0 || n > a.budget || L < 0) {
    if (tid == 0) flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_ATTN, uint32_t(row));
    n = 0;
  }
  const int slots = n * a.S;
  // The row's splits that hold slots (at least one, so that an empty row is merged to 0).
  // CTA x of the row's gridDim.x takes splits x, x + gridDim.x, ...: the grid has as many
  // splits per row as a full selection needs when they fit in one wave of resident CTAs,
  // fewer otherwise, so that short selections under a large budget (token lists of
  // clusters) do not leave most of the grid's CTAs empty.
  const int nsp = max(1, (slots + a.g_tokens_per_split - 1) / a.g_tokens_per_split);
  __shared__ int s_last;
  for (int split = blockIdx.x; split < nsp; split += gridDim.x) {
    const int s0 = split * a.g_tokens_per_split;
    const int s1 = min(s0 + a.g_tokens_per_split, slots);
    // slots of this split; none when the row selected fewer slots than the splits before it
    // cover (s0 >= slots), so that every index below stays inside the split's table
    const int cnt = max(0, s1 - s0);

    // ---------------- token table of this split: cache row index of each slot, or -1.
    // Slots [lo, hi) are resolved on demand: for blocks of >= 16 tokens each selection entry
    // (a block inside one page) is looked up once into a small staging table; for smaller
    // blocks each slot looks up its own block. Lookups are issued 8 per thread at a time.
    // The first two tiles are resolved first so that their loads start before the rest of
    // the table is built.
    __shared__ int e_base[kGEntCap], e_len[kGEntCap];
    const int32_t* selr = a.sel + size_t(row) * a.budget;
    const int nbr = (L + a.S - 1) / a.S;
    auto lookup = [&](int blk, int& pg) {      // physical page of a selected block, or -1
      pg = -1;
      if (blk < 0 || blk >= nbr) {
        flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_ATTN, uint32_t(row));
        return;
      }
      const int pi = blk * a.S / kPage;
      pg = pi < a.max_pages_per_seq ? a.page_table[size_t(b) * a.max_pages_per_seq + pi] : -1;
      if (pg < 0 || pg >= a.num_pages) {
        flag_error(a.hdr, QS_ERR_DEVICE_BOUNDS, KID_ATTN, uint32_t(row));
        pg = -1;
      }
    };
    auto resolve = [&](int lo, int hi) {       // slots [lo, hi) of this split, hi <= cnt
      if (hi <= lo) return;
      if (a.S >= 16) {
        const int e0 = (s0 + lo) / a.S, ne = (s0 + hi - 1) / a.S + 1 - e0;
        for (int u0 = 0; u0 < ne; u0 += 128 * 8) {
          int blk[8], pg[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int u = u0 + j * 128 + tid;
            blk[j] = u < ne ? selr[e0 + u] : -1;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int u = u0 + j * 128 + tid;
            pg[j] = -1;
            if (u < ne) lookup(blk[j], pg[j]);
            if (u < ne) {
              const int t0 = blk[j] * a.S;
              e_base[u] = pg[j] >= 0 ? (pg[j] * a.Hkv + g) * kPage + (t0 % kPage) : -1;
              e_len[u] = pg[j] >= 0 ? min(a.S, L - t0) : 0;
            }
          }
        }
        __syncthreads();
        for (int i = lo + tid; i < hi; i += 128) {
          const int gs = s0 + i;
          const int u = gs / a.S - e0, off = gs % a.S;
          s_rows[i] = off < e_len[u] ? e_base[u] + off : -1;
        }
        __syncthreads();
      } else {
        for (int i0 = lo; i0 < hi; i0 += 128 * 8) {
          int blk[8], pg[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * 128 + tid;
            blk[j] = i < hi ? selr[(s0 + i) / a.S] : -1;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int i = i0 + j * 128 + tid;
            if (i < hi) {
              lookup(blk[j], pg[j]);
              const int t = blk[j] * a.S + (s0 + i) % a.S;
              s_rows[i] = (pg[j] >= 0 && t < L) ? (pg[j] * a.Hkv + g) * kPage + (t % kPage) : -1;
            }
          }
        }
      }
    };
    const int tiles = (cnt + kGTileT - 1) / kGTileT;
    for (int i = cnt + tid; i < tiles * kGTileT; i += 128) s_rows[i] = -1;
    const int head = min(cnt, 2 * kGTileT);
    resolve(0, head);

    // ---------------- query fragments (B operand of S^T): head = lane/4, dims 2*(lane%4)+{0,1}
    uint32_t qb[KS][2];
    {
      const int h = lane >> 2;
      const uint16_t* qr = a.q + (size_t(b) * Hq + g * a.G + (h < a.G ? h : 0)) * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int d0 = ks * 16 + 2 * (lane & 3);
        qb[ks][0] = h < a.G ? *reinterpret_cast<const uint32_t*>(qr + d0) : 0u;
        qb[ks][1] = h < a.G ? *reinterpret_cast<const uint32_t*>(qr + d0 + 8) : 0u;
      }
    }
    __syncthreads();

    const uint8_t* kbase = reinterpret_cast<const uint8_t*>(a.k);
    const uint8_t* vbase = reinterpret_cast<const uint8_t*>(a.v);

    auto issue = [&](int tile) {
      if (tile < tiles) {
        uint8_t* st = smem + (tile % kGStages) * SM::kStageBytes;
#pragma unroll
        for (int it = 0; it < kGTileT * CH / 128; ++it) {
          const int idx = it * 128 + tid;
          const int r = idx / CH, c = idx % CH;
          const int cr = s_rows[tile * kGTileT + r];
          const size_t off = size_t(cr < 0 ? 0 : cr) * (D * 2) + c * 16;
          cp_async16_zfill(st + gswz<D>(r, c), kbase + off, cr >= 0);
          cp_async16_zfill(st + SM::kTileBytes + gswz<D>(r, c), vbase + off, cr >= 0);
        }
      }
      cp_async_commit();
    };

    // online-softmax state for heads h0 = 2*(lane%4), h1 = h0 + 1 (replicated across lanes
    // with equal lane%4); l is this lane's partial sum over its own tokens
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
    float o[KS][4];
#pragma unroll
    for (int m = 0; m < KS; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.0f;

    issue(0);
    issue(1);
    resolve(head, cnt);        // the rest of the table, while the first two tiles load
    for (int tile = 0; tile < tiles; ++tile) {
      cp_async_wait<1>();
      __syncthreads();
      issue(tile + 2);
      const uint8_t* st = smem + (tile % kGStages) * SM::kStageBytes;
      const uint32_t kst = smem_u32(st), vst = smem_u32(st + SM::kTileBytes);

      const int tl = tile * kGTileT + warp * 16 + (lane >> 2);
      const auto sw = [](int r, int c) { return gswz<D>(r, c); };
      attn_warp_tile<D, V_F16, AGG_F16>(KFragLdsm<decltype(sw)>{kst, warp, lane, sw}, vst, qb,
                                        s_rows[tl] >= 0, s_rows[tl + 8] >= 0, a.scale_log2, m0,
                                        m1, l0, l1, o, warp, lane, sw);
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---------------- merge the 4 warps' states, write this split's partial
#pragma unroll
    for (int o2 = 4; o2 < 32; o2 <<= 1) {
      l0 += __shfl_xor_sync(kFull, l0, o2);
      l1 += __shfl_xor_sync(kFull, l1, o2);
    }
    float* s_m = reinterpret_cast<float*>(smem);          // [4][8]
    float* s_l = s_m + 32;                                // [4][8]
    float* s_o = s_l + 32;                                // [4][8][D]
    if (lane < 4) {
      s_m[warp * 8 + 2 * lane] = m0;
      s_m[warp * 8 + 2 * lane + 1] = m1;
      s_l[warp * 8 + 2 * lane] = l0;
      s_l[warp * 8 + 2 * lane + 1] = l1;
    }
    {
      const int h0 = 2 * (lane & 3);
#pragma unroll
      for (int m = 0; m < KS; ++m) {
        const int d0 = m * 16 + (lane >> 2);
        float* ow = s_o + warp * 8 * D;
        ow[h0 * D + d0] = o[m][0];
        ow[(h0 + 1) * D + d0] = o[m][1];
        ow[h0 * D + d0 + 8] = o[m][2];
        ow[(h0 + 1) * D + d0 + 8] = o[m][3];
      }
    }
    __syncthreads();
    for (int idx = tid; idx < a.G * D; idx += 128) {
      const int h = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w * 8 + h]);
      const float base = M == -INFINITY ? 0.0f : M;
      float lsum = 0.0f, osum = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float wt = ex2(s_m[w * 8 + h] - base);
        lsum += wt * s_l[w * 8 + h];
        osum += wt * s_o[(w * 8 + h) * D + d];
      }
      const size_t rq = size_t(b) * Hq + g * a.G + h;
      const size_t pidx = rq * a.gsplits + split;
      a.part_o[pidx * D + d] = osum;
      if (d == 0) {
        a.part_ml[pidx * 2] = M;
        a.part_ml[pidx * 2 + 1] = lsum;
      }
    }

    // ---------------- the last split of the row to finish merges all splits (LSE combine):
    // out[h][d] = sum_s 2^(m_s - M) o_s[d] / sum_s 2^(m_s - M) l_s; a row with no tokens -> 0
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const unsigned prev = atomicAdd(a.row_ctr + row, 1u);
      s_last = prev == unsigned(nsp - 1);
    }
    __syncthreads();
    if (s_last) gather_merge_row<D>(a, row, nsp, smem);
    __syncthreads();               // shared memory is reused by the CTA's next split
  }
}

// The last split of row `row` to finish merges all of the row's splits (LSE combine).
template <int D>
QS_DEV void gather_merge_row(const AttnParams& a, int row, int nsp, uint8_t* smem) {
  const int b = row / a.Hkv, g = row % a.Hkv, Hq = a.Hkv * a.G, tid = threadIdx.x;
  __threadfence();
  float* s_w = reinterpret_cast<float*>(smem);          // [G][splits] weights, then [G] 1/den
  const int ns = nsp, stride = a.gsplits;              // splits merged; partials per head
  for (int i = tid; i < a.G * ns; i += 128) {
    const int h = i / ns, sp = i % ns;
    const size_t pidx = (size_t(b) * Hq + g * a.G + h) * stride + sp;
    s_w[i] = __ldcg(a.part_ml + pidx * 2);
    s_w[a.G * ns + i] = __ldcg(a.part_ml + pidx * 2 + 1);
  }
  __syncthreads();
  if (tid < a.G) {
    const int h = tid;
    float M = -INFINITY;
    for (int sp = 0; sp < ns; ++sp)
      if (s_w[a.G * ns + h * ns + sp] > 0.0f) M = fmaxf(M, s_w[h * ns + sp]);
    float den = 0.0f;
    for (int sp = 0; sp < ns; ++sp) {
      const float l = s_w[a.G * ns + h * ns + sp];
      const float wt = l > 0.0f ? ex2(s_w[h * ns + sp] - M) : 0.0f;
      s_w[h * ns + sp] = wt;
      den += wt * l;
    }
    s_w[2 * a.G * ns + h] = den > 0.0f ? 1.0f / den : 0.0f;
  }
  __syncthreads();
  for (int idx = tid; idx < a.G * D; idx += 128) {
    const int h = idx / D, d = idx % D;
    const size_t rq = size_t(b) * Hq + g * a.G + h;
    float num = 0.0f;
    for (int sp = 0; sp < ns; ++sp) {
      const float wt = s_w[h * ns + sp];
      if (wt != 0.0f) num += wt * __ldcg(a.part_o + (rq * stride + sp) * D + d);
    }
    const float r = num * s_w[2 * a.G * ns + h];
    if (a.out_bf16)
      reinterpret_cast<uint16_t*>(a.out)[rq * D + d] = f32_to_bf16_rn(r);
    else
      reinterpret_cast<float*>(a.out)[rq * D + d] = r;
  }
  if (tid == 0) a.row_ctr[row] = 0u;
}

template <int D, bool VF, bool AF>
static cudaError_t launch_gather_t(const AttnParams& a, cudaStream_t s, bool pdl) {
  auto k = attn_gather_kernel<D, VF, AF>;
  const int smem = GatherSmem<D>::kTotal;
  const cudaError_t attr = set_smem_limit(k, smem);
  if (attr != cudaSuccess) return attr;
  // splits per row in the grid: all of the plan's when the grid fits in one wave of
  // resident CTAs (2 per SM), else as many as one wave gives each row (>= 1)
  int gx = a.gsplits;
  if ((long long)a.gsplits * a.rows > 2LL * num_sms())
    gx = max(1, min(a.gsplits, 2 * num_sms() / a.rows));
  return launch_k(k, dim3(gx, a.rows), dim3(128), smem, s, pdl, a);
}

cudaError_t launch_attn_gather(const Plan& p, const AttnParams& a, cudaStream_t s, bool pdl) {
  const bool vf = p.v_dtype == QS_F16, af = p.v_agg_dtype == QS_F16;
  if (p.d == 128) {
    if (vf) return launch_gather_t<128, true, true>(a, s, pdl);
    if (af) return launch_gather_t<128, false, true>(a, s, pdl);
    return launch_gather_t<128, false, false>(a, s, pdl);
  }
  if (p.d == 64) {
    if (vf) return launch_gather_t<64, true, true>(a, s, pdl);
    if (af) return launch_gather_t<64, false, true>(a, s, pdl);
    return launch_gather_t<64, false, false>(a, s, pdl);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qs
