// attn_core.cuh - one warp's share of one 64-token tile of sparse attention: 16 tokens'
// tensor-core logits, online softmax and value aggregation. Shared by the two attention
// kernels (attn.cu, attn_gather.cu), which differ in how tiles reach shared memory.
//
// Tensor-core mapping (mma.m16n8k16, FP32 accumulate), transposed so that the group's
// <= 8 query heads fill the N = 8 side:
//   S^T[16 tok x 8 heads]  = K[16 tok x d] . Q^T[d x 8 heads]      (A = K via ldmatrix)
//   O^T[d x 8 heads]      += V^T[d x 16 tok] . P^T[16 tok x 8 heads] (A = V via ldmatrix.trans,
//                                                                    B = P via movmatrix)
// Lane layout: this lane's heads are h0 = 2 * (lane % 4) and h0 + 1, its tokens
// lane / 4 and lane / 4 + 8 of the warp's 16; m (running max, base 2) is replicated over
// the lanes with equal lane % 4, l is this lane's partial sum over its own tokens, and
// o[m] holds O^T entries (d0, h0), (d0, h0 + 1), (d0 + 8, h0), (d0 + 8, h0 + 1) with
// d0 = 16 m + lane / 4.
#pragma once

#include "qs_device.cuh"

namespace qs {

// K fragments (A operand of S^T) of k-step ks for this warp's 16 tokens, read from a BF16
// tile in shared memory by ldmatrix: `swz(r, c)` is the byte offset of 16-byte chunk c of
// token row r inside the tile.
template <typename Swz>
struct KFragLdsm {
  uint32_t kst;
  int warp, lane;
  Swz swz;
  QS_DEV void operator()(int ks, uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) const {
    ldsm_x4(a0, a1, a2, a3, kst + swz(warp * 16 + (lane & 15), ks * 2 + (lane >> 4)));
  }
  QS_DEV void fix(float (&)[4]) const {}     // the accumulator is the logit
};

// K fragments of one 64-token tile of NVFP4 keys in shared memory (the storage variant of
// "Jet-QSparse ...", Full text). The attended key is the dequantised, un-centred value
// k = g_k (e sigma) + mu. The A operand is e * sigma, which is exact in BF16 (an E2M1 value
// has at most 2 significant bits and a UE4M3 scale 4); the products with the BF16 query
// are then exact and the MMA sums them in float32, so the logit q . k is
// g_k (q . (e sigma)) + q . mu, formed in `fix` from the accumulator and the head's q . mu.
//   codes:  [4 chunks][64 tokens][16 bytes]; chunk c holds elements 32c..32c+31 of a
//           token, element 2i + u in nibble u of byte i;
//   scales: the page's 1,024 bytes; token slot m's scale of elements 16j..16j+15 at
//           (j / 4) * 512 + 16 * (m % 32) + 4 * (m / 32) + j % 4; m0 = the page slot of
//           the tile's first token.
// This lane's rows are tokens r0 = 16 warp + lane / 4 and r0 + 8 of the tile, its elements
// 2t, 2t + 1, 2t + 8, 2t + 9 of each k-step (t = lane % 4), as the mma A fragment holds them.
struct KFragNvfp4 {
  const uint8_t* codes;
  float gk, qmu0, qmu1;    // g_k; q . mu of this lane's heads 2t and 2t + 1
  int r0, t;
  uint32_t sc[2][2];       // scale words: [row r0, r0 + 8][elements 0-63, 64-127]

  QS_DEV KFragNvfp4(const uint8_t* codes_, const uint8_t* scales, float gk_, float qmu0_,
                    float qmu1_, int m0, int warp, int lane)
      : codes(codes_), gk(gk_), qmu0(qmu0_), qmu1(qmu1_), r0(warp * 16 + (lane >> 2)), t(lane & 3) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int m = m0 + r0 + 8 * r;
#pragma unroll
      for (int h = 0; h < 2; ++h)
        sc[r][h] = *reinterpret_cast<const uint32_t*>(scales + h * 512 + 16 * (m & 31) + 4 * (m >> 5));
    }
  }
  // sigma of k-step ks of row r as an f16 pair (both halves)
  QS_DEV uint32_t sig2(int r, int ks) const {
    const uint32_t f = e4m3x2_to_f16x2(sc[r][ks >> 2] >> (8 * (ks & 3))) & 0xffffu;
    return f | (f << 16);
  }
  // byte t of w (two codes) times sigma -> bf16x2, exact
  QS_DEV uint32_t dec(uint32_t w, uint32_t s2) const {
    const uint32_t e = e2m1x2_to_f16x2(w >> (8 * t));
    uint32_t p;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p) : "r"(e), "r"(s2));
    return __byte_perm(__float_as_uint(f16_lo(p)), __float_as_uint(f16_hi(p)), 0x7632);
  }
  QS_DEV void operator()(int ks, uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) const {
    const int c = ks >> 1, h = ks & 1;
    const uint2 w0 = *reinterpret_cast<const uint2*>(codes + c * 1024 + r0 * 16 + 8 * h);
    const uint2 w1 = *reinterpret_cast<const uint2*>(codes + c * 1024 + (r0 + 8) * 16 + 8 * h);
    const uint32_t s0 = sig2(0, ks), s1 = sig2(1, ks);
    a0 = dec(w0.x, s0);
    a1 = dec(w1.x, s1);
    a2 = dec(w0.y, s0);
    a3 = dec(w1.y, s1);
  }
  // accumulator (tokens r0 / r0 + 8 x heads 2t, 2t + 1) -> logits q . k
  QS_DEV void fix(float (&c)[4]) const {
    c[0] = fmaf(c[0], gk, qmu0);
    c[1] = fmaf(c[1], gk, qmu1);
    c[2] = fmaf(c[2], gk, qmu0);
    c[3] = fmaf(c[3], gk, qmu1);
  }
};

// kf(ks, a0..a3): the K fragments of k-step ks (see KFragLdsm). qb: the query fragments (B
// operand of S^T), valid0 / valid1: whether this lane's two tokens are selected (masked
// ones get probability 0), scale_log2: softmax scale * log2 e; `swz` addresses the V tile.
template <int D, bool V_F16, bool AGG_F16, typename KF, typename Swz>
QS_DEV void attn_warp_tile(const KF& kf, uint32_t vst, const uint32_t (&qb)[D / 16][2],
                           bool valid0, bool valid1, float scale_log2, float& m0, float& m1,
                           float& l0, float& l1, float (&o)[D / 16][4], int warp, int lane,
                           Swz swz) {
  constexpr int KS = D / 16;
  // S^T = K Q^T for this warp's 16 tokens
  float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    uint32_t a0, a1, a2, a3;
    kf(ks, a0, a1, a2, a3);
    mma_bf16(c, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
  }
  kf.fix(c);
  const float x0 = valid0 ? c[0] * scale_log2 : -INFINITY;
  const float x1 = valid0 ? c[1] * scale_log2 : -INFINITY;
  const float x2 = valid1 ? c[2] * scale_log2 : -INFINITY;
  const float x3 = valid1 ? c[3] * scale_log2 : -INFINITY;
  float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
  for (int o2 = 4; o2 < 32; o2 <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o2));
  }
  const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
  const float base0 = mn0 == -INFINITY ? 0.0f : mn0;
  const float base1 = mn1 == -INFINITY ? 0.0f : mn1;
  const float al0 = ex2(m0 - base0), al1 = ex2(m1 - base1);
  m0 = mn0;
  m1 = mn1;
  const float p0 = ex2(x0 - base0), p1 = ex2(x1 - base1);
  const float p2 = ex2(x2 - base0), p3 = ex2(x3 - base1);
  l0 = l0 * al0 + p0 + p2;
  l1 = l1 * al1 + p1 + p3;
#pragma unroll
  for (int m = 0; m < KS; ++m) {
    o[m][0] *= al0;
    o[m][1] *= al1;
    o[m][2] *= al0;
    o[m][3] *= al1;
  }
  // P^T as the B operand: transpose the two 8x8 (token x head) quadrants
  uint32_t pb0, pb1;
  if constexpr (AGG_F16) {
    pb0 = movmatrix_t(pack_f16x2(p0, p1));
    pb1 = movmatrix_t(pack_f16x2(p2, p3));
  } else {
    pb0 = movmatrix_t(pack_bf16x2(p0, p1));
    pb1 = movmatrix_t(pack_bf16x2(p2, p3));
  }
  // O^T += V^T P^T over the head dimension
#pragma unroll
  for (int m = 0; m < KS; ++m) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4_t(a0, a1, a2, a3,
              vst + swz(warp * 16 + (lane & 7) + ((lane >> 4) << 3), m * 2 + ((lane >> 3) & 1)));
    if constexpr (AGG_F16) {
      if constexpr (!V_F16) {
        a0 = bf16x2_to_f16x2(a0);
        a1 = bf16x2_to_f16x2(a1);
        a2 = bf16x2_to_f16x2(a2);
        a3 = bf16x2_to_f16x2(a3);
      }
      mma_f16(o[m], a0, a1, a2, a3, pb0, pb1);
    } else {
      mma_bf16(o[m], a0, a1, a2, a3, pb0, pb1);
    }
  }
}

}  // namespace qs
