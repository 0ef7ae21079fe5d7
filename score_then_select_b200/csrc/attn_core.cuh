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
  // c += K Q^T over k-step ks (BF16 keys and queries)
  QS_DEV void qk(float (&c)[4], int ks, const uint32_t (&qb)[2]) const {
    uint32_t a0, a1, a2, a3;
    ldsm_x4(a0, a1, a2, a3, kst + swz(warp * 16 + (lane & 15), ks * 2 + (lane >> 4)));
    mma_bf16(c, a0, a1, a2, a3, qb[0], qb[1]);
  }
  QS_DEV void fix(float (&)[4]) const {}     // the accumulator is the logit
};

// K fragments of one 64-token tile of NVFP4 keys in shared memory (the storage variant of
// "Jet-QSparse ...", Full text). The attended key is the dequantised, un-centred value
// k = g_k (e sigma) + mu. The A operand is e * sigma, exact in FP16 (an E2M1 value has at
// most 2 significant bits and a UE4M3 scale 4; the product lies in [2^-10, 2688]), made by
// one conversion of two codes and one f16x2 multiply; the B operand is the query in FP16,
// scaled by 2^-qexp (qexp > 0 only for queries beyond FP16's range), so the products are
// exact and the MMA sums them in float32. The logit is then
// q . k = 2^qexp g_k (q' . (e sigma)) + q . mu, formed in `fix`.
//   codes:  [4 chunks][64 tokens][16 bytes]; chunk c holds elements 32c..32c+31 of a
//           token, element 2i + u in nibble u of byte i;
//   scales: the page's 1,024 bytes; token slot m's scale of elements 16j..16j+15 at
//           (j / 4) * 512 + 16 * (m % 32) + 4 * (m / 32) + j % 4; m0 = the page slot of
//           the tile's first token.
// This lane's rows are tokens r0 = 16 warp + lane / 4 and r0 + 8 of the tile, its elements
// 2t, 2t + 1, 2t + 8, 2t + 9 of each k-step (t = lane % 4), as the mma A fragment holds them.
template <int KS>
struct KFragNvfp4 {
  const uint8_t* codes;
  const uint32_t (&qh)[KS][2];  // FP16 query fragments (B operand), scaled by 2^-qexp
  float gks, qmu0, qmu1;        // 2^qexp g_k; q . mu of this lane's heads 2t and 2t + 1
  int r0, t;
  uint32_t sg[2][KS];           // sigma of each k-step of rows r0, r0 + 8, as f16 pairs

  QS_DEV KFragNvfp4(const uint8_t* codes_, const uint8_t* scales, const uint32_t (&qh_)[KS][2],
                    float gks_, float qmu0_, float qmu1_, int m0, int warp, int lane)
      : codes(codes_), qh(qh_), gks(gks_), qmu0(qmu0_), qmu1(qmu1_), r0(warp * 16 + (lane >> 2)),
        t(lane & 3) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int m = m0 + r0 + 8 * r;
#pragma unroll
      for (int h = 0; h < KS / 4; ++h) {
        const uint32_t w =
            *reinterpret_cast<const uint32_t*>(scales + h * 512 + 16 * (m & 31) + 4 * (m >> 5));
        const uint32_t lo = e4m3x2_to_f16x2(w), hi = e4m3x2_to_f16x2(w >> 16);
        sg[r][4 * h + 0] = __byte_perm(lo, 0u, 0x1010);      // low half in both halves
        sg[r][4 * h + 1] = __byte_perm(lo, 0u, 0x3232);      // high half in both halves
        sg[r][4 * h + 2] = __byte_perm(hi, 0u, 0x1010);
        sg[r][4 * h + 3] = __byte_perm(hi, 0u, 0x3232);
      }
    }
  }
  // byte t of w (two codes) times sigma: f16x2, exact
  QS_DEV uint32_t dec(uint32_t w, uint32_t s2) const {
    const uint32_t e = e2m1x2_to_f16x2(w >> (8 * t));
    uint32_t p;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p) : "r"(e), "r"(s2));
    return p;
  }
  // c += K Q^T over k-step ks (FP16 e * sigma and queries)
  QS_DEV void qk(float (&c)[4], int ks, const uint32_t (&)[2]) const {
    const int cc = ks >> 1, h = ks & 1;
    const uint2 w0 = *reinterpret_cast<const uint2*>(codes + cc * 1024 + r0 * 16 + 8 * h);
    const uint2 w1 = *reinterpret_cast<const uint2*>(codes + cc * 1024 + (r0 + 8) * 16 + 8 * h);
    mma_f16(c, dec(w0.x, sg[0][ks]), dec(w1.x, sg[1][ks]), dec(w0.y, sg[0][ks]),
            dec(w1.y, sg[1][ks]), qh[ks][0], qh[ks][1]);
  }
  // accumulator (tokens r0 / r0 + 8 x heads 2t, 2t + 1) -> logits q . k
  QS_DEV void fix(float (&c)[4]) const {
    c[0] = fmaf(c[0], gks, qmu0);
    c[1] = fmaf(c[1], gks, qmu1);
    c[2] = fmaf(c[2], gks, qmu0);
    c[3] = fmaf(c[3], gks, qmu1);
  }
};

// kf.qk(c, ks, qb): c += K Q^T over k-step ks; kf.fix(c): accumulator -> logits. qb: the query fragments (B
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
  for (int ks = 0; ks < KS; ++ks) kf.qk(c, ks, qb[ks]);
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
