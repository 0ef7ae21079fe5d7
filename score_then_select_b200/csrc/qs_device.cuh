// qs_device.cuh - device helpers shared by the libqs kernels (sm_100a only).
//
// Thin wrappers over PTX: mbarriers with bounded waits, the bulk (TMA) global->shared
// copy, 16-byte cp.async, ldmatrix / movmatrix, the m16n8k16 tensor-core MMA, ex2, and
// the workspace status word.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "qs_internal.h"

#define QS_DEV __device__ __forceinline__

namespace qs {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start before the kernel
// ahead of it in the stream has finished; pdl_wait() blocks until that kernel has
// completed and its memory is visible (a no-op for a normal launch). pdl_trigger() lets
// the next kernel in the stream begin launching early.
QS_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
QS_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- status word
// ws header (uint32 words): [0] first error code, [1] kernel id, [2] index, [16..] counters.
QS_DEV void flag_error(uint32_t* hdr, uint32_t code, uint32_t kernel, uint32_t info) {
  if (atomicCAS(hdr, 0u, code) == 0u) {
    atomicExch(hdr + 1, kernel);
    atomicExch(hdr + 2, info);
  }
}

// ---------------------------------------------------------------- number formats
QS_DEV float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
QS_DEV float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }
QS_DEV float bf16_to_f32(uint16_t x) { return __uint_as_float(uint32_t(x) << 16); }
QS_DEV uint16_t f32_to_bf16_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// ---------------------------------------------------------------- shared-memory addresses
QS_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
QS_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
QS_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
QS_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
QS_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
QS_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false after `limit` unsuccessful polls (each poll may suspend the
// thread for a hardware-defined interval), so a lost arrival cannot hang the GPU.
QS_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = 1u << 22) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// ---------------------------------------------------------------- bulk copy (TMA unit)
// Contiguous global -> shared copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned) that signals completion on `bar` through its transaction count.
QS_DEV void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst_smem)), "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 2-D tiled tensor copy (TMA unit) of one box at element coordinates (x, y) of the tensor
// map, signalling completion on `bar` through its transaction count. x * element size
// must be a multiple of 16 bytes; y may lie outside the tensor (out-of-range rows are
// filled with zeros). No cluster multicast.
QS_DEV void tma_load_2d(void* dst_smem, const void* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst_smem)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y),
        "r"(smem_u32(bar))
      : "memory");
}
// Arrive on `bar` once every cp.async this thread issued before has landed; the arrival
// is not added to the pending count (the barrier's expected count includes it).
QS_DEV void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- cp.async (16 bytes)
// 16-byte copy into shared memory; `valid` false writes zeros (source size 0)
QS_DEV void cp_async16_zfill(void* dst_smem, const void* src_gmem, bool valid) {
  // src-size 0 writes 16 zero bytes without reading global memory
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst_smem)),
               "l"(src_gmem), "r"(valid ? 16 : 0)
               : "memory");
}
QS_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
QS_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- ldmatrix / movmatrix
QS_DEV void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
QS_DEV void ldsm_x4_t(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// Transpose of an 8x8 matrix of 16-bit elements held one row pair per lane.
QS_DEV uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// ---------------------------------------------------------------- tensor-core MMA
QS_DEV void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                     uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
QS_DEV void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                    uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// pack two floats into bf16x2 / f16x2 (low half = first argument), round to nearest even
QS_DEV uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
QS_DEV uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two FP8 E4M3 codes (byte 0 -> low half, byte 1 -> high half) -> f16x2; exact (every
// E4M3 value is an FP16 value). Used to decode the FP8 projected-key cache.
QS_DEV uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(uint16_t(two_codes)));
  return r;
}
// UE4M3 (bias 7, 3 mantissa bits, subnormal step 2^-9, largest finite 448 = 0x7E):
// nearest even, saturating; non-positive and NaN inputs give code 0.
QS_DEV uint32_t ue4m3_encode(float sf) {
  if (!(sf > 0.0f)) return 0u;
  if (sf >= 448.0f) return 0x7Eu;
  const uint32_t u = __float_as_uint(sf);
  const int e = int(u >> 23) - 127;
  if (e < -6) return __float2uint_rn(sf * 512.0f);  // subnormal range: m * 2^-9, m <= 8
  const uint32_t mant = u & 0x7FFFFFu;
  uint32_t code = (uint32_t(e + 7) << 3) | (mant >> 20);
  const uint32_t rem = mant & 0xFFFFFu;
  if (rem > 0x80000u || (rem == 0x80000u && (code & 1u))) code += 1u;
  return code > 0x7Eu ? 0x7Eu : code;
}
// Signed E4M3 (the FP8 projected-key cache): the magnitude as UE4M3 above, bit 7 the sign
// (kept for negative values that round to zero, and for -0).
QS_DEV uint32_t e4m3_encode(float x) {
  return ue4m3_encode(fabsf(x)) | (signbit(x) ? 0x80u : 0u);
}
// two E2M1 codes (low byte of v: the low nibble is the first element) -> f16x2, exact
QS_DEV uint32_t e2m1x2_to_f16x2(uint32_t v) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
      : "=r"(r) : "r"(v));
  return r;
}
QS_DEV float f16_lo(uint32_t x) { return __half2float(__ushort_as_half(uint16_t(x))); }
QS_DEV float f16_hi(uint32_t x) { return __half2float(__ushort_as_half(uint16_t(x >> 16))); }
// bf16x2 -> f16x2 (for FP16 value aggregation of BF16-stored values)
QS_DEV uint32_t bf16x2_to_f16x2(uint32_t x) { return pack_f16x2(bf16_lo(x), bf16_hi(x)); }

// 2^x (hardware approximation; inputs <= 0 in the softmax, -inf -> 0)
QS_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- tcgen05 (5th-gen tensor cores)
// Tensor memory (TMEM) is allocated in columns by one full warp; addresses are
// (lane << 16) | column. A warp may read only lanes 32*(warp%4) .. +31.
QS_DEV void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(smem_dst)), "r"(ncols) : "memory");
}
QS_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
QS_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
QS_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
QS_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major, no swizzle: 8-row x 16-byte core matrices,
// `lbo` bytes between the core matrices along K, `sbo` bytes between 8-row groups.
QS_DEV uint64_t smem_desc_kmajor(const void* p, uint32_t lbo, uint32_t sbo) {
  const uint64_t start = (smem_u32(p) >> 4) & 0x3FFFu;
  return start | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) | (uint64_t((sbo >> 4) & 0x3FFFu) << 32) |
         (uint64_t(1) << 46);  // descriptor version 1; base offset 0; layout: no swizzle
}

// Copy one 32-row x 16-byte block from shared memory to TMEM columns [taddr, taddr+4),
// replicated to each of the four 32-lane groups.
QS_DEV void tc_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D[tmem] (+)= A(smem, FP4 E2M1) x B(smem, FP4 E2M1)^T with per-16-element UE4M3 scales of A
// and B read from TMEM; M = 128, K = 64 per instruction.
QS_DEV void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                        uint32_t sfa_tmem, uint32_t sfb_tmem, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}\n"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(uint32_t(accumulate)),
        "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
QS_DEV void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// This warp's 32 lanes x 8 consecutive 32-bit columns.
QS_DEV void tc_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  // the load and its completion wait sit in one asm block, so no use of r can be moved
  // between them
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
}

// ---------------------------------------------------------------- warp reductions
QS_DEV float warp_max(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
  return v;
}
QS_DEV float warp_min(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fminf(v, __shfl_xor_sync(kFull, v, m));
  return v;
}


}  // namespace qs
