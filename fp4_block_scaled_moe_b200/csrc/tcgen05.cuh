// sm_100a tensor-core primitives: TMEM allocation, shared-memory matrix descriptors,
// block-scaled tcgen05.mma (kind::mxf8f6f4), 16-bit tcgen05.mma (kind::f16), scale-factor
// copies into TMEM, and TMEM loads.  Inline PTX only; the descriptor bit layouts follow the PTX ISA for sm_100
// (the same fields CUTLASS's UMMA descriptors describe).
#pragma once

#include "common.cuh"

namespace fp4 {
namespace tc {

// ---- TMEM allocation (one full warp executes these) --------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- shared-memory matrix descriptors ----------------------------------------------
// K-major operand in 128-byte swizzled rows (8 rows = one 1024-byte swizzle atom):
// start address >> 4, leading offset 1 (unused for swizzled K-major), stride between
// 8-row groups 1024 bytes, descriptor version 1, layout SWIZZLE_128B (2).
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;                 // leading byte offset (16 B units)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;         // stride byte offset (16 B units)
  d |= static_cast<uint64_t>(1u) << 46;                 // version
  d |= static_cast<uint64_t>(2u) << 61;                 // SWIZZLE_128B
  return d;
}
// Plain (no swizzle) K-major core matrices of 8 rows x 16 bytes stacked contiguously:
// used as the source of the 32x128b scale-factor copy.
__device__ __forceinline__ uint64_t desc_k_interleave(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;                 // leading byte offset: unused (one 16 B column)
  d |= static_cast<uint64_t>(128u >> 4) << 32;          // 8-row groups are 128 bytes apart
  d |= static_cast<uint64_t>(1u) << 46;
  return d;                                             // layout type 0 = no swizzle
}

// ---- instruction descriptor: kind::mxf8f6f4 with UE8M0 block scales ----------------
// a/b format: 0 = E4M3, 5 = E2M1; both K-major; M = 128; N multiple of 8 in [8, 256].
__host__ __device__ __forceinline__ uint32_t idesc_mxf8f6f4(uint32_t a_fmt, uint32_t b_fmt, uint32_t M,
                                                            uint32_t N) {
  uint32_t d = 0;
  d |= a_fmt << 7;
  d |= b_fmt << 10;
  d |= (N >> 3) << 17;
  d |= 1u << 23;          // scale format UE8M0
  d |= (M >> 4) << 24;
  return d;
}

// D[tmem] (+)= A[smem] x B[smem]^T with per-32-element scales read from TMEM.
// sf_id (0..3) selects the byte of the 32-bit TMEM scale word (the K block).
__device__ __forceinline__ void mma_mxf8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t sf_id,
                                             uint32_t accumulate) {
  const uint32_t id = idesc | (sf_id << 29) | (sf_id << 4);
  const uint32_t sfa = sfa_tmem | (sf_id << 30), sfb = sfb_tmem | (sf_id << 30);
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(id), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// ---- instruction descriptor: kind::f16 -----------------------------------------------
// D float32; A and B both f16 (ab_fmt 0) or both bf16 (1), both K-major; M = 128, N a
// multiple of 16 in [16, 256].
__host__ __device__ __forceinline__ uint32_t idesc_f16(uint32_t M, uint32_t N, uint32_t ab_fmt = 0u) {
  uint32_t d = 0;
  d |= 1u << 4;           // D format F32
  d |= ab_fmt << 7;       // A format
  d |= ab_fmt << 10;      // B format
  d |= (N >> 3) << 17;
  d |= (M >> 4) << 24;
  return d;
}

// D[tmem] (+)= A[smem] x B[smem]^T, K = 16 (16-bit operands).
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation issued so far by this thread is done.
__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Copy a 128-row x 4-byte scale block, stored as 32 rows of 16 bytes (row m0 holds
// rows m0, m0+32, m0+64, m0+96, 4 bytes each), into 4 TMEM columns: lane m0 + 32q of
// column c gets the 4 K-block scales of row m0 + 32c (replicated over the quadrants q).
__device__ __forceinline__ void cp_sf_32x128b_x4(uint32_t tmem_col, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem_col), "l"(src_desc) : "memory");
}

// Each thread of a warp loads 16 consecutive 32-bit columns of its TMEM lane.
__device__ __forceinline__ void ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

}  // namespace tc
}  // namespace fp4
