// umma.cuh -- inline-PTX wrappers for the 5th-generation tensor cores of
// sm_100a (tcgen05): tensor-memory allocation, shared-memory operand
// descriptors, the block-scaled MMA with e2m1 operands on both sides
// (kind::mxf4, one e8m0 scale per 32 K elements on each side, K = 64 per
// instruction), the bf16 MMA (kind::f16, K = 16), scale copies into tensor
// memory, commit to an mbarrier and loads of the fp32 accumulator.
//
// Layouts used here (all K-major, no swizzle):
//   - an operand is a grid of "core matrices", each 8 rows x 16 bytes stored
//     as 128 contiguous bytes (row r at byte 16 r); the descriptor gives the
//     byte distance between core matrices adjacent along K (leading, LBO)
//     and along M/N (stride, SBO);
//   - e2m1 operands are packed: 16 bytes of a core-matrix row hold 32
//     elements, element 2t in the low nibble of byte t; bf16 operands hold
//     8 elements a core-matrix row;
//   - scale factors: one byte per (row, 32-wide K block); four K blocks of
//     128 rows form a 512-byte unit, byte (m % 32) * 16 + (m / 32) * 4 + kb,
//     which one copy broadcasts into tensor-memory lanes 0-127, 4 columns:
//     lane 32 q + r, column j holds the scales of row r + 32 j, byte kb
//     selecting the K block.  An MMA of K = 64 takes the two bytes starting
//     at its scale id (0 or 2).
#pragma once
#include <cstdint>

namespace moe {
namespace umma {

// ---- tensor memory ----------------------------------------------------------
// One warp allocates `cols` columns (a power of two, 32..512) and writes the
// base address to *dst_smem; then gives up the right to allocate more.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem))),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
               : "memory");
}
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- shared-memory matrix descriptor (K-major, no swizzle) --------------------
// bits 0-13 start address >> 4, 16-29 leading byte offset >> 4, 32-45 stride
// byte offset >> 4, 46-47 version (1), 49-51 base offset (0), 52 leading
// offset mode (0), 61-63 layout (0: no swizzle).
__device__ __forceinline__ uint64_t smem_desc(const void* smem, uint32_t lbo, uint32_t sbo) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  uint64_t d = 0;
  d |= (uint64_t)((a >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// ---- instruction descriptor, kind::mxf4 block-scaled ---------------------------
// bits 4-5 B scale id, 7-9 A format (1: e2m1), 10-12 B format (1: e2m1),
// 15/16 A/B major (0: K), 17-22 N >> 3, 23 scale format (1: e8m0),
// 24-28 M >> 4, 29-30 A scale id, 31 K size (0: K = 64).
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, int a_sf_id, int b_sf_id) {
  return (uint32_t)(b_sf_id & 3) << 4 | 1u << 7 | 1u << 10 | (uint32_t)(N >> 3) << 17 | 1u << 23 |
         (uint32_t)(M >> 4) << 24 | (uint32_t)(a_sf_id & 3) << 29;
}

// D[tmem] (+)= A . B^T, K = 64, with per-32 scales from tensor memory;
// issued by one thread.
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate), "r"(sfa_tmem),
      "r"(sfb_tmem)
      : "memory");
}

// ---- instruction descriptor, kind::f16 with bf16 operands ----------------------
// bits 4-5 D format (1: f32), 7-9 A format (1: bf16), 10-12 B format (1: bf16),
// 15/16 A/B major (0: K), 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return 1u << 4 | 1u << 7 | 1u << 10 | (uint32_t)(N >> 3) << 17 | (uint32_t)(M >> 4) << 24;
}

// D[tmem] (+)= A . B^T, bf16 operands, K = 16; issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem), "l"(a_desc),
      "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// 32 rows x 16 bytes of scales (one 512-byte unit) from shared memory into
// tensor memory, broadcast to the four lane quarters; one thread issues it.
__device__ __forceinline__ void cp_scales(uint32_t taddr, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc)
               : "memory");
}

// The MMAs and copies this thread issued arrive on the mbarrier when done.
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(bar)))
               : "memory");
}

// A warp reads 8 consecutive fp32 columns of its 32 lanes (lane quarter
// warp % 4): lane i gets row 32 (warp % 4) + i.
__device__ __forceinline__ void ld_32x32b_x8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// generic-proxy shared-memory writes made visible to the tensor core
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace umma
}  // namespace moe
