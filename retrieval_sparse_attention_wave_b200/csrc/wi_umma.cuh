// Fifth-generation tensor-core primitives (tcgen05, sm_100a): tensor-memory
// allocation, the single-thread MMA from shared-memory descriptors with its
// completion on an mbarrier, and the warp's tensor-memory loads.
//
// Operand layout used throughout: K-major tiles of 128-byte rows with the
// 128-byte swizzle (16-byte chunk c of row r at r * 128 + ((c ^ (r % 8)) * 16),
// eight-row groups 1024 bytes apart, a tile 1024-byte aligned); a K extent
// of 64 bf16 per 128-byte row block, further K blocks rows * 128 bytes on.
#pragma once
#include <cstdint>

#include "wi_common.cuh"

namespace wi {

// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled operand
// starting at shared address `saddr`: start address >> 4 in bits 0..13, the
// leading byte offset (unused by this layout; 16 bytes) in bits 16..29, the
// 1024-byte stride between eight-row groups in bits 32..45, descriptor
// version 1 in bits 46..47, base offset 0, swizzle mode 2 (128 bytes) in
// bits 61..63.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of a dense bf16 x bf16 -> fp32 MMA of M x N, both
// operands K-major: accumulator format 1 (fp32) in bits 4..5, A and B format
// 1 (bf16) in bits 7..9 and 10..12, N / 8 in bits 17..22, M / 16 in bits
// 24..28.
template <int M, int N>
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32() {
  static_assert(M == 64 || M == 128, "M is 64 or 128 on one CTA");
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N is a multiple of 16 in 16..256");
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A * B^T; issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// The barrier receives one arrival once every MMA this thread issued before
// has completed (their shared-memory operands are free, their results in
// tensor memory).
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

// Tensor-memory allocation of `ncols` columns (a power of two, 32..512) by
// one whole warp; the base address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of the calling thread's tensor-memory lane
// (warp w of a warpgroup reads lanes 32 (w % 4) .. 32 (w % 4) + 31; `taddr`
// carries the warp's first lane in bits 16..31 and the first column in bits
// 0..15), and the wait for the load in the same statement (the registers
// are valid only after it).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace wi
