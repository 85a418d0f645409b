// 5th-generation tensor-core helpers (tcgen05, sm_100a): shared-memory matrix and instruction
// descriptors, MMA issue with accumulators in tensor memory, commits, tensor-memory loads, stores,
// allocation. Used by the MLA decode kernel (kind::f16) and the LM decode kernel (kind::i8).
//
// Formats follow the PTX ISA's definitions for tcgen05:
//  * shared-memory descriptor, no swizzle: start address >> 4 (bits 0-13), leading-dimension byte
//    offset >> 4 (16-29), stride-dimension byte offset >> 4 (32-45), descriptor version 1 (bit 46).
//    Operands are "core matrices" of 8 rows x 16 bytes (128 contiguous bytes, row r at 16 r); for
//    a K-major operand the leading offset steps between core matrices along K and the stride offset
//    between 8-row groups.
//  * instruction descriptor (kind::f16 / kind::i8): D format (bits 4-5: 1 = f32, 2 = s32), A and
//    B formats (bits 7-9, 10-12: kind::f16 0 = f16, 1 = bf16; kind::i8 0 = u8, 1 = s8), A and B
//    major (bits 15, 16: 1 = MN-major), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
//  * tensor-memory address: lane in bits 16-31, column in bits 0-15. Warp w of a CTA reaches lanes
//    32 (w % 4) .. 32 (w % 4) + 31. An M = 128 accumulator keeps row i in lane i; an A operand in
//    tensor memory likewise keeps row i in lane i with its K elements packed along the columns
//    (four 8-bit elements per 32-bit column).
#pragma once

#include <cstdint>

namespace kvq {
namespace tc {

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for tcgen05
  return d;
}

// kind::f16 with f32 accumulation. fmt: 0 = f16, 1 = bf16 (A and B alike); a_mn / b_mn: MN-major.
__host__ __device__ constexpr uint32_t idesc_f16(int fmt, int a_mn, int b_mn, int M, int N) {
  return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((uint32_t)a_mn << 15) |
         ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// kind::i8 with s32 accumulation, K-major A and B. a_signed / b_signed: 1 = s8, 0 = u8.
__host__ __device__ constexpr uint32_t idesc_i8(int a_signed, int b_signed, int M, int N) {
  return (2u << 4) | ((uint32_t)a_signed << 7) | ((uint32_t)b_signed << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// D (tensor memory) = or += A (shared memory) . B (shared memory), kind::f16.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// D (tensor memory) = or += A (tensor memory) . B (shared memory), kind::i8.
__device__ __forceinline__ void umma_i8_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrives once on the mbarrier when every MMA this thread issued before has completed.
__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

#define KVQ_R4(r, i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3])
#define KVQ_W4(r, i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3])

// 32 lanes x 32 bit, N consecutive columns: thread l of the warp gets lane (base lane + l).
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n" : KVQ_R4(r, 0) : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : KVQ_R4(r, 0), KVQ_R4(r, 4) : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : KVQ_R4(r, 0), KVQ_R4(r, 4), KVQ_R4(r, 8), KVQ_R4(r, 12) : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : KVQ_R4(r, 0), KVQ_R4(r, 4), KVQ_R4(r, 8), KVQ_R4(r, 12), KVQ_R4(r, 16), KVQ_R4(r, 20), KVQ_R4(r, 24),
        KVQ_R4(r, 28)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr), KVQ_W4(r, 0),
               KVQ_W4(r, 4) : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      ::"r"(taddr), KVQ_W4(r, 0), KVQ_W4(r, 4), KVQ_W4(r, 8), KVQ_W4(r, 12), KVQ_W4(r, 16), KVQ_W4(r, 20),
        KVQ_W4(r, 24), KVQ_W4(r, 28) : "memory");
}
#undef KVQ_R4
#undef KVQ_W4

// Allocation by one whole warp; the base address lands in shared memory at dst_smem.
__device__ __forceinline__ void alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}

}  // namespace tc
}  // namespace kvq
