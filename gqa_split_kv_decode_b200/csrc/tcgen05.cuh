// Fifth-generation tensor-core (tcgen05) building blocks for sm_100a: tensor
// memory (TMEM) allocation, shared-memory matrix descriptors, the
// single-thread MMA issue, its completion signal, and the warp-wide TMEM
// loads and stores.  Encodings follow the public sm_100 descriptor formats
// (the same bit layout CUTLASS's cute::UMMA descriptors use).
#pragma once

#include <stdint.h>

namespace gqa {

// ------------------------------------------------------------ descriptors

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32
// accumulator, M x N tile.  `b_mn_major` selects an MN-major B operand (its N
// index contiguous in shared memory) instead of K-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4)                          // accumulator format: fp32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16)   // B major-ness
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.  The
// swizzle atom is 8 rows of 128 bytes (1024-byte aligned); `lbo_bytes` and
// `sbo_bytes` are the leading- and stride-dimension byte offsets:
//   K-major:  rows (M or N) at 128 B, 8-row groups at sbo = 1024, lbo unused (16);
//   MN-major: 64-element MN atoms at lbo, 8-row K groups at sbo = 1024.
__device__ __forceinline__ uint64_t umma_sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                     uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version of sm_100
  d |= (uint64_t)2u << 61;  // layout: 128-byte swizzle
  return d;
}

// The same descriptor as two 32-bit halves: the low half holds the start
// address (bits 0-13) and the leading byte offset, so stepping through a
// tile is one 32-bit add of (byte offset >> 4) to `lo` (no carry leaves the
// 14-bit field for addresses inside the 228 KiB of shared memory).
struct SDesc {
  uint32_t lo, hi;
};
__device__ __forceinline__ SDesc umma_sdesc_sw128_split(uint32_t saddr, uint32_t lbo_bytes,
                                                        uint32_t sbo_bytes) {
  const uint64_t d = umma_sdesc_sw128(saddr, lbo_bytes, sbo_bytes);
  return SDesc{(uint32_t)d, (uint32_t)(d >> 32)};
}

// ------------------------------------------------------------ MMA issue

// D[tmem] (+)= A[smem] * B[smem], issued by one thread; `accumulate` = 0
// overwrites D.  Both descriptors are given as 32-bit halves, their start
// addresses advanced by `a_step` / `b_step` (16-byte units): the issuing
// thread spends two integer adds per MMA instead of rebuilding descriptors.
__device__ __forceinline__ void umma_bf16_ss_step(uint32_t d_tmem, SDesc a, uint32_t a_step, SDesc b,
                                                  uint32_t b_step, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "mov.b64 da, {%1, %2};\n\t"
      "mov.b64 db, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}"
      ::"r"(d_tmem), "r"(a.lo + a_step), "r"(a.hi), "r"(b.lo + b_step), "r"(b.hi), "r"(idesc),
        "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem] (A read from tensor memory: lane = row,
// two consecutive bf16 K elements per 32-bit column, 8 columns per K = 16),
// the B descriptor given as 32-bit halves (see above).
__device__ __forceinline__ void umma_bf16_ts_step(uint32_t d_tmem, uint32_t a_tmem, SDesc b,
                                                  uint32_t b_step, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "r"(b.lo + b_step), "r"(b.hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05.mma this thread issued before it
// has completed (its shared-memory reads and TMEM writes included).
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// ------------------------------------------------------------ TMEM

// Whole warp: allocates `ncols` TMEM columns (a power of two >= 32) and
// writes the base address to shared memory at `slot`.
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// Whole warp: frees what tmem_alloc returned.
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Whole warp: thread i reads 32 consecutive 32-bit columns of TMEM lane
// (lane base of `taddr`) + i.  Complete only after tmem_wait_ld().
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Whole warp: thread i writes 16 consecutive 32-bit columns of its TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Whole warp: the inverse of tmem_ld32.  Complete only after tmem_wait_st().
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
        "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

}  // namespace gqa
