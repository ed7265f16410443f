// Fifth-generation tensor cores on sm_100a: tensor-memory (TMEM) allocation,
// tcgen05.mma with operands described in shared memory, commits to mbarriers,
// and TMEM <-> register moves.  Inline PTX only.
//
// Shared-memory operand layout used here: 128-byte swizzled rows (the layout
// a TMA copy with CU_TENSOR_MAP_SWIZZLE_128B writes), grouped in atoms of 8
// rows x 128 bytes (1024 bytes, 1024-byte aligned).
//   K-major operand (the reduction dimension contiguous): an atom holds 8 rows
//   of 64 16-bit elements; atoms follow each other every 1024 bytes along the
//   rows; one 16-element step of the reduction dimension is +32 bytes of start
//   address, and the next 64 elements live in another region.
//   MN-major operand (the output dimension contiguous): rows run along the
//   reduction dimension, 64 output elements per 128-byte row; the byte
//   distance between 64-element output chunks goes in the leading-byte-offset
//   field, the distance between 8-row groups (1024) in the stride field.
#pragma once

#include <stdint.h>

#include "pa_device.cuh"

namespace pa {

// ---------------------------------------------------------------- descriptors

// Shared-memory matrix descriptor, 128-byte swizzle.  Fields (bit offsets):
// start address >> 4 at 0, leading byte offset >> 4 at 16, stride byte
// offset >> 4 at 32, descriptor version 1 at 46, layout type 2 (128-byte
// swizzle) at 61.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of a dense kind::f16 MMA with fp32 accumulation:
// accumulator format 1 (f32) at bit 4, A and B format (0 f16, 1 bf16) at bits
// 7 and 10, A and B major-ness (0 K, 1 MN) at bits 15 and 16, N >> 3 at
// bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t umma_idesc_f16(bool bf16, int M, int N, bool a_mn,
                                                      bool b_mn) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- TMEM

// Allocate `ncols` TMEM columns (a power of two >= 32); the base address is
// written to *dst (shared memory).  Executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Order tcgen05 operations around a thread synchronisation.
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// The MMA and commit wrappers below are executed by a whole warp with
// warp-uniform operands; one lane, chosen by elect.sync, issues the
// instructions (a fully active warp always elects the same lane, so commits
// track every MMA of the warp).  Keeping the issuing code warp-uniform lets
// the compiler hold the descriptors in uniform registers instead of moving
// them there before every MMA, which measurably speeds up issue when the
// issuing warp shares its scheduler with busy warps.

// Groups of MMAs in one statement: one elect and one predicate set-up for
// all of them, each step's descriptors the group's base plus an immediate
// added to the low word (the start-address field, 16-byte units; bases and
// offsets keep it inside its 14 bits).  The first step accumulates into D
// when acc0 != 0, the others always.  Operands: %0 D (TMEM), %1 A, %2 B,
// %3 instruction descriptor, %4 acc0, then the step offsets.

// One step with A and B in shared memory, both moved by operand OP.
#define PA_UMMA_SS_STEP(OP, PRED)                                               \
  "add.u32 al, a0, %" #OP ";\n\tadd.u32 bl, b0, %" #OP ";\n\t"                  \
  "mov.b64 da, {al, ah};\n\tmov.b64 db, {bl, bh};\n\t"                          \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, " PRED ";\n\t"
// One step with A in tensor memory (column offset operand OA) and B in shared
// memory (start-address offset operand OB).
#define PA_UMMA_TS_STEP(OA, OB, PRED)                                           \
  "add.u32 at, %1, %" #OA ";\n\tadd.u32 bl, b0, %" #OB ";\n\t"                  \
  "mov.b64 db, {bl, bh};\n\t"                                                   \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [at], db, %3, " PRED ";\n\t"
#define PA_UMMA_GROUP_HEAD                                                      \
  "{\n\t.reg .pred e, p, t;\n\t.reg .b32 a0, ah, b0, bh, al, bl, at;\n\t"       \
  ".reg .b64 da, db;\n\t"                                                       \
  "elect.sync _|e, 0xffffffff;\n\t"                                             \
  "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, %4, %4;\n\t"                          \
  "mov.b64 {b0, bh}, %2;\n\t"

// Eight kind::f16 steps, A and B in shared memory, both moved by O0..O7.
template <uint32_t O0, uint32_t O1, uint32_t O2, uint32_t O3, uint32_t O4, uint32_t O5,
          uint32_t O6, uint32_t O7>
__device__ __forceinline__ void umma_ss_group8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                               uint32_t acc0) {
  asm volatile(PA_UMMA_GROUP_HEAD "mov.b64 {a0, ah}, %1;\n\t"
               PA_UMMA_SS_STEP(5, "p") PA_UMMA_SS_STEP(6, "t") PA_UMMA_SS_STEP(7, "t")
               PA_UMMA_SS_STEP(8, "t") PA_UMMA_SS_STEP(9, "t") PA_UMMA_SS_STEP(10, "t")
               PA_UMMA_SS_STEP(11, "t") PA_UMMA_SS_STEP(12, "t") "}" ::"r"(d),
               "l"(a), "l"(b), "r"(idesc), "r"(acc0), "n"(O0), "n"(O1), "n"(O2), "n"(O3),
               "n"(O4), "n"(O5), "n"(O6), "n"(O7)
               : "memory");
}

// Four such steps.
template <uint32_t O0, uint32_t O1, uint32_t O2, uint32_t O3>
__device__ __forceinline__ void umma_ss_group4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                               uint32_t acc0) {
  asm volatile(PA_UMMA_GROUP_HEAD "mov.b64 {a0, ah}, %1;\n\t"
               PA_UMMA_SS_STEP(5, "p") PA_UMMA_SS_STEP(6, "t") PA_UMMA_SS_STEP(7, "t")
               PA_UMMA_SS_STEP(8, "t") "}" ::"r"(d),
               "l"(a), "l"(b), "r"(idesc), "r"(acc0), "n"(O0), "n"(O1), "n"(O2), "n"(O3)
               : "memory");
}

// Eight steps with A in tensor memory (column offsets A0..A7 from a_tmem; row
// i of A in lane i, two 16-bit elements per 32-bit column, the lower index in
// the low half) and B in shared memory (start-address offsets B0..B7).
template <uint32_t A0, uint32_t A1, uint32_t A2, uint32_t A3, uint32_t A4, uint32_t A5,
          uint32_t A6, uint32_t A7, uint32_t B0, uint32_t B1, uint32_t B2, uint32_t B3,
          uint32_t B4, uint32_t B5, uint32_t B6, uint32_t B7>
__device__ __forceinline__ void umma_ts_group8(uint32_t d, uint32_t a_tmem, uint64_t b,
                                               uint32_t idesc, uint32_t acc0) {
  asm volatile(PA_UMMA_GROUP_HEAD
               PA_UMMA_TS_STEP(5, 13, "p") PA_UMMA_TS_STEP(6, 14, "t") PA_UMMA_TS_STEP(7, 15, "t")
               PA_UMMA_TS_STEP(8, 16, "t") PA_UMMA_TS_STEP(9, 17, "t") PA_UMMA_TS_STEP(10, 18, "t")
               PA_UMMA_TS_STEP(11, 19, "t") PA_UMMA_TS_STEP(12, 20, "t") "}" ::"r"(d),
               "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc0), "n"(A0), "n"(A1), "n"(A2), "n"(A3),
               "n"(A4), "n"(A5), "n"(A6), "n"(A7), "n"(B0), "n"(B1), "n"(B2), "n"(B3), "n"(B4),
               "n"(B5), "n"(B6), "n"(B7)
               : "memory");
}

#undef PA_UMMA_SS_STEP
#undef PA_UMMA_TS_STEP
#undef PA_UMMA_GROUP_HEAD

// Arrive once on `bar` when every MMA the warp issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_addr(bar))
      : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane -> registers, and
// wait for them (the wait is in the same statement, so no use of the
// registers can be scheduled before it).  taddr: lane in bits 31..16 (the
// warp's 32-lane quarter), column in bits 15..0.  Whole warp.
__device__ __forceinline__ void tmem_load32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane -> registers (and wait).
__device__ __forceinline__ void tmem_load16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// 8 consecutive 32-bit TMEM columns of this thread's lane <- registers (and wait).
__device__ __forceinline__ void tmem_store8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// 8 consecutive TMEM columns <- registers, without waiting (the registers are
// read at issue; tmem_store_wait() before anything depends on the columns).
__device__ __forceinline__ void tmem_store8_async(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}
// 16 consecutive TMEM columns <- registers, without waiting.
__device__ __forceinline__ void tmem_store16_async(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_store_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 3-D tiled tensor copy global -> shared (x innermost, in elements; callers
// keep x * elem_size a multiple of 16 bytes).
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y,
                                            int z, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// 3-D tiled tensor copy shared -> global (a TMA store), tracked in the
// issuing thread's bulk async-group; coordinates as for tma_load_3d, never
// negative.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int x,
                                             int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_addr(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every bulk store this thread committed has read its
// shared-memory source (which may then be reused or freed; the global
// writes complete on their own, before the grid counts as finished).
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Barrier among `count` threads of the CTA on hardware barrier `id` (1..15).
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace pa
