// Thin inline-PTX wrappers for the sm_100a features the tensor-core decode
// uses: mbarriers, 1-D bulk async copies (TMA), tcgen05 tensor-memory
// allocation, UMMA issue/commit and tensor-memory loads and stores.  Each wrapper is one
// PTX instruction (or a bounded loop around one).
#pragma once

#include <stdint.h>

namespace kvq {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking: whether phase `parity` of the barrier has completed.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// As mbar_try_wait, but the thread may stay suspended (not polling) for up to
// `ns` nanoseconds while the phase is incomplete; it resumes as soon as the
// phase completes.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Wait for phase `parity` of the barrier, giving up after `limit` polls (each
// poll itself suspends for a bounded, hardware-chosen time).  Returns false on
// give-up so the caller can flag the result instead of hanging.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t limit = 1u << 22) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// ---------------------------------------------------------------- bulk copy
// 1-D bulk copy global -> shared, completion counted in bytes on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// generic-proxy shared-memory writes -> visible to the async proxy (UMMA operands)
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- tensor memory
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, no swizzle: start address, leading-dim
// byte offset (LBO), stride-dim byte offset (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// Instruction descriptor for kind::f16 with f16 A/B and f32 accumulation.
// a_mn / b_mn: operand stored MN-major (1) or K-major (0).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                        // D format: f32
         | (0u << 7) | (0u << 10)         // A, B format: f16
         | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16)
         | ((uint32_t)(N >> 3) << 17)     // N / 8
         | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
// D[tmem] (+)= A[tmem] * B[smem]^T, issued by one thread.  A sits in tensor
// memory: row m of A in lane m, its K elements packed two per 32-bit column.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Instruction descriptor for kind::i8: unsigned 8-bit A, signed 8-bit B, s32 accumulation, both K-major.
__host__ __device__ constexpr uint32_t idesc_u8s8_s32(int M, int N) {
  return (2u << 4)                        // D format: s32
         | (0u << 7) | (1u << 10)         // A: unsigned 8-bit, B: signed 8-bit
         | ((uint32_t)(N >> 3) << 17)     // N / 8
         | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// Instruction descriptor for kind::i8: unsigned 8-bit A (K-major) and B
// (MN-major), s32 accumulation.
__host__ __device__ constexpr uint32_t idesc_u8u8_s32_bmn(int M, int N) {
  return (2u << 4)                        // D format: s32
         | (0u << 7) | (0u << 10)         // A, B: unsigned 8-bit
         | (1u << 16)                     // B stored MN-major
         | ((uint32_t)(N >> 3) << 17)     // N / 8
         | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// D[tmem] (+)= A[tmem] * B[smem]^T on 8-bit integers (K = 32 per instruction), issued by one thread.
__device__ __forceinline__ void umma_i8_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Arrive once on `bar` when every UMMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Register budget of the calling warpgroup (all four warps execute the same
// instruction): dec releases registers down to N per thread, inc waits until
// N per thread are free in the pool the block was launched with.
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Each thread of the warp reads N consecutive 32-bit columns of its own lane.
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]);

template <>
__device__ __forceinline__ void tmem_ld<2>(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<1>(uint32_t taddr, uint32_t (&r)[1]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Loads that complete inside the same asm statement: the destination
// registers of tcgen05.ld are only defined after tcgen05.wait::ld, so the
// wait is issued before the compiler may touch them.
// N consecutive columns at taddr.
template <int N>
__device__ __forceinline__ void tmem_ld_wait(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld_wait<1>(uint32_t taddr, uint32_t (&r)[1]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0])
      : "r"(taddr)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_wait<2>(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1])
      : "r"(taddr)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_wait<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "r"(taddr)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_wait<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_wait<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_wait<32>(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// A load split in two: tmem_ld_start issues it, tmem_ld_finish waits for it
// (the registers are tied through the wait, so nothing reads them before).
template <int N>
__device__ __forceinline__ void tmem_ld_start(uint32_t taddr, uint32_t (&r)[N]);
template <int N>
__device__ __forceinline__ void tmem_ld_finish(uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld_start<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_finish<4>(uint32_t (&r)[4]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]) : : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_start<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];" : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_finish<8>(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]) : : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_start<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];" : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_finish<16>(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]) : : "memory");
}

// Scores and PV sums of an epilogue tile in one round trip: four runs of
// 2 HH columns at taddr + g * stride (g = 0..3) and one run of 4 HH columns at
// paddr, then one wait for all of them.
template <int HH>
__device__ __forceinline__ void tmem_ld_sc_pv(uint32_t taddr, uint32_t stride, uint32_t paddr, uint32_t (&s)[4][2 * HH],
                                              uint32_t (&p)[4 * HH]);
template <>
__device__ __forceinline__ void tmem_ld_sc_pv<1>(uint32_t taddr, uint32_t stride, uint32_t paddr,
                                                   uint32_t (&s)[4][2], uint32_t (&p)[4]) {
  asm volatile(
      "{\n\t.reg .b32 a;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%12];\n\t"
      "mov.u32 a, %12;\n\t"
      "add.u32 a, a, %13;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%2, %3}, [a];\n\t"
      "add.u32 a, a, %13;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%4, %5}, [a];\n\t"
      "add.u32 a, a, %13;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%6, %7}, [a];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%8, %9, %10, %11}, [%14];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=r"(s[0][0]), "=r"(s[0][1]), "=r"(s[1][0]), "=r"(s[1][1]), "=r"(s[2][0]), "=r"(s[2][1]), "=r"(s[3][0]), "=r"(s[3][1]), "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3])
      : "r"(taddr), "r"(stride), "r"(paddr)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_sc_pv<2>(uint32_t taddr, uint32_t stride, uint32_t paddr,
                                                   uint32_t (&s)[4][4], uint32_t (&p)[8]) {
  asm volatile(
      "{\n\t.reg .b32 a;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%24];\n\t"
      "mov.u32 a, %24;\n\t"
      "add.u32 a, a, %25;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4, %5, %6, %7}, [a];\n\t"
      "add.u32 a, a, %25;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%8, %9, %10, %11}, [a];\n\t"
      "add.u32 a, a, %25;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%12, %13, %14, %15}, [a];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%16, %17, %18, %19, %20, %21, %22, %23}, [%26];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=r"(s[0][0]), "=r"(s[0][1]), "=r"(s[0][2]), "=r"(s[0][3]), "=r"(s[1][0]), "=r"(s[1][1]), "=r"(s[1][2]), "=r"(s[1][3]), "=r"(s[2][0]), "=r"(s[2][1]), "=r"(s[2][2]), "=r"(s[2][3]), "=r"(s[3][0]), "=r"(s[3][1]), "=r"(s[3][2]), "=r"(s[3][3]), "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3]), "=r"(p[4]), "=r"(p[5]), "=r"(p[6]), "=r"(p[7])
      : "r"(taddr), "r"(stride), "r"(paddr)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld_sc_pv<4>(uint32_t taddr, uint32_t stride, uint32_t paddr,
                                                   uint32_t (&s)[4][8], uint32_t (&p)[16]) {
  asm volatile(
      "{\n\t.reg .b32 a;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%48];\n\t"
      "mov.u32 a, %48;\n\t"
      "add.u32 a, a, %49;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%8, %9, %10, %11, %12, %13, %14, %15}, [a];\n\t"
      "add.u32 a, a, %49;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%16, %17, %18, %19, %20, %21, %22, %23}, [a];\n\t"
      "add.u32 a, a, %49;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%24, %25, %26, %27, %28, %29, %30, %31}, [a];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47}, [%50];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=r"(s[0][0]), "=r"(s[0][1]), "=r"(s[0][2]), "=r"(s[0][3]), "=r"(s[0][4]), "=r"(s[0][5]), "=r"(s[0][6]), "=r"(s[0][7]), "=r"(s[1][0]), "=r"(s[1][1]), "=r"(s[1][2]), "=r"(s[1][3]), "=r"(s[1][4]), "=r"(s[1][5]), "=r"(s[1][6]), "=r"(s[1][7]), "=r"(s[2][0]), "=r"(s[2][1]), "=r"(s[2][2]), "=r"(s[2][3]), "=r"(s[2][4]), "=r"(s[2][5]), "=r"(s[2][6]), "=r"(s[2][7]), "=r"(s[3][0]), "=r"(s[3][1]), "=r"(s[3][2]), "=r"(s[3][3]), "=r"(s[3][4]), "=r"(s[3][5]), "=r"(s[3][6]), "=r"(s[3][7]), "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3]), "=r"(p[4]), "=r"(p[5]), "=r"(p[6]), "=r"(p[7]), "=r"(p[8]), "=r"(p[9]), "=r"(p[10]), "=r"(p[11]), "=r"(p[12]), "=r"(p[13]), "=r"(p[14]), "=r"(p[15])
      : "r"(taddr), "r"(stride), "r"(paddr)
      : "memory");
}
// Four runs of N columns at taddr + k * stride (k = 0..3), one wait for all.
template <int N>
__device__ __forceinline__ void tmem_ld4_wait(uint32_t taddr, uint32_t stride, uint32_t (&r)[4][N]);
template <>
__device__ __forceinline__ void tmem_ld4_wait<1>(uint32_t taddr, uint32_t stride, uint32_t (&r)[4][1]) {
  asm volatile(
      "{\n\t.reg .b32 a;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%4];\n\t"
      "add.u32 a, %4, %5;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%1}, [a];\n\t"
      "add.u32 a, a, %5;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%2}, [a];\n\t"
      "add.u32 a, a, %5;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%3}, [a];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=r"(r[0][0]), "=r"(r[1][0]), "=r"(r[2][0]), "=r"(r[3][0])
      : "r"(taddr), "r"(stride)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld4_wait<2>(uint32_t taddr, uint32_t stride, uint32_t (&r)[4][2]) {
  asm volatile(
      "{\n\t.reg .b32 a;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%8];\n\t"
      "add.u32 a, %8, %9;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%2, %3}, [a];\n\t"
      "add.u32 a, a, %9;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%4, %5}, [a];\n\t"
      "add.u32 a, a, %9;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%6, %7}, [a];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[2][0]), "=r"(r[2][1]), "=r"(r[3][0]),
        "=r"(r[3][1])
      : "r"(taddr), "r"(stride)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld4_wait<4>(uint32_t taddr, uint32_t stride, uint32_t (&r)[4][4]) {
  asm volatile(
      "{\n\t.reg .b32 a;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%16];\n\t"
      "add.u32 a, %16, %17;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4, %5, %6, %7}, [a];\n\t"
      "add.u32 a, a, %17;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%8, %9, %10, %11}, [a];\n\t"
      "add.u32 a, a, %17;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%12, %13, %14, %15}, [a];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]),
        "=r"(r[1][3]), "=r"(r[2][0]), "=r"(r[2][1]), "=r"(r[2][2]), "=r"(r[2][3]), "=r"(r[3][0]), "=r"(r[3][1]),
        "=r"(r[3][2]), "=r"(r[3][3])
      : "r"(taddr), "r"(stride)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld4_wait<8>(uint32_t taddr, uint32_t stride, uint32_t (&r)[4][8]) {
  asm volatile(
      "{\n\t.reg .b32 a;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%32];\n\t"
      "add.u32 a, %32, %33;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%8, %9, %10, %11, %12, %13, %14, %15}, [a];\n\t"
      "add.u32 a, a, %33;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%16, %17, %18, %19, %20, %21, %22, %23}, [a];\n\t"
      "add.u32 a, a, %33;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%24, %25, %26, %27, %28, %29, %30, %31}, [a];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t}"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]), "=r"(r[0][6]),
        "=r"(r[0][7]), "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3]), "=r"(r[1][4]), "=r"(r[1][5]),
        "=r"(r[1][6]), "=r"(r[1][7]), "=r"(r[2][0]), "=r"(r[2][1]), "=r"(r[2][2]), "=r"(r[2][3]), "=r"(r[2][4]),
        "=r"(r[2][5]), "=r"(r[2][6]), "=r"(r[2][7]), "=r"(r[3][0]), "=r"(r[3][1]), "=r"(r[3][2]), "=r"(r[3][3]),
        "=r"(r[3][4]), "=r"(r[3][5]), "=r"(r[3][6]), "=r"(r[3][7])
      : "r"(taddr), "r"(stride)
      : "memory");
}


// Each thread of the warp writes N consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
// N = 1, 2, 4 or 8 consecutive columns of this thread's lane.
template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_st_n<1>(uint32_t taddr, const uint32_t (&r)[1]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r[0]) : "memory");
}
template <>
__device__ __forceinline__ void tmem_st_n<2>(uint32_t taddr, const uint32_t (&r)[2]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(r[0]), "r"(r[1]) : "memory");
}
template <>
__device__ __forceinline__ void tmem_st_n<4>(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_st_n<8>(uint32_t taddr, const uint32_t (&r)[8]) { tmem_st8(taddr, r); }
// The calling thread's earlier tcgen05.st have completed.
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- paired fp32
// (d.x, d.y) = (a.x * b.x + c.x, a.y * b.y + c.y), each rounded once: one
// instruction for both lanes of the pair.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// ---------------------------------------------------------------- code -> f16
// Value codes enter the PV MMA centred, as c - L/2 (exact f16 values): the
// products then average out instead of all being positive, which keeps the
// fp32 accumulator near the size of the result (the zero point takes the L/2).
//
// Eight 4-bit codes n0..n7 (n_i in bits 4i..4i+3 of x) -> f16 (n_i - 7.5) as
// half2 pairs (n0,n4) (n1,n5) (n2,n6) (n3,n7).  Each nibble is moved to bits
// 4..7 of its half and OR-ed into the mantissa of 1024.0 (0x6400), giving
// 1024 + 16 n; one fma (x 1/16, - 71.5) leaves n - 7.5; all exact in f16.
__device__ __forceinline__ void codes4_to_f16(uint32_t x, uint32_t (&r)[4]) {
  const uint32_t magic = 0x64006400u;
  const uint32_t sel = 0x00F000F0u;
  uint32_t a, b, c, d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(a) : "r"(x << 4), "r"(sel), "r"(magic));
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(b) : "r"(x), "r"(sel), "r"(magic));
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(c) : "r"(x >> 4), "r"(sel), "r"(magic));
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(x >> 8), "r"(sel), "r"(magic));
  const uint32_t mul16 = 0x2C002C00u;  // (1/16, 1/16)
  const uint32_t add = 0xD478D478u;    // (-71.5, -71.5)
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r[0]) : "r"(a), "r"(mul16), "r"(add));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r[1]) : "r"(b), "r"(mul16), "r"(add));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r[2]) : "r"(c), "r"(mul16), "r"(add));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r[3]) : "r"(d), "r"(mul16), "r"(add));
}

// Sixteen 2-bit codes f0..f15 (f_i in bits 2i..2i+1) -> f16 (f_i - 1.5) as
// half2 pairs (f0,f8) (f1,f9) ... (f7,f15).  Field k (k = 1..3) of each half,
// OR-ed in place into 1024.0, is 1024 + 4^k f; one fma (x 4^-k, -1024 4^-k -
// 1.5) leaves f - 1.5.  Field 0 is first moved to field 1's bits (-1025.5 is
// not an f16 value).  All exact in f16.
__device__ __forceinline__ void codes2_to_f16(uint32_t x, uint32_t (&r)[8]) {
  const uint32_t magic = 0x64006400u;
  const uint32_t mul[4] = {0x34003400u, 0x34003400u, 0x2C002C00u, 0x24002400u};  // 1/4, 1/4, 1/16, 1/64
  const uint32_t add[4] = {0xDC06DC06u, 0xDC06DC06u, 0xD418D418u, 0xCC60CC60u};  // -257.5, -257.5, -65.5, -17.5
  const uint32_t xs[2] = {x, x >> 8};
#pragma unroll
  for (int half = 0; half < 2; ++half)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t t;
      const uint32_t src = k == 0 ? xs[half] << 2 : xs[half];
      const uint32_t m = 0x00030003u << (2 * (k == 0 ? 1 : k));
      asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(t) : "r"(src), "r"(m), "r"(magic));
      asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r[half * 4 + k]) : "r"(t), "r"(mul[k]), "r"(add[k]));
    }
}

}  // namespace sm100
}  // namespace kvq
