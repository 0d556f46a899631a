// Inline-PTX wrappers for the 5th-generation tensor cores of sm_100a
// (tcgen05): tensor-memory allocation, shared-memory matrix descriptors, the
// 8-bit integer MMA with its completion commit, and tensor-memory loads.
// Field layouts follow the PTX ISA's tcgen05 descriptor definitions.
#pragma once
#include <cstdint>

#include "tern_ptx.cuh"

namespace tern {
namespace tc {

// Allocate `ncols` tensor-memory columns (power of two >= 32) for this CTA; the
// base address is written to shared memory at `dst`. Executed by one whole warp.
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

// Ordering of tcgen05 operations across thread synchronisation.
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, no swizzle (canonical K-major layout of
// 8-row x 16-byte core matrices): start address, leading byte offset (between
// core matrices adjacent along K), stride byte offset (between core matrices
// adjacent along M or N), descriptor version 1 at bits 46-47, swizzle mode 0.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Shared-memory matrix descriptor, 64-byte swizzle, K-major: rows of 64 bytes,
// 8-row atoms of 512 bytes (16-byte chunk c of row r stored at chunk
// c ^ ((r >> 1) & 3)); stride byte offset between 8-row groups, leading byte
// offset unused (1), swizzle mode 4 at bits 61-63. The atom base must be
// 512-byte aligned; a K offset inside the 64-byte row is added to the start.
__device__ __forceinline__ uint64_t smem_desc_sw64(uint32_t addr, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (4ull << 61);
}

// Instruction descriptor of kind::i8 with signed A and B, int32 accumulator,
// both operands K-major, M = 128 rows, N columns (16..256, multiple of 16).
__host__ __device__ constexpr uint32_t idesc_i8_s32(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Eight consecutive 32-bit columns of this warp's 32 lanes (lane quarter
// warp_id % 4); thread i receives lane 32 * (warp_id % 4) + i. The load and
// its completion wait are one statement, so no use of the registers can be
// scheduled before the data has arrived.
__device__ __forceinline__ void ld_x8_sync(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
      : "r"(taddr)
      : "memory");
}

// Four consecutive 32-bit columns of this warp's lane quarter, as ld_x8_sync.
__device__ __forceinline__ void ld_x4_sync(uint32_t taddr, uint32_t (&v)[4]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
      : "r"(taddr)
      : "memory");
}

// Words after the mbarriers of a tensor-core kernel: the tensor-memory base
// address, the abort flag of its bounded waits, the last-arrival flag.
constexpr int kMiscTmem = 0, kMiscAbort = 1, kMiscLast = 2;

// Non-blocking test of a phase.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait by polling (a suspended try_wait resumes too late for the
// one-thread roles on the critical path). Gives up at once when another thread
// of the CTA has already given up (misc[kMiscAbort]), so that a failure costs
// about one time limit, not one per wait.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* misc) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test(bar, parity)) return true;
    if ((it & 255u) == 0u) {
      if (misc[kMiscAbort]) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        atomicOr(&g_dev_error, TERN_DEVERR_TIMEOUT);
        misc[kMiscAbort] = 1u;
        return false;
      }
    }
  }
}

// The same bounded wait for roles of many warps: they sleep between tests, so
// that hundreds of waiting threads do not crowd the issue slots and the
// shared-memory pipe that the single-thread producer and MMA roles need.
__device__ __forceinline__ bool tc_wait_many(uint64_t* bar, uint32_t parity, volatile uint32_t* misc) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (mbar_test(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (misc[kMiscAbort]) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        atomicOr(&g_dev_error, TERN_DEVERR_TIMEOUT);
        misc[kMiscAbort] = 1u;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bulk copy without a cache-policy hint (a tile's weights are read again by
// its next token pass, so they should stay in L2).
__device__ __forceinline__ void bulk_g2s_plain(uint32_t dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst_smem),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

}  // namespace tc
}  // namespace tern
