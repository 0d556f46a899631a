// Thin inline-PTX wrappers for sm_100a: 1-D bulk async copies (TMA bulk engine)
// completing on shared-memory mbarriers, bounded mbarrier waits, programmatic
// dependent launch controls and the byte dot-product instruction.
#pragma once
#include <cstdint>

#include <cuda_runtime.h>

#include "tern_internal.h"

namespace tern {

// Device error word of this translation unit (bit flags TERN_DEVERR_*); each
// kernel file exposes a host accessor that reads and clears it, and
// tern_device_error() collects them all.
static __device__ unsigned int g_dev_error = 0;

static inline int read_clear_dev_error_tu(void* stream, unsigned* out) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_dev_error, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_dev_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  *out |= v;
  return (int)e;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before later
// async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Evict-first L2 policy for streamed-once weights.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Bulk copy global -> shared of `bytes` (multiple of 16, both addresses 16-byte
// aligned), completing `bytes` transactions on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// One potentially blocking test of the phase: the thread may be suspended
// for up to about 0.5 ms waiting for the phase to complete (so a waiting warp
// does not spin on the issue slots).
// kCluster: acquire at cluster scope, for phases that other CTAs' st.async
// stores complete.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  if constexpr (kCluster)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(500000u)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(500000u)
        : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of `bar` to complete, giving up after about
// limit_ns (kWaitLimitNs in every GEMV kernel); on expiry the device error
// word records a timeout and false is returned (the caller then stops using
// the stage).
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait_bounded_ns(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait<kCluster>(bar, parity)) return true;
  // back off between tests so that waiting warps leave the issue slots to the
  // warps that have data; check the time limit only now and then
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(it < 4 ? 32u : 128u);
    if (mbar_try_wait<kCluster>(bar, parity)) return true;
    if ((it & 63u) == 0u && global_timer_ns() - t0 > limit_ns) {
      atomicOr(&g_dev_error, TERN_DEVERR_TIMEOUT);
      return false;
    }
  }
}

template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  return mbar_wait_bounded_ns<kCluster>(bar, parity, kWaitLimitNs);
}

// Programmatic dependent launch: wait until the preceding grid on the stream
// has completed and its memory is visible (no-op without the launch attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next grid on the stream to be scheduled now.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- thread-block clusters (distributed shared memory)
// Every thread of every CTA in the cluster executes each barrier exactly once,
// in the same order, so these waits always complete.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_cluster_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
// Store into a CTA's shared memory that completes its byte count on that CTA's
// mbarrier (`addr` and `bar` mapped into the same CTA of the cluster): the
// receiver learns of the data by waiting on its own barrier, with no
// cluster-wide barrier.
__device__ __forceinline__ void st_async_u32(uint32_t addr, uint32_t v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(addr), "r"(v),
               "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async_u64(uint32_t addr, unsigned long long v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u64 [%0], %1, [%2];" ::"r"(addr), "l"(v),
               "r"(bar)
               : "memory");
}

// 16-byte shared-memory loads from a 32-bit shared address plus an immediate offset.
template <int OFF>
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4+%5];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr), "n"(OFF));
  return v;
}
__device__ __forceinline__ int4 u4_as_i4(uint4 v) { return make_int4((int)v.x, (int)v.y, (int)v.z, (int)v.w); }

// Four-way byte dot products with 32-bit accumulation.
__device__ __forceinline__ int dp4a_ss(int a, int b, int c) { return __dp4a(a, b, c); }
__device__ __forceinline__ unsigned dp4a_uu(unsigned a, unsigned b, unsigned c) { return __dp4a(a, b, c); }
// unsigned bytes of a times signed bytes of b
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t lop3_ternary_digit(uint32_t w) {
  // Per 2-bit field with code c (00 -> 0, 01 -> +1, 10 -> -1) produce the
  // digit F = 1 - t in {1, 0, 2}: high bit = c_hi, low bit = NOR(c_lo, c_hi).
  uint32_t f;
  const uint32_t w1 = w >> 1;
  // f = odd bits ? w : ~(w | w1)   with mask 0x55555555 selecting even bits
  asm("lop3.b32 %0, %1, %2, %3, 0x52;" : "=r"(f) : "r"(w), "r"(w1), "r"(0x55555555u));
  return f;
}

}  // namespace tern
