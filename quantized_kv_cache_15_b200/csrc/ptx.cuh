// Thin inline-PTX wrappers: mbarriers, bulk copies global -> shared, timers.
// Every wait is bounded: after the limit the caller gets `false` and latches an
// error bit; no kernel in this library can spin forever.
#pragma once

#include <cstdint>

namespace kvq {

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of the same condition (never suspends the thread): for a
// thread that polls several barriers in turn.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete; gives up after limit_ns
// (2 s by default).  A thread that expects a long wait (a producer whose ring is
// full while the consumers compute) passes max_sleep_ns > 0: between tries it then
// sleeps, 64 ns at first and doubling up to max_sleep_ns, so that it takes few issue
// slots from the warps that share its scheduler.  Others retry at once (try_wait
// itself blocks for a short while), so they resume as soon as the phase completes.
// The timer is read every 16 tries.  The slow path is a separate function so that
// it takes no registers in the callers' loops.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                   uint32_t max_sleep_ns) {
  const uint64_t t0 = globaltimer_ns();
  uint32_t sleep_ns = 64;
  for (uint32_t i = 0; i < (1u << 26); ++i) {
    if (max_sleep_ns) {
      __nanosleep(sleep_ns);
      if (sleep_ns < max_sleep_ns) sleep_ns <<= 1;
    }
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15) == 15 && globaltimer_ns() - t0 > limit_ns) break;
  }
  return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = 2000000000ull,
                                          uint32_t max_sleep_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, limit_ns, max_sleep_ns);
}

// Bulk copy (TMA, untiled) of `bytes` (multiple of 16, both addresses 16-byte
// aligned) from global memory into this CTA's shared memory; completion is
// signalled on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Atomic add at gpu scope with acquire-release semantics: publishes the writes that
// happen before it and makes the other publishers' writes visible after it.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
// Order this thread's ordinary (generic-proxy) memory accesses before its later
// bulk-copy (async-proxy) accesses: to global memory / to this CTA's shared memory.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Programmatic dependent launch (kernels launched with the programmatic
// stream-serialization attribute).  launch_dependents lets the next kernel in the
// stream be scheduled before this grid finishes; wait blocks until every
// prerequisite grid has completed and its memory is visible.  A kernel calls wait
// before touching anything an earlier kernel may write.
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace kvq
