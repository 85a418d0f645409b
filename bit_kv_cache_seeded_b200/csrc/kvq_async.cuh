// Asynchronous global -> shared copies (cp.async, 16 bytes per thread per call), shared by the
// kernels that stage tiles or the sketch matrix in shared memory. Both addresses must be
// 16-byte aligned. A thread's copies complete at cp_async_wait<N>() (all but its N most recent
// commit groups); other threads see them only after a barrier that follows the wait.
#pragma once

#include <cstdint>

namespace kvq {

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
// Arrives once on the mbarrier when every cp.async this thread issued before has completed (the
// barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Bulk (TMA 1-D) copies global -> shared that complete on an mbarrier. One thread arms the
// barrier with the byte count it expects (arrive + expect_tx) and issues the copies; every thread
// then waits on the barrier's phase parity. Addresses and sizes must be multiples of 16 bytes.
__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
// Makes initialised barriers visible to the bulk-copy unit (before the first copy names them).
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
// One arrival (count 1) on the barrier, releasing this thread's earlier shared-memory accesses.
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// Orders this thread's earlier generic-proxy shared-memory accesses (after a barrier, those of
// the whole CTA) before later bulk copies into the same buffer.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
// One non-blocking test of the barrier's phase with parity `parity`: true if it has completed.
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred q;\n mbarrier.test_wait.parity.shared::cta.b64 q, [%1], %2;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(done) : "r"(bar), "r"(parity) : "memory");
  return done != 0;
}

// Waits until the barrier's phase with parity `parity` has completed, giving up after `limit`
// SM clock cycles. Returns false if it gave up. Each try_wait may suspend the thread (up to the
// hint, 100 us) until the phase completes, so a waiting warp takes no issue slots meanwhile.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  while (true) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2, %3;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(done) : "r"(bar), "r"(parity), "r"(100000u) : "memory");
    if (done) return true;
    if (clock64() - t0 > limit) return false;
  }
}

// The same wait without a suspend-time hint: each try_wait returns after the hardware's own short
// limit, so a thread that waits on a neighbour in a pipeline resumes as soon as the phase completes.
__device__ __forceinline__ bool mbar_wait_spin(uint32_t bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  while (true) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(done) : "r"(bar), "r"(parity) : "memory");
    if (done) return true;
    if (clock64() - t0 > limit) return false;
  }
}

// The same wait polling with the non-blocking test (and a short sleep between tests), for warps
// that wait on a neighbour in a pipeline: a blocking try_wait would hold the barrier unit while
// other warps of the CTA need it.
__device__ __forceinline__ bool mbar_wait_poll(uint32_t bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  while (!mbar_try(bar, parity)) {
    if (clock64() - t0 > limit) return false;
    __nanosleep(20);
  }
  return true;
}

// Programmatic dependent launch (sm_90+). A kernel launched with programmatic stream
// serialization may start while its predecessor in the stream is still running; grid_dep_wait()
// blocks until that predecessor has completed and its memory is visible, so everything that
// reads the predecessor's output must follow it. grid_dep_launch() lets the successor be
// scheduled before this grid ends. Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

}  // namespace kvq
