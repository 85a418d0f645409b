// Asynchronous global -> shared copies (cp.async, 16 bytes per thread per call), shared by the
// kernels that stage tiles or the sketch matrix in shared memory. Both addresses must be
// 16-byte aligned. A thread's copies complete at cp_async_wait<N>() (all but its N most recent
// commit groups); other threads see them only after a barrier that follows the wait.
#pragma once

namespace kvq {

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Programmatic dependent launch (sm_90+). A kernel launched with programmatic stream
// serialization may start while its predecessor in the stream is still running; grid_dep_wait()
// blocks until that predecessor has completed and its memory is visible, so everything that
// reads the predecessor's output must follow it. grid_dep_launch() lets the successor be
// scheduled before this grid ends. Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

}  // namespace kvq
