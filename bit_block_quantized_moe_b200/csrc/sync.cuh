// Device-side synchronisation primitives with bounded waits (sm_100a).
//
// Every wait here gives up after kWaitLimitNs of %globaltimer time, reports
// the timeout through the caller's status word and returns false, so that no
// kernel can spin forever.
#pragma once

#include "common.cuh"

namespace moe {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier ------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One hardware wait for the phase with the given parity: the thread may be
// suspended until the phase completes or a system-dependent time limit passes;
// true once the phase has completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete; false after the limit.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// ---- cp.async (load/store-unit path, 16 B per thread) ----------------------------
// Many threads each moving 16-byte pieces keep far more bytes in flight per SM
// than one thread issuing large bulk copies.
__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed cp.async groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// A warp copies `bytes` (a multiple of 16, both addresses 16-byte aligned): lane i moves pieces i, i + 32, ...
__device__ __forceinline__ void warp_cp_async(void *dst_smem, const void *src, uint32_t bytes, int lane) {
  uint8_t *d = static_cast<uint8_t *>(dst_smem);
  const uint8_t *sp = static_cast<const uint8_t *>(src);
  for (uint32_t o = (uint32_t)lane * 16u; o < bytes; o += 512u) cp_async16(d + o, sp + o);
}

__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---- CTA-level ---------------------------------------------------------------------
__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint4 lds128(const void *p) { return *reinterpret_cast<const uint4 *>(p); }

// ---- grid-level ----------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Loads through L2 only (data written earlier in the same kernel by other CTAs).
__device__ __forceinline__ float4 ldg_cg_f4(const void *p) { return __ldcg(reinterpret_cast<const float4 *>(p)); }

__device__ __forceinline__ uint64_t ld_acquire_gpu_u64(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Grid barriers of a cooperatively launched (all CTAs resident) grid over one
// monotonic 64-bit arrival counter (zeroed once with the workspace, never
// reset: every CTA adds 1 per barrier, and every launch passes the same number
// of barriers), each split in two so that independent work can run between
// arriving and waiting.  The leader reads the counter at kernel start and
// derives the targets; grid_arrive_release: the participating threads meet at
// named barrier `bar_id`, the leader's release add publishes the CTA's earlier
// writes.  grid_wait: the leader polls (acquire) until the counter reaches the
// target, then the threads meet again; it returns false (and sets the status
// timeout bit) if the wait hit the limit.

// Arrival with the target known in advance: the leader read the counter at kernel start, before this CTA
// arrived anywhere, so it held (earlier launches x barriers per launch) x grid plus fewer than grid; the
// first barrier's target is the next multiple of the grid size, the i-th one i - 1 grid sizes beyond it.
// The arrival is a release add whose value nobody waits for.
__device__ __forceinline__ void grid_arrive_release(uint64_t *count, int bar_id, int nthreads, bool leader) {
  named_bar(bar_id, nthreads);
  if (leader) asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(count) : "memory");
}

__device__ __forceinline__ bool grid_wait(const uint64_t *count, uint64_t target, int bar_id, int nthreads,
                                          bool leader, uint32_t *status, int *flag_smem) {
  if (leader) {
    bool ok = true;
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_gpu_u64(count) < target) {
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        set_status(status, kStatusTimeout);
        ok = false;
        break;
      }
      __nanosleep(32);
    }
    *flag_smem = ok ? 0 : 1;
  }
  named_bar(bar_id, nthreads);
  return *(volatile int *)flag_smem == 0;
}

}  // namespace moe
