// sm_100a primitives for kernels that stage tiles through shared memory with
// the Tensor Memory Accelerator: mbarriers with bounded waits, tiled bulk
// tensor loads and stores of this CTA's own boxes, the async-proxy
// fence, and named barriers.  Inline PTX, written from the PTX ISA's
// descriptions of mbarrier, cp.async.bulk.tensor and bar.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace cmr {
namespace tma {

// A wait gives up after this long (ns of %globaltimer); steady-state waits
// here last microseconds.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Limit of the consumers' waits for a stage's data.  Builds of the library
// use kWaitLimitNs; the time-out test compiles a separate copy with
// -DCMR_CONSUMER_WAIT_LIMIT_NS=0, so that these waits give up on ordinary
// copies and the time-out path runs, while the producer's drain keeps the
// full limit and still sees every load it issued land.
#ifdef CMR_CONSUMER_WAIT_LIMIT_NS
constexpr uint64_t kConsumerWaitLimitNs = CMR_CONSUMER_WAIT_LIMIT_NS;
#else
constexpr uint64_t kConsumerWaitLimitNs = kWaitLimitNs;
#endif

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t arrivals) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(arrivals) : "memory");
}

// Makes the initialisations above visible to the async proxy (TMA).
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Arrive and announce `bytes` of incoming TMA transactions for this phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Whether the phase of parity `parity` has completed, without waiting.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for the phase of parity `parity` to complete; false after `limit_ns`
// without it.  A limit of 0 only looks once: try_wait itself may suspend the
// thread for a while before it returns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (limit_ns == 0) return mbar_test_wait(bar, parity);
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > limit_ns) return false;
  return true;
}

// 4-D tiled load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x,
                                        int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// 4-D tiled store of one box from shared memory (bulk async-group).  Box
// elements outside the tensor are not written.
__device__ __forceinline__ void store_4d(const CUtensorMap* map, uint32_t src, int x, int y, int z,
                                         int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(map),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// An L2 policy that marks the lines an access touches as first to evict.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// load_4d / store_4d with an L2 cache policy.
__device__ __forceinline__ void load_4d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                             int x, int y, int z, int w, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
      "l"(map), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void store_4d_hint(const CUtensorMap* map, uint32_t src, int x, int y,
                                              int z, int w, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4, %5}], [%1], %6;" ::"l"(map),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w), "l"(policy)
      : "memory");
}

// 5-D tiled store of one box from shared memory (bulk async-group), plain and
// with an L2 cache policy.
__device__ __forceinline__ void store_5d(const CUtensorMap* map, uint32_t src, int x, int y, int z,
                                         int w, int v) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::"l"(
          map),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w), "r"(v)
      : "memory");
}

__device__ __forceinline__ void store_5d_hint(const CUtensorMap* map, uint32_t src, int x, int y,
                                              int z, int w, int v, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4, %5, %6}], [%1], %7;" ::"l"(map),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w), "r"(v), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Order this thread's shared-memory writes before later async-proxy reads.
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier `id` over `threads` threads (a multiple of 32).
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier that also ORs `v` over the participating threads, so that
// they all take the same branch after their bounded waits.
__device__ __forceinline__ bool named_any(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n"
      " .reg .pred q, p;\n"
      " setp.ne.u32 q, %1, 0;\n"
      " bar.red.or.pred p, %2, %3, q;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

}  // namespace tma
}  // namespace cmr
