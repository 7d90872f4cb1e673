// Shared-memory staging for the sm_100a kernels that move their inputs with
// the Tensor Memory Accelerator: 1-D bulk copies (cp.async.bulk) from this
// GPU's global memory into a ring of shared-memory stages of the CTA itself,
// completion counted in bytes on an mbarrier per stage.  No cluster multicast.
//
// Every wait is bounded (kWaitNs of %globaltimer wall time): a kernel whose
// wait runs out records an error code, stops issuing, drains the copies it has
// in flight and ends, so the host sees an error status instead of a hung GPU.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.cuh"

namespace zsm {
namespace pipe {

constexpr int kConsumerWarps = 8;                   // warps of one consumer group
constexpr int kConsumers = kConsumerWarps * 32;     // 256 threads per group, 8 elements each
constexpr int kTile = kConsumers * kVec;            // 2048 elements per tile

// G consumer groups, each with its own producer warp: G * (32 + 256) threads.
template <int G>
__host__ __device__ constexpr int tma_threads() { return G * (32 + kConsumers); }
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s per wait

static __device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

static __device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

static __device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

static __device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

static __device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

static __device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of whether the phase with the given parity has completed.
static __device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; false after `limit`
// nanoseconds of %globaltimer.  limit = 0 tests once without blocking (a
// phase not already complete counts as run out: the tests' way to make a
// bounded wait expire without stalling anything).
static __device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity,
                                                 unsigned long long limit = kWaitNs) {
  if (limit == 0) return mbar_test_wait(bar, parity);
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!mbar_try_wait(bar, parity))
    if (now_ns() - t0 > limit) return false;
  return true;
}

// A stage is refilled by bulk copies (async proxy) after its consumers'
// ordinary shared-memory reads (generic proxy) -- ordered by the empty
// barrier the producer has just waited on, which orders generic-proxy
// accesses only.  This fence orders those reads before the async-proxy
// writes that follow; without it a consumer's read still in flight when it
// released the stage could return the next tile's data.
static __device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// L2 policy for the bulk loads: every input byte is read exactly once, so it
// is marked first to evict and leaves L2 room for the write-back traffic.
static __device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 1-D bulk copy global -> this CTA's shared memory, completion on `bar`.
static __device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes, uint64_t* bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Wait for the phase with the given parity, giving up when `abort_flag` is set
// (another role of the CTA stopped) or after `limit` ns (0: one non-blocking
// test): 0 = done, 1 = timed out, 2 = aborted.
static __device__ __forceinline__ int mbar_wait_or_abort(uint64_t* bar, unsigned parity, volatile int* abort_flag,
                                                         unsigned long long limit) {
  if (limit == 0) return mbar_test_wait(bar, parity) ? 0 : 1;
  if (mbar_try_wait(bar, parity)) return 0;
  const unsigned long long t0 = now_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return 2;
    if (now_ns() - t0 > limit) return 1;
  }
  return 0;
}

// 1-D bulk copy from this CTA's shared memory to this GPU's global memory,
// tracked in the issuing thread's bulk async-group.  The shared-memory
// source must have been written before a fence.proxy.async by its writers.
static __device__ __forceinline__ void bulk_store(void* dst, const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
               "r"(bytes)
               : "memory");
}

static __device__ __forceinline__ void bulk_store(void* dst, const void* src, unsigned bytes, uint64_t policy) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes), "l"(policy)
               : "memory");
}

static __device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Until at most `Pending` of this thread's committed bulk groups still read
// their shared-memory source (the source may then be overwritten).
template <int Pending>
static __device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(Pending) : "memory");
}

// Until at most `Pending` of this thread's committed bulk groups are incomplete
// (their writes to global memory performed).
template <int Pending>
static __device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(Pending) : "memory");
}

// Plain (write-back) 16-byte stores for the consumers' outputs; measured ~1 %
// faster than streaming stores in this kernel on B200.
static __device__ __forceinline__ void st_out(uint16_t* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }
static __device__ __forceinline__ void st_out(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
static __device__ __forceinline__ void st_out(uint16_t* p, uint2 v) { *reinterpret_cast<uint2*>(p) = v; }

}  // namespace pipe
}  // namespace zsm
