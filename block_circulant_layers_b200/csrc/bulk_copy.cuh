// Bulk (TMA engine) copies between global and shared memory, and the mbarrier that
// tracks their completion, for sm_100a (PTX ISA 8.x, non-tensor cp.async.bulk; no
// cluster multicast).
//
// Every wait on an mbarrier is bounded: after about `kWaitCycles` SM cycles without
// completion the waiting thread gives up, records RDFFT_DEVICE_TIMEOUT in the module's
// error word (read and cleared by rdfft_take_device_error()) and the kernel skips its
// work instead of hanging the GPU.
#pragma once

#include <stdint.h>

#include "pdl.cuh"

namespace rdfft {

// Error word of the kernels of the translation unit that includes this header (bit 0:
// a bounded wait timed out); each such unit provides a host accessor for it.
static __device__ unsigned int g_device_error = 0;
constexpr unsigned int kDeviceTimeout = 1u;
constexpr long long kWaitCycles = 2000000000LL;     // about one second at 1.9 GHz

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* m, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(m)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive once and announce `bytes` of transactions to come.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* m, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(m)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* m, unsigned parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(m)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for phase `parity` of m; false (and the error word set) on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* m, unsigned parity,
                                                  long long limit_cycles = kWaitCycles) {
  if (mbar_try_wait(m, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(m, parity)) {
    if (clock64() - t0 > limit_cycles) {
      atomicOr(&g_device_error, kDeviceTimeout);
      return false;
    }
  }
  return true;
}

// Global -> shared bulk copy completing `bytes` transactions on m. dst, src 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes, uint64_t* m) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(m))
      : "memory");
}

// Makes this thread's generic-proxy shared-memory writes visible to bulk copies.
__device__ __forceinline__ void fence_smem_to_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared -> global bulk copy (bulk-group completion).
__device__ __forceinline__ void bulk_store(void* dst, const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_addr(src)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Waits until this thread's committed bulk stores have read their shared-memory
// sources, so the CTA may exit and its shared memory be reused. The global writes
// finish on their own; like any write of the kernel they are visible to later work
// in the stream once the kernel has completed.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

}  // namespace rdfft
