// Raising a kernel's dynamic shared-memory limit once per device.
//
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) applies to the current
// device only, so a process that launches on several GPUs must raise it on
// each.  SmemAllowed remembers, per device ordinal, the largest size already
// allowed for one kernel; it is zero-initialised static storage, and threads
// that race to raise it only repeat a harmless call.  Used by the kernel
// launchers of the .cu files (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>

#include <atomic>

namespace lse_detail {

constexpr int kMaxSmemDevices = 64;

struct SmemAllowed {
  std::atomic<int> bytes[kMaxSmemDevices];
};

template <class K>
int allow_dynamic_smem(K kernel, int smem, SmemAllowed &allowed) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  const bool cached = dev >= 0 && dev < kMaxSmemDevices;
  if (cached && allowed.bytes[dev].load(std::memory_order_relaxed) >= smem) return 0;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  if (cached) {
    int cur = allowed.bytes[dev].load(std::memory_order_relaxed);
    while (cur < smem && !allowed.bytes[dev].compare_exchange_weak(cur, smem)) {
    }
  }
  return 0;
}

}  // namespace lse_detail
